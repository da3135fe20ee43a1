// Miss streaming by the SMs: one expert block read from mapped pinned host
// memory over PCIe and written to its HBM slot by a grid of small CTAs on the
// copy stream ("游戏电脑如何跑动2840亿参数大模型": missing weights cross PCIe
// while the GPU computes on the resident ones).  Each thread keeps four
// 16-byte loads in flight; a warp's loads cover 512 contiguous bytes.
#include "common.cuh"

namespace moe {

constexpr int kPullThreads = 128;   // one warp per SM sub-partition
constexpr int kPullUnroll = 4;

__global__ void __launch_bounds__(kPullThreads) pull_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                            size_t n16) {
    const size_t T = (size_t)gridDim.x * blockDim.x;
    for (size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n16; i0 += kPullUnroll * T) {
        uint4 v[kPullUnroll];
#pragma unroll
        for (int u = 0; u < kPullUnroll; u++) {
            const size_t i = i0 + u * T;
            if (i < n16) v[u] = src[i];
        }
#pragma unroll
        for (int u = 0; u < kPullUnroll; u++) {
            const size_t i = i0 + u * T;
            if (i < n16) dst[i] = v[u];
        }
    }
}

// Enqueue the copy of `bytes` (a multiple of 16; both addresses 16-byte aligned).
cudaError_t launch_pull(const uint8_t* src_d, uint8_t* dst, size_t bytes, int num_sms, cudaStream_t s) {
    const size_t n16 = bytes / 16;
    const size_t per_pass = (size_t)kPullThreads * kPullUnroll;
    const int grid = (int)std::max<size_t>(1, std::min<size_t>((size_t)num_sms, (n16 + per_pass - 1) / per_pass));
    pull_kernel<<<grid, kPullThreads, 0, s>>>(reinterpret_cast<const uint4*>(src_d), reinterpret_cast<uint4*>(dst),
                                              n16);
    return cudaGetLastError();
}

int preload_pull_kernels() {
    cudaFuncAttributes fa;
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, pull_kernel));
    // the largest shared-memory carve-out, the one the decode FFN runs with: a
    // CTA of this kernel must fit on an SM beside an FFN CTA that waits for it
    MOE_CUDA_TRY(cudaFuncSetAttribute(pull_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                      cudaSharedmemCarveoutMaxShared));
    return MOE_OK;
}

}  // namespace moe
