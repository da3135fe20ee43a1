// K1 router: logits in a fixed fp32 order, then top-k and routing weights.
//
// Each warp owns EPW experts and a tile of TT tokens.  Lane j accumulates, by
// fmaf in ascending h, the 8-element chunks c with c % 32 == j (16-byte,
// warp-coalesced loads of W_r; x staged in shared memory as fp32); the 32 lane
// sums are added by a xor butterfly (16, 8, 4, 2, 1) and the bias is added
// last.  That order is part of the contract: any implementation following it
// gets bit-identical logits, hence identical expert indices.
//
// The last CTA to finish a token tile (an atomic ticket per tile, reset by that
// CTA) selects the top-k of each token with one warp (descending logit, ties to
// the lower index) and writes the softmax weights.
#include "common.cuh"
#include "router_topk.cuh"

namespace moe {

constexpr int kRouterWarps = 4;
constexpr int kRouterTileMax = 8;

template <int EPW, int TT>
__global__ void __launch_bounds__(kRouterWarps * 32)
router_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ wr,
              const float* __restrict__ bias, int T, int H, int E, int k, int renorm,
              int32_t* __restrict__ idx, float* __restrict__ wout, float* __restrict__ logits,
              unsigned int* __restrict__ tile_cnt) {
    extern __shared__ float xs[];  // [TT][H] fp32
    __shared__ int s_last;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    pdl_trigger();   // the slot lookup may launch now; it waits for this grid to finish
    const int t0 = blockIdx.y * TT;
    const int nt = min(TT, T - t0);
    const int e0 = (blockIdx.x * kRouterWarps + warp) * EPW;

    // H % 256 == 0, so every lane owns exactly H / 256 chunks of a row: c = lane + 32 q.
    // They are taken kPre at a time, all loads of a batch issued before any use; the
    // first batch (the router's own weights) before waiting for the previous kernel.
    const int nper = H / 256;
    constexpr int kPre = EPW == 1 ? 8 : 4;
    uint4 pre[EPW][kPre];
    auto load_batch = [&](int q0) {
#pragma unroll
        for (int a = 0; a < EPW; a++)
#pragma unroll
            for (int q = 0; q < kPre; q++) {
                const int e = e0 + a;
                pre[a][q] = (q0 + q < nper && e < E)
                                ? __ldg(reinterpret_cast<const uint4*>(wr + size_t(e) * H) + lane + 32 * (q0 + q))
                                : make_uint4(0, 0, 0, 0);
            }
    };
    load_batch(0);
    pdl_wait();      // x (and the buffers this kernel writes) belong to earlier kernels

    for (int v = threadIdx.x; v < TT * H / 8; v += blockDim.x) {
        const int t = (v * 8) / H, h = v * 8 - t * H;
        uint4 q = make_uint4(0, 0, 0, 0);
        if (t < nt) q = *reinterpret_cast<const uint4*>(x + size_t(t0 + t) * H + h);
        const uint32_t u[4] = {q.x, q.y, q.z, q.w};
        float4* dst = reinterpret_cast<float4*>(xs + t * H + h);
        dst[0] = make_float4(__uint_as_float(u[0] << 16), __uint_as_float(u[0] & 0xFFFF0000u),
                             __uint_as_float(u[1] << 16), __uint_as_float(u[1] & 0xFFFF0000u));
        dst[1] = make_float4(__uint_as_float(u[2] << 16), __uint_as_float(u[2] & 0xFFFF0000u),
                             __uint_as_float(u[3] << 16), __uint_as_float(u[3] & 0xFFFF0000u));
    }
    __syncthreads();

    float acc[EPW][TT];
#pragma unroll
    for (int a = 0; a < EPW; a++)
#pragma unroll
        for (int t = 0; t < TT; t++) acc[a][t] = 0.0f;

    for (int q0 = 0; q0 < nper; q0 += kPre) {
        if (q0 > 0) load_batch(q0);
#pragma unroll
        for (int q = 0; q < kPre; q++) {
            if (q0 + q >= nper) break;
            const int c = lane + 32 * (q0 + q);
            float wf[EPW][8];
#pragma unroll
            for (int a = 0; a < EPW; a++) {
                const uint32_t u[4] = {pre[a][q].x, pre[a][q].y, pre[a][q].z, pre[a][q].w};
#pragma unroll
                for (int r = 0; r < 4; r++) {
                    wf[a][2 * r] = __uint_as_float(u[r] << 16);
                    wf[a][2 * r + 1] = __uint_as_float(u[r] & 0xFFFF0000u);
                }
            }
#pragma unroll
            for (int t = 0; t < TT; t++) {
                const float4 xa = *reinterpret_cast<const float4*>(xs + t * H + c * 8);
                const float4 xb = *reinterpret_cast<const float4*>(xs + t * H + c * 8 + 4);
                const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
                for (int a = 0; a < EPW; a++)
#pragma unroll
                    for (int r = 0; r < 8; r++) acc[a][t] = fmaf(xv[r], wf[a][r], acc[a][t]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < EPW; a++)
#pragma unroll
        for (int t = 0; t < TT; t++) {
            float v = acc[a][t];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) v = v + __shfl_xor_sync(0xffffffffu, v, off);
            const int e = e0 + a;
            if (lane == 0 && e < E && t < nt)
                logits[size_t(t0 + t) * E + e] = v + (bias ? bias[e] : 0.0f);
        }

    // last CTA of this token tile does the selection
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(tile_cnt + blockIdx.y, 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    __shared__ float s_l[kRouterWarps][kMaxE];
    __shared__ unsigned char s_taken[kRouterWarps][kMaxE];
    for (int t = warp; t < nt; t += kRouterWarps) {
        const float* row = logits + size_t(t0 + t) * E;
        for (int e = lane; e < E; e += 32) s_l[warp][e] = __ldcg(row + e);
        __syncwarp();
        router_topk_warp(s_l[warp], s_taken[warp], E, k, renorm, lane, idx + size_t(t0 + t) * k,
                         wout + size_t(t0 + t) * k);
    }
    if (threadIdx.x == 0) tile_cnt[blockIdx.y] = 0;
}

static size_t round_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

template <int EPW, int TT>
static cudaError_t launch_router(const uint16_t* x, const uint16_t* wr, const float* bias, int T,
                                 int H, int E, int k, int renorm, int32_t* idx, float* w,
                                 float* logits, unsigned int* cnt, cudaStream_t s) {
    const size_t smem = size_t(TT) * H * sizeof(float);
    auto kern = router_kernel<EPW, TT>;
    // the x tile is at most 200 KiB (checked by the caller); raise the limit once per device
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    dim3 grid((E + kRouterWarps * EPW - 1) / (kRouterWarps * EPW), (T + TT - 1) / TT);
    return launch_pdl(kern, grid, dim3(kRouterWarps * 32), smem, s, x, wr, bias, T, H, E, k, renorm, idx, w,
                      logits, cnt);
}

// Shared by the entry points that own their scratch differently.
int route_impl(const void* x_bf16, const void* wr_bf16, const float* bias, int T, int H, int E,
               int k, int renorm, int32_t* idx, float* w, float* logits, unsigned int* cnt,
               cudaStream_t s) {
    if (!x_bf16 || !wr_bf16 || !idx || !w || !logits || !cnt) return fail(MOE_EINVAL, "null pointer");
    if (T <= 0 || H <= 0 || H % 256 || E <= 0 || E > kMaxE || k <= 0 || k > kMaxK || k > E)
        return fail(MOE_EINVAL, "route: need T > 0, H % 256 == 0, 0 < k <= min(E, 32), E <= 1024");
    if ((reinterpret_cast<uintptr_t>(x_bf16) | reinterpret_cast<uintptr_t>(wr_bf16)) & 15)
        return fail(MOE_EINVAL, "route: x and W_r must be 16-byte aligned");
    if (size_t(kRouterTileMax) * H * sizeof(float) > 200 * 1024)
        return fail(MOE_EINVAL, "route: H too large for the shared-memory x tile");
    const uint16_t* x = (const uint16_t*)x_bf16;
    const uint16_t* wr = (const uint16_t*)wr_bf16;
    cudaError_t e;
    if (T == 1) e = launch_router<1, 1>(x, wr, bias, T, H, E, k, renorm, idx, w, logits, cnt, s);
    else if (T == 2) e = launch_router<1, 2>(x, wr, bias, T, H, E, k, renorm, idx, w, logits, cnt, s);
    else if (T <= 4) e = launch_router<1, 4>(x, wr, bias, T, H, E, k, renorm, idx, w, logits, cnt, s);
    else if (T <= 8) e = launch_router<2, 8>(x, wr, bias, T, H, E, k, renorm, idx, w, logits, cnt, s);
    else e = launch_router<4, 8>(x, wr, bias, T, H, E, k, renorm, idx, w, logits, cnt, s);
    if (e != cudaSuccess) return cuda_fail(e, "router launch");
    return MOE_OK;
}

// Load every router instantiation now (module loading may wait for the device).
int preload_router_kernels() {
    cudaFuncAttributes fa;
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, router_kernel<1, 1>));
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, router_kernel<1, 2>));
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, router_kernel<1, 4>));
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, router_kernel<2, 8>));
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, router_kernel<4, 8>));
    return MOE_OK;
}

size_t route_logits_bytes(int T, int E) { return round_up(size_t(T) * E * sizeof(float), 256); }

}  // namespace moe

using namespace moe;

extern "C" size_t moe_route_workspace_bytes(int T, int E) {
    if (T <= 0 || E <= 0) return 0;
    return route_logits_bytes(T, E) + round_up(size_t((T + kRouterTileMax - 1) / kRouterTileMax) * 4, 256);
}

extern "C" int moe_route(const void* x_bf16, const void* wr_bf16, const float* bias, int T, int H,
                         int E, int k, int renormalize, int32_t* idx, float* w, void* workspace,
                         size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < moe_route_workspace_bytes(T, E))
        return fail(MOE_EINVAL, "route: workspace missing or smaller than moe_route_workspace_bytes");
    float* logits = (float*)workspace;
    unsigned int* cnt = (unsigned int*)((char*)workspace + route_logits_bytes(T, E));
    return route_impl(x_bf16, wr_bf16, bias, T, H, E, k, renormalize, idx, w, logits, cnt,
                      (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Router without allocation.  Some callers cannot allocate device memory where
// they route: a serving loop that handed every byte of HBM to its KV cache and
// expert slots at start-up, or code that must not pay cudaMalloc's latency and
// implicit device-wide synchronisation in the middle of a decode step.  For
// them the scratch lives in this file-scope array instead of a caller
// workspace: logits of at most kNoAllocMaxLogits = T*E floats, then one counter
// per 8-token tile.  Every GPU that loads the library holds the array until the
// process exits.  All calls share it, and it keeps the last call's contents, so
// calls that overlap on the GPU race: issue them on one stream, one at a time.
#include <mutex>

namespace moe {

constexpr int kNoAllocMaxLogits = 1 << 16;   // T*E <= 65536 floats (256 KiB)
constexpr int kNoAllocMaxT = 4096;           // so at most 512 tile counters
constexpr size_t kNoAllocLogitBytes = size_t(kNoAllocMaxLogits) * sizeof(float);
constexpr size_t kNoAllocCounterBytes = size_t(kNoAllocMaxT / kRouterTileMax) * sizeof(unsigned int);

static __device__ __align__(256) unsigned char g_route_scratch[kNoAllocLogitBytes + kNoAllocCounterBytes];

// In host code g_route_scratch names a host-side stand-in, not device memory;
// the device address is fetched once per device (with that device current).
constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
static void* g_scratch_ptr[kMaxDevices] = {};

static int route_scratch(void** out) {
    int dev = -1;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_EINVAL, "route_noalloc: device ordinal out of range");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p) return cuda_fail(e, "cudaGetSymbolAddress(route scratch)");
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return MOE_OK;
}

}  // namespace moe

extern "C" int moe_route_noalloc(const void* x_bf16, const void* wr_bf16, const float* bias, int T,
                                 int H, int E, int k, int renormalize, int32_t* idx, float* w,
                                 void* stream) {
    if (T <= 0 || E <= 0 || T > kNoAllocMaxT || (long long)T * E > kNoAllocMaxLogits)
        return fail(MOE_EINVAL, "route_noalloc: needs 0 < T <= 4096 and T*E <= 65536 "
                                "(the static scratch holds 65536 logits)");
    void* base = nullptr;
    int rc = route_scratch(&base);
    if (rc) return rc;
    float* logits = (float*)base;
    unsigned int* cnt = (unsigned int*)((char*)base + kNoAllocLogitBytes);
    const int tiles = (T + kRouterTileMax - 1) / kRouterTileMax;
    // the tile counters must start at zero whatever the previous call left
    MOE_CUDA_TRY(cudaMemsetAsync(cnt, 0, size_t(tiles) * sizeof(unsigned int), (cudaStream_t)stream));
    return route_impl(x_bf16, wr_bf16, bias, T, H, E, k, renormalize, idx, w, logits, cnt,
                      (cudaStream_t)stream);
}
