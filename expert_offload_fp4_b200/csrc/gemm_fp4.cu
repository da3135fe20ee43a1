// Block-scaled NVFP4 GEMM on the 5th-generation tensor cores (tcgen05).
//
// D[M, N] (fp32) = sum_k dq(A)[m, k] * dq(B)[n, k], with A [M, K] and B [N, K]
// E2M1 codes (K-contiguous, two per byte, lower index in the low nibble) and
// E4M3 scales per 16 elements along K, both in the canonical row-major layout
// [rows, K/16].
//
// One CTA computes one 128 x 128 tile over K in steps of 256 (128 code bytes
// per row: one 128-byte swizzle row).  Warp roles:
//   warp 0  TMA producer: codes (128-byte swizzle) and canonical scale rows of
//           A and B into a ring of stages;
//   warp 2  scale arranger: rewrites each stage's canonical scales (row m holds
//           the 16 scales of its K step) into the tensor core's scale-factor
//           atoms (per 64-element K step, 512 bytes: byte 16*(m%32) + 4*(m/32) + j
//           holds the j-th 16-element scale of row m);
//   warp 1  MMA issuer: owns the TMEM allocation; copies the atoms to TMEM
//           (tcgen05.cp 32x128b.warpx4), issues 4 tcgen05.mma kind::mxf4nvf4
//           (M=128, N=128, K=64 each) per stage, and commits to free the stage;
//   warps 4-7 epilogue: TMEM -> registers (tcgen05.ld 32x32b) -> global fp32.
// All waits are bounded; a timeout sets bit 16 of *status and the CTA drains.
#include "tcgen05.cuh"

namespace moe {

constexpr int kBM = 128, kBN = 128;
constexpr int kKT = 256;                    // K elements per stage (128 code bytes)
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 256;
constexpr uint32_t kTmemCols = 256;         // 128 accumulator + 4 stages x 32 scale columns

struct GemmSmem {                           // offsets from the 1024-aligned base
    static constexpr int a_codes = 0;                         // [stage][128 rows][128 B]
    static constexpr int b_codes = a_codes + kGemmStages * 16384;
    static constexpr int a_sf = b_codes + kGemmStages * 16384;  // [stage][128 rows][16 B] canonical
    static constexpr int b_sf = a_sf + kGemmStages * 2048;
    static constexpr int a_atom = b_sf + kGemmStages * 2048;    // [stage][4 steps][512 B]
    static constexpr int b_atom = a_atom + kGemmStages * 2048;
    static constexpr int bars = b_atom + kGemmStages * 2048;    // full, sfready, empty [stage], acc
    static constexpr int tmem_slot = bars + (3 * kGemmStages + 1) * 8;
    static constexpr int total = tmem_slot + 16;
};

__device__ __forceinline__ void arrange_sf(const uint8_t* canon, uint8_t* atom, int lane) {
    // lane handles rows lane, lane+32, lane+64, lane+96; each row's 16 bytes are
    // the 4 scales of each of the 4 K steps
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const int m = lane + 32 * q;
        const uint4 v = *reinterpret_cast<const uint4*>(canon + 16 * m);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int s = 0; s < 4; s++)
            *reinterpret_cast<uint32_t*>(atom + 512 * s + 16 * lane + 4 * q) = w[s];
    }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                  const __grid_constant__ CUtensorMap map_sfa, const __grid_constant__ CUtensorMap map_sfb,
                  int M, int N, int K, float* __restrict__ D, int* status, unsigned long long limit_ns) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + GemmSmem::bars);
    uint64_t* sfready = full + kGemmStages;
    uint64_t* empty = sfready + kGemmStages;
    uint64_t* accf = empty + kGemmStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + GemmSmem::tmem_slot);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;
    const int KT = K / kKT;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGemmStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&sfready[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
        fence_mbar_init();
        prefetch_tmap(&map_a);
        prefetch_tmap(&map_b);
        prefetch_tmap(&map_sfa);
        prefetch_tmap(&map_sfb);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            for (int kt = 0; kt < KT; kt++) {
                const int s = kt % kGemmStages, r = kt / kGemmStages;
                if (!mbar_wait(&empty[s], (r & 1) ^ 1, limit_ns)) atomicOr(status, 1 << 16);
                mbar_arrive_expect_tx(&full[s], 16384 * 2 + 2048 * 2);
                tma_load_2d(sm + GemmSmem::a_codes + s * 16384, &map_a, kt * 128, m0, &full[s]);
                tma_load_2d(sm + GemmSmem::b_codes + s * 16384, &map_b, kt * 128, n0, &full[s]);
                tma_load_2d(sm + GemmSmem::a_sf + s * 2048, &map_sfa, kt * 16, m0, &full[s]);
                tma_load_2d(sm + GemmSmem::b_sf + s * 2048, &map_sfb, kt * 16, n0, &full[s]);
            }
        }
    } else if (warp == 2) {
        for (int kt = 0; kt < KT; kt++) {
            const int s = kt % kGemmStages, r = kt / kGemmStages;
            if (!mbar_wait(&full[s], r & 1, limit_ns) && lane == 0) atomicOr(status, 1 << 16);
            arrange_sf(sm + GemmSmem::a_sf + s * 2048, sm + GemmSmem::a_atom + s * 2048, lane);
            arrange_sf(sm + GemmSmem::b_sf + s * 2048, sm + GemmSmem::b_atom + s * 2048, lane);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sfready[s]);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_fp4(kBM, kBN, false);
            for (int kt = 0; kt < KT; kt++) {
                const int s = kt % kGemmStages, r = kt / kGemmStages;
                if (!mbar_wait(&sfready[s], r & 1, limit_ns)) atomicOr(status, 1 << 16);
                tc_fence_after();
                const uint32_t sfa = tbase + 128 + s * 32, sfb = sfa + 16;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    tmem_cp_sf_atom(sfa + 4 * i, smem_desc(sm + GemmSmem::a_atom + s * 2048 + 512 * i, 16, 128, 0));
                    tmem_cp_sf_atom(sfb + 4 * i, smem_desc(sm + GemmSmem::b_atom + s * 2048 + 512 * i, 16, 128, 0));
                }
                const uint64_t ad = smem_desc(sm + GemmSmem::a_codes + s * 16384, 16, 1024, 2);
                const uint64_t bd = smem_desc(sm + GemmSmem::b_codes + s * 16384, 16, 1024, 2);
#pragma unroll
                for (int i = 0; i < 4; i++)   // K = 64 elements = 32 bytes per MMA
                    mma_nvfp4(tbase, ad + 2 * i, bd + 2 * i, idesc, sfa + 4 * i, sfb + 4 * i,
                              (kt > 0 || i > 0) ? 1u : 0u);
                tc_commit(&empty[s]);
            }
            tc_commit(accf);
        }
        __syncwarp();
    } else if (warp >= 4) {
        const int e = warp - 4;
        if (!mbar_wait(accf, 0, limit_ns) && lane == 0) atomicOr(status, 1 << 16);
        tc_fence_after();
        const int m = m0 + 32 * e + lane;
#pragma unroll
        for (int c = 0; c < kBN / 32; c++) {
            uint32_t r[32];
            tmem_ld_32x32(tbase + ((uint32_t)(32 * e) << 16) + 32 * c, r);
            if (m < M) {
                float4* dst = reinterpret_cast<float4*>(D + (size_t)m * N + n0 + 32 * c);
#pragma unroll
                for (int q = 0; q < 8; q++)
                    dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                         __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
            }
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------- host helpers

typedef CUresult (*encode_tiled_fn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static encode_tiled_fn encode_fn() {
    static encode_tiled_fn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (encode_tiled_fn)p;
    }
    return fn;
}

// A 2-D byte tensor [rows, row_bytes] (row pitch `pitch` bytes) with a box of
// box_rows x box_bytes; swizzle128 for FP4 code tiles.
int make_tmap_2d(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t pitch,
                 uint32_t box_bytes, uint32_t box_rows, bool swizzle128) {
    encode_tiled_fn fn = encode_fn();
    if (!fn) return fail(MOE_ECUDA, "cuTensorMapEncodeTiled entry point not available");
    const cuuint64_t dims[2] = {row_bytes, rows};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_bytes, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_EINVAL, "cuTensorMapEncodeTiled rejected a tensor map");
    return MOE_OK;
}

int preload_gemm_kernels() {
    cudaFuncAttributes fa;
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, nvfp4_gemm_kernel));
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" int moe_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                              const uint8_t* b_scales, int M, int N, int K, float* D, int* status,
                              void* stream) {
    if (!a_codes || !a_scales || !b_codes || !b_scales || !D || !status) return fail(MOE_EINVAL, "null argument");
    if (M <= 0 || N <= 0 || K <= 0 || M % kBM || N % kBN || K % kKT)
        return fail(MOE_EINVAL, "nvfp4 gemm: M and N must be multiples of 128, K of 256");
    if (((uintptr_t)a_codes | (uintptr_t)b_codes | (uintptr_t)a_scales | (uintptr_t)b_scales) & 15)
        return fail(MOE_EINVAL, "nvfp4 gemm: operands must be 16-byte aligned");
    CUtensorMap ma, mb, msa, msb;
    int rc;
    if ((rc = make_tmap_2d(&ma, a_codes, K / 2, M, K / 2, 128, 128, true))) return rc;
    if ((rc = make_tmap_2d(&mb, b_codes, K / 2, N, K / 2, 128, 128, true))) return rc;
    if ((rc = make_tmap_2d(&msa, a_scales, K / 16, M, K / 16, 16, 128, false))) return rc;
    if ((rc = make_tmap_2d(&msb, b_scales, K / 16, N, K / 16, 16, 128, false))) return rc;
    const int smem = GemmSmem::total + 1024;
    // the shared-memory limit is a per-device setting: raise it once per device
    static bool attr_done[64] = {};
    int dev = 0;
    MOE_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        if (dev >= 0 && dev < 64) attr_done[dev] = true;
    }
    dim3 grid(N / kBN, M / kBM);
    nvfp4_gemm_kernel<<<grid, kGemmThreads, smem, (cudaStream_t)stream>>>(ma, mb, msa, msb, M, N, K, D, status,
                                                                          2000000000ull);
    MOE_CUDA_TRY(cudaGetLastError());
    return MOE_OK;
}
