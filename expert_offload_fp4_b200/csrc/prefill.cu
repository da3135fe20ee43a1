// Prefill expert FFN (K6 + K7): activation quantisation and expert grouping,
// then two grouped block-scaled NVFP4 GEMMs on tcgen05 with fused epilogues.
//
//   plan      one CTA: tokens per expert, 128-padded row offsets, M-tile table,
//             the slot of every chosen expert;
//   quant     one warp per token: x_t -> NVFP4 with the per-token FP32 scale
//             S_x = amax(x_t)/(6*448), E4M3 per 16 (round-to-nearest-even,
//             saturating), codes E2M1; the row is written once per chosen expert
//             into that expert's row block (A operand of GEMM1);
//   GEMM1     per (M tile, 64 columns of I): A = quantised tokens, B = 64 gate
//             rows + the same 64 up rows of the expert (TMA from its slot);
//             epilogue h = silu(S_x S_g acc_g) * (S_x S_u acc_u), quantised to
//             NVFP4 with tensor scale 1 (A operand of GEMM2);
//   GEMM2     per (M tile, 128 columns of H): A = quantised h, B = down rows;
//             epilogue y[t, :] += w[t, j] * S_d * acc (fp32 vector reductions).
// moe_combine(y, T, 1, H) then rounds y to bf16.  The mainloop is the one of
// moe_nvfp4_gemm (TMA ring, scale-atom rearrangement, tcgen05.cp + mma), made
// persistent with two TMEM accumulators (see grouped_gemm_kernel).
#include "tcgen05.cuh"

namespace moe {

int make_tmap_2d(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t pitch,
                 uint32_t box_bytes, uint32_t box_rows, bool swizzle128);

// ---------------------------------------------------------------- NVFP4 quantiser

// E4M3 code (round-to-nearest-even, saturating at 448) of a ratio >= 0; 0 when
// the ratio is 0 or not a number.
__device__ __forceinline__ uint32_t e4m3_code(float r) {
    if (!(r > 0.0f)) return 0u;
    uint16_t v;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(v) : "f"(r));
    return v & 0xFFu;
}

__device__ __forceinline__ float e4m3_value(uint32_t b) {
    uint32_t h2;
    asm("{ .reg .b16 lo; cvt.u16.u32 lo, %1; cvt.rn.f16x2.e4m3x2 %0, lo; }" : "=r"(h2) : "r"(b));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

// two values -> one byte of E2M1 codes (lo -> low nibble), round-to-nearest-even, saturating
__device__ __forceinline__ uint32_t e2m1_pair(float lo, float hi) {
    uint32_t b;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }" : "=r"(b) : "f"(hi), "f"(lo));
    return b;
}

// h's block quantiser in the gate/up epilogue: the same steps with a reciprocal
// multiply (h is re-rounded to FP4, so the last bit of the quotient is immaterial).
__device__ __forceinline__ void quant_block16_fast(const float (&v)[16], uint32_t (&codes)[2], uint32_t& scale) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) amax = fmaxf(amax, fabsf(v[i]));
    const uint32_t sc = e4m3_code(amax * (1.0f / 6.0f));
    const float q = e4m3_value(sc);
    codes[0] = codes[1] = 0u;
    if (q != 0.0f) {
        const float rq = __frcp_rn(q);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            codes[0] |= e2m1_pair(v[i] * rq, v[i + 1] * rq) << (4 * i);
            codes[1] |= e2m1_pair(v[8 + i] * rq, v[8 + i + 1] * rq) << (4 * i);
        }
    }
    scale = sc;
}

// One 16-element block: scale s = E4M3(amax / (6 S)), q = e4m3(s) * S,
// codes E2M1(v / q) (all zero when q == 0).  The fp32 operations are the ones
// the CPU reference performs, in the same order.
__device__ __forceinline__ void quant_block16(const float (&v)[16], float S, uint32_t (&codes)[2], uint32_t& scale) {
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i++) amax = fmaxf(amax, fabsf(v[i]));
    const float denom = 6.0f * S;
    const uint32_t sc = e4m3_code(amax / denom);
    const float q = e4m3_value(sc) * S;
    codes[0] = codes[1] = 0u;
    if (q != 0.0f) {
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            codes[0] |= e2m1_pair(v[i] / q, v[i + 1] / q) << (4 * i);
            codes[1] |= e2m1_pair(v[8 + i] / q, v[8 + i + 1] / q) << (4 * i);
        }
    }
    scale = sc;
}

// ---------------------------------------------------------------- plan

struct PrefillWs {              // pointers into the caller's workspace
    int* cnt;                   // [E] tokens per expert
    int* row_off;               // [E] first row of the expert's block (multiple of 128)
    int* cursor;                // [E] rows handed out so far
    int* slot_e;                // [E] slot holding the expert, -1 if unused
    int* n_mtiles;              // [1]
    int* tile_expert;           // [MT] expert of each 128-row tile
    int* tile_row0;             // [MT]
    int* perm_tok;              // [R] token of each row, -1 for padding
    int* perm_rank;             // [R]
    float* perm_sx;             // [R] per-token activation scale
    uint8_t* xq;                // [R][H/2]
    uint8_t* xsf;               // [R][H/16]
    uint8_t* hq;                // [R][I/2]
    uint8_t* hsf;               // [R][I/16]
    int R, MT;
};

__global__ void __launch_bounds__(1024) prefill_plan_kernel(const int32_t* __restrict__ idx,
                                                           const int32_t* __restrict__ slot_of, int n, int E,
                                                           PrefillWs ws, int* status) {
    __shared__ int s_cnt[kMaxE];
    __shared__ int s_tiles[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        s_cnt[e] = 0;
        ws.slot_e[e] = -1;
        ws.cursor[e] = 0;
    }
    __syncthreads();
    // eight entries per thread per round, their loads issued before any is used
    for (int i0 = threadIdx.x; i0 < n; i0 += 8 * blockDim.x) {
        int ev[8];
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int i = i0 + u * blockDim.x;
            ev[u] = i < n ? idx[i] : -2;
        }
#pragma unroll
        for (int u = 0; u < 8; u++) {
            const int e = ev[u];
            if (e == -2) continue;
            if (e < 0 || e >= E) {
                atomicOr(status, MOE_STATUS_BAD_EXPERT);
                continue;
            }
            // every entry of an expert names the same slot: the first one records it
            if (atomicAdd(&s_cnt[e], 1) == 0) ws.slot_e[e] = slot_of[i0 + u * blockDim.x];
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int row = 0, mt = 0;
        for (int e = 0; e < E; e++) {
            const int c = s_cnt[e];
            ws.cnt[e] = c;
            ws.row_off[e] = row;
            const int tiles = (c + 127) / 128;
            s_tiles[e] = mt;
            row += tiles * 128;
            mt += tiles;
        }
        *ws.n_mtiles = mt;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int tiles = (s_cnt[e] + 127) / 128;
        for (int t = 0; t < tiles; t++) {
            ws.tile_expert[s_tiles[e] + t] = e;
            ws.tile_row0[s_tiles[e] + t] = ws.row_off[e] + 128 * t;
        }
    }
    __syncthreads();
    // rows of an expert's last tile past its count are padding (no token)
    for (int i = threadIdx.x; i < E * 128; i += blockDim.x) {
        const int e = i >> 7, r = i & 127, c = s_cnt[e];
        if (r < (c + 127) / 128 * 128 - c) ws.perm_tok[128 * s_tiles[e] + c + r] = -1;
    }
}

// ---------------------------------------------------------------- quantise + scatter

__global__ void __launch_bounds__(256) prefill_quant_kernel(const uint16_t* __restrict__ x, int T, int H, int k,
                                                           int E, const int32_t* __restrict__ idx, PrefillWs ws,
                                                           uint8_t* __restrict__ out_codes,
                                                           uint8_t* __restrict__ out_scales,
                                                           float* __restrict__ out_sx) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= T) return;
    const int t = warp;
    const uint16_t* xr = x + (size_t)t * H;
    float amax = 0.0f;
    // H / 256 (<= 16 for H <= 4096) 16-byte loads per lane, four issued at a time
    for (int h0 = lane * 8; h0 < H; h0 += 4 * 256) {
        uint4 q[4];
#pragma unroll
        for (int u = 0; u < 4; u++) q[u] = h0 + u * 256 < H ? *reinterpret_cast<const uint4*>(xr + h0 + u * 256)
                                                            : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const uint32_t w4[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
            for (int i = 0; i < 4; i++)
                amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w4[i] << 16)), fabsf(__uint_as_float(w4[i] & 0xFFFF0000u))));
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float S = amax / 2688.0f;
    int rows[kMaxK];
    if (idx) {
        // lane j claims the row of rank j (the k claims run in parallel)
        int r = -1;
        if (lane < k) {
            const int e = idx[t * k + lane];
            if (e >= 0 && e < E) {              // invalid ids are reported by the planner
                const int pos = atomicAdd(ws.cursor + e, 1);
                r = ws.row_off[e] + pos;
                ws.perm_tok[r] = t;
                ws.perm_rank[r] = lane;
                ws.perm_sx[r] = S;
            }
        }
        for (int j = 0; j < k; j++) rows[j] = __shfl_sync(0xffffffffu, r, j);
    }
    // 16-element blocks, lane-strided
    for (int b = lane; b < H / 16; b += 32) {
        const uint4 q0 = *reinterpret_cast<const uint4*>(xr + 16 * b);
        const uint4 q1 = *reinterpret_cast<const uint4*>(xr + 16 * b + 8);
        const uint32_t u[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        float v[16];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            v[2 * i] = __uint_as_float(u[i] << 16);
            v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
        }
        uint32_t codes[2], sc;
        quant_block16(v, S, codes, sc);
        if (idx) {
            for (int j = 0; j < k; j++) {
                if (rows[j] < 0) continue;
                *reinterpret_cast<uint2*>(ws.xq + (size_t)rows[j] * (H / 2) + 8 * b) = make_uint2(codes[0], codes[1]);
                ws.xsf[(size_t)rows[j] * (H / 16) + b] = (uint8_t)sc;
            }
        } else {
            *reinterpret_cast<uint2*>(out_codes + (size_t)t * (H / 2) + 8 * b) = make_uint2(codes[0], codes[1]);
            out_scales[(size_t)t * (H / 16) + b] = (uint8_t)sc;
        }
    }
    if (!idx && lane == 0) out_sx[t] = S;
}

// ---------------------------------------------------------------- grouped GEMMs

constexpr int kPStages = 5;
constexpr int kPThreads = 256;
constexpr uint32_t kPTmemCols = 512;        // 2 accumulators x 128 + 5 stages x 32 scale columns

struct PSmem {
    static constexpr int a_codes = 0;
    static constexpr int b_codes = a_codes + kPStages * 16384;
    static constexpr int a_sf = b_codes + kPStages * 16384;
    static constexpr int b_sf = a_sf + kPStages * 2048;
    static constexpr int a_atom = b_sf + kPStages * 2048;
    static constexpr int b_atom = a_atom + kPStages * 2048;
    static constexpr int bars = b_atom + kPStages * 2048;       // full, sfready, empty [stage]; accf, acce [2]
    static constexpr int tmem_slot = bars + (3 * kPStages + 4) * 8;
    static constexpr int total = tmem_slot + 16;
};

// 128 rows x 16 scale bytes (row m: the 4 scales of each of the stage's four K=64
// blocks) -> four 512-byte scale-factor atoms (atom s, 16-byte row r: the block-s
// scales of rows r, r+32, r+64, r+96).  One warp; 16-byte loads and stores, no
// bank conflicts.
__device__ __forceinline__ void p_arrange_sf(const uint8_t* canon, uint8_t* atom, int lane) {
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; q++) v[q] = *reinterpret_cast<const uint4*>(canon + 16 * (lane + 32 * q));
    *reinterpret_cast<uint4*>(atom + 16 * lane) = make_uint4(v[0].x, v[1].x, v[2].x, v[3].x);
    *reinterpret_cast<uint4*>(atom + 512 + 16 * lane) = make_uint4(v[0].y, v[1].y, v[2].y, v[3].y);
    *reinterpret_cast<uint4*>(atom + 1024 + 16 * lane) = make_uint4(v[0].z, v[1].z, v[2].z, v[3].z);
    *reinterpret_cast<uint4*>(atom + 1536 + 16 * lane) = make_uint4(v[0].w, v[1].w, v[2].w, v[3].w);
}

struct GemmArgs {
    PrefillWs ws;
    const float* tscale;        // [L*E*3]
    const float* w;             // [T*k]
    float* y;                   // y_part [T, k, H] fp32: one row per (token, rank)
    int* status;
    int layer, E, k, H, I, NT;  // NT: N tiles per M tile
    long long b_gate_row, b_up_row, b_gsf_row, b_usf_row;  // row offsets inside a slot (GEMM1)
    long long b_rows_per_slot, b_sf_rows_per_slot;
    long long d_row, d_sf_row;                             // GEMM2
    unsigned long long limit_ns;
};

// Persistent, warp-specialised grouped GEMM over the (M tile, N tile) list of
// this call; CTA c takes tiles c, c + grid, ...  Warp 0 streams every tile's K
// steps through the stage ring without pausing between tiles; warps 2 and 3 turn
// the A and B scale rows into scale-factor atoms; warp 1 issues the MMAs into one of two
// TMEM accumulators, so warps 4-7 drain tile i while tile i+1 is multiplied.
// MODE 1: gate/up with the SiLU * up + NVFP4 epilogue; MODE 2: down with the
// routing weight, each row stored to its (token, rank) row of y_part.
template <int MODE>
__global__ void __launch_bounds__(kPThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_asf,
                    const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_bsf,
                    const GemmArgs g) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + PSmem::bars);
    uint64_t* sfready = full + kPStages;
    uint64_t* empty = sfready + kPStages;
    uint64_t* accf = empty + kPStages;     // [2]
    uint64_t* acce = accf + 2;             // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + PSmem::tmem_slot);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = *g.ws.n_mtiles * g.NT;
    const int KT = (MODE == 1 ? g.H : g.I) / 256;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&sfready[s], 2);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&accf[0], 1);
        mbar_init(&accf[1], 1);
        mbar_init(&acce[0], 4);
        mbar_init(&acce[1], 4);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, kPTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
                const int mt = tile / g.NT, nt = tile % g.NT;
                const int e = g.ws.tile_expert[mt], row0 = g.ws.tile_row0[mt];
                const long long slot = g.ws.slot_e[e];
                const long long sbase = slot * g.b_rows_per_slot, sfbase = slot * g.b_sf_rows_per_slot;
                for (int kt = 0; kt < KT; kt++, it++) {
                    const int s = it % kPStages, r = it / kPStages;
                    if (!mbar_wait(&empty[s], (r & 1) ^ 1, g.limit_ns)) atomicOr(g.status, 1 << 16);
                    mbar_arrive_expect_tx(&full[s], 16384 * 2 + 2048 * 2);
                    uint8_t* bc = sm + PSmem::b_codes + s * 16384;
                    uint8_t* bs = sm + PSmem::b_sf + s * 2048;
                    tma_load_2d(sm + PSmem::a_codes + s * 16384, &map_a, kt * 128, row0, &full[s]);
                    tma_load_2d(sm + PSmem::a_sf + s * 2048, &map_asf, kt * 16, row0, &full[s]);
                    if (MODE == 1) {
                        const int i0 = nt * 64;
                        tma_load_2d(bc, &map_b, kt * 128, (int)(sbase + g.b_gate_row + i0), &full[s]);
                        tma_load_2d(bc + 8192, &map_b, kt * 128, (int)(sbase + g.b_up_row + i0), &full[s]);
                        tma_load_2d(bs, &map_bsf, kt * 16, (int)(sfbase + g.b_gsf_row + i0), &full[s]);
                        tma_load_2d(bs + 1024, &map_bsf, kt * 16, (int)(sfbase + g.b_usf_row + i0), &full[s]);
                    } else {
                        const int n0 = nt * 128;
                        tma_load_2d(bc, &map_b, kt * 128, (int)(sbase + g.d_row + n0), &full[s]);
                        tma_load_2d(bs, &map_bsf, kt * 16, (int)(sfbase + g.d_sf_row + n0), &full[s]);
                    }
                }
            }
        }
    } else if (warp == 2 || warp == 3) {
        // warp 2 arranges the A scales, warp 3 the B scales of every stage, and
        // copies them into the stage's TMEM scale columns itself; the commit
        // arrives on sfready once the copies are done, so the MMA warp issues
        // only the MMAs
        const int off_sf = warp == 2 ? PSmem::a_sf : PSmem::b_sf;
        const int off_atom = warp == 2 ? PSmem::a_atom : PSmem::b_atom;
        const uint32_t col = warp == 2 ? 0u : 16u;
        int it = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            for (int kt = 0; kt < KT; kt++, it++) {
                const int s = it % kPStages, r = it / kPStages;
                if (!mbar_wait(&full[s], r & 1, g.limit_ns) && lane == 0) atomicOr(g.status, 1 << 16);
                p_arrange_sf(sm + off_sf + s * 2048, sm + off_atom + s * 2048, lane);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    // the stage's previous MMAs (which read these columns) completed
                    // before its loads were reissued, which the full wait above saw
                    tc_fence_after();
                    const uint32_t sf = tbase + 256 + s * 32 + col;
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        tmem_cp_sf_atom(sf + 4 * i, smem_desc(sm + off_atom + s * 2048 + 512 * i, 16, 128, 0));
                    tc_commit(&sfready[s]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_fp4(128, 128, false);
            int it = 0, tc = 0;
            for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, tc++) {
                const int a = tc & 1, ra = tc >> 1;
                if (!mbar_wait(&acce[a], (ra & 1) ^ 1, g.limit_ns)) atomicOr(g.status, 1 << 16);
                tc_fence_after();
                const uint32_t acc = tbase + 128 * a;
                for (int kt = 0; kt < KT; kt++, it++) {
                    const int s = it % kPStages, r = it / kPStages;
                    if (!mbar_wait(&sfready[s], r & 1, g.limit_ns)) atomicOr(g.status, 1 << 16);
                    tc_fence_after();
                    const uint32_t sfa = tbase + 256 + s * 32, sfb = sfa + 16;
                    const uint64_t ad = smem_desc(sm + PSmem::a_codes + s * 16384, 16, 1024, 2);
                    const uint64_t bd = smem_desc(sm + PSmem::b_codes + s * 16384, 16, 1024, 2);
#pragma unroll
                    for (int i = 0; i < 4; i++)
                        mma_nvfp4(acc, ad + 2 * i, bd + 2 * i, idesc, sfa + 4 * i, sfb + 4 * i,
                                  (kt > 0 || i > 0) ? 1u : 0u);
                    tc_commit(&empty[s]);
                }
                tc_commit(&accf[a]);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        const int q4 = warp - 4;
        int tc = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, tc++) {
            const int a = tc & 1, ra = tc >> 1;
            const int mt = tile / g.NT, nt = tile % g.NT;
            const int e = g.ws.tile_expert[mt], row0 = g.ws.tile_row0[mt];
            if (!mbar_wait(&accf[a], ra & 1, g.limit_ns) && lane == 0) atomicOr(g.status, 1 << 16);
            tc_fence_after();
            const int row = row0 + 32 * q4 + lane;
            const int tok = g.ws.perm_tok[row];
            const uint32_t lane_base = tbase + 128 * a + ((uint32_t)(32 * q4) << 16);
            const float* ts = g.tscale + ((size_t)g.layer * g.E + e) * 3;
            if (MODE == 1) {
                const float sx = tok >= 0 ? g.ws.perm_sx[row] : 0.0f;
                const float cg = sx * ts[0], cu = sx * ts[1];
                for (int half = 0; half < 2; half++) {
                    uint32_t rg[32], ru[32];
                    tmem_ld_32x32(lane_base + 32 * half, rg);
                    tmem_ld_32x32(lane_base + 64 + 32 * half, ru);
                    if (tok >= 0) {
                        // h for 32 columns of I, then two NVFP4 blocks with tensor scale 1
                        const int i0 = nt * 64 + 32 * half;
#pragma unroll
                        for (int b = 0; b < 2; b++) {
                            float hv[16];
#pragma unroll
                            for (int c = 0; c < 16; c++) {
                                const float gv = __uint_as_float(rg[16 * b + c]) * cg;
                                const float uv = __uint_as_float(ru[16 * b + c]) * cu;
                                hv[c] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
                            }
                            uint32_t codes[2], sc;
                            quant_block16_fast(hv, codes, sc);
                            *reinterpret_cast<uint2*>(g.ws.hq + (size_t)row * (g.I / 2) + (i0 + 16 * b) / 2) =
                                make_uint2(codes[0], codes[1]);
                            g.ws.hsf[(size_t)row * (g.I / 16) + (i0 + 16 * b) / 16] = (uint8_t)sc;
                        }
                    }
                }
            } else {
                const int n0 = nt * 128;
                float coef = 0.0f;
                float* dst = nullptr;
                if (tok >= 0) {
                    const int j = g.ws.perm_rank[row];
                    coef = g.w[tok * g.k + j] * ts[2];
                    dst = g.y + ((size_t)tok * g.k + j) * g.H + n0;
                }
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    uint32_t r[32];
                    tmem_ld_32x32(lane_base + 32 * c, r);
                    if (tok >= 0) {
#pragma unroll
                        for (int q = 0; q < 8; q++)
                            *reinterpret_cast<float4*>(dst + 32 * c + 4 * q) =
                                make_float4(coef * __uint_as_float(r[4 * q]), coef * __uint_as_float(r[4 * q + 1]),
                                            coef * __uint_as_float(r[4 * q + 2]), coef * __uint_as_float(r[4 * q + 3]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[a]);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kPTmemCols);
    }
}

static size_t al256(size_t n) { return (n + 255) & ~size_t(255); }

struct PrefillLayout {
    size_t off[14];
    size_t bytes;
    int R, MT;
};

static PrefillLayout prefill_layout(int T, int k, int E, int H, int I) {
    PrefillLayout L{};
    const int n = T * k;
    const int used = n < E ? n : E;
    L.R = ((n + 127) / 128 + used) * 128;
    L.MT = L.R / 128;
    const size_t sz[14] = {size_t(E) * 4, size_t(E) * 4, size_t(E) * 4, size_t(E) * 4, 4, size_t(L.MT) * 4,
                           size_t(L.MT) * 4, size_t(L.R) * 4, size_t(L.R) * 4, size_t(L.R) * 4,
                           size_t(L.R) * H / 2, size_t(L.R) * H / 16, size_t(L.R) * I / 2, size_t(L.R) * I / 16};
    size_t o = 0;
    for (int i = 0; i < 14; i++) {
        L.off[i] = o;
        o += al256(sz[i]);
    }
    L.bytes = o;
    return L;
}

int preload_prefill_kernels() {
    cudaFuncAttributes fa;
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, prefill_plan_kernel));
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, prefill_quant_kernel));
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, grouped_gemm_kernel<1>));
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, grouped_gemm_kernel<2>));
    // on the pool's device (current while the pool is created)
    const int smem = PSmem::total + 1024;
    MOE_CUDA_TRY(cudaFuncSetAttribute(grouped_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    MOE_CUDA_TRY(cudaFuncSetAttribute(grouped_gemm_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_prefill_workspace_bytes(const moe_pool* p, int T) {
    if (!p || T <= 0) return 0;
    const moe_config& c = p->cfg;
    return prefill_layout(T, c.k, c.E, c.H, c.I).bytes;
}

extern "C" int moe_nvfp4_quantize(const void* x_bf16, int T, int H, uint8_t* codes, uint8_t* scales, float* sx,
                                  void* stream) {
    if (!x_bf16 || !codes || !scales || !sx) return fail(MOE_EINVAL, "null argument");
    if (T <= 0 || H <= 0 || H % 256) return fail(MOE_EINVAL, "quantize: T > 0 and H % 256 == 0");
    PrefillWs ws{};
    const int blocks = (T * 32 + 255) / 256;
    prefill_quant_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>((const uint16_t*)x_bf16, T, H, 0, 0, nullptr, ws,
                                                                   codes, scales, sx);
    MOE_CUDA_TRY(cudaGetLastError());
    return MOE_OK;
}

extern "C" int moe_prefill_ffn(moe_pool* p, int layer, const void* x_bf16, int T, const int32_t* idx,
                               const float* w, const int32_t* slot_of, float* y, void* workspace,
                               size_t workspace_bytes, int* status, void* stream) {
    if (!p || !x_bf16 || !idx || !w || !slot_of || !y || !workspace || !status)
        return fail(MOE_EINVAL, "null argument");
    const moe_config& c = p->cfg;
    if (layer < 0 || layer >= c.L) return fail(MOE_EBOUNDS, "layer outside the pool");
    if (c.fmt != MOE_NVFP4) return fail(MOE_EINVAL, "prefill: NVFP4 experts only");
    if (T <= 0 || c.H % 256 || c.I % 256) return fail(MOE_EINVAL, "prefill: H and I multiples of 256");
    const PrefillLayout PL = prefill_layout(T, c.k, c.E, c.H, c.I);
    if (workspace_bytes < PL.bytes) return fail(MOE_EINVAL, "prefill: workspace smaller than moe_prefill_workspace_bytes");
    const BlockLayout& B = p->lay;
    const size_t gr = c.H / 2, gs = c.H / 16, dr = c.I / 2, ds = c.I / 16;
    // the pool-wide tensor maps index a slot's rows by (slot * rows_per_slot + tensor row)
    if (B.bytes % gr || B.bytes % gs || B.bytes % dr || B.bytes % ds || B.off[0] % gr || B.off[2] % gr ||
        B.off[1] % gs || B.off[3] % gs || B.off[4] % dr || B.off[5] % ds)
        return fail(MOE_EINVAL, "prefill: expert block layout not divisible by the row pitches");
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* base = (uint8_t*)workspace;
    PrefillWs ws;
    ws.cnt = (int*)(base + PL.off[0]);
    ws.row_off = (int*)(base + PL.off[1]);
    ws.cursor = (int*)(base + PL.off[2]);
    ws.slot_e = (int*)(base + PL.off[3]);
    ws.n_mtiles = (int*)(base + PL.off[4]);
    ws.tile_expert = (int*)(base + PL.off[5]);
    ws.tile_row0 = (int*)(base + PL.off[6]);
    ws.perm_tok = (int*)(base + PL.off[7]);
    ws.perm_rank = (int*)(base + PL.off[8]);
    ws.perm_sx = (float*)(base + PL.off[9]);
    ws.xq = base + PL.off[10];
    ws.xsf = base + PL.off[11];
    ws.hq = base + PL.off[12];
    ws.hsf = base + PL.off[13];
    ws.R = PL.R;
    ws.MT = PL.MT;
    prefill_plan_kernel<<<1, 1024, 0, s>>>(idx, slot_of, T * c.k, c.E, ws, status);
    MOE_CUDA_TRY(cudaGetLastError());
    prefill_quant_kernel<<<(T * 32 + 255) / 256, 256, 0, s>>>((const uint16_t*)x_bf16, T, c.H, c.k, c.E, idx, ws,
                                                              nullptr, nullptr, nullptr);
    MOE_CUDA_TRY(cudaGetLastError());

    const size_t pool_bytes = size_t(c.n_slots) * B.bytes;
    CUtensorMap ma1, msa1, mb1, msb1, ma2, msa2, mb2, msb2;
    int rc;
    if ((rc = make_tmap_2d(&ma1, ws.xq, gr, PL.R, gr, 128, 128, true))) return rc;
    if ((rc = make_tmap_2d(&msa1, ws.xsf, gs, PL.R, gs, 16, 128, false))) return rc;
    if ((rc = make_tmap_2d(&mb1, p->slots, gr, pool_bytes / gr, gr, 128, 64, true))) return rc;
    if ((rc = make_tmap_2d(&msb1, p->slots, gs, pool_bytes / gs, gs, 16, 64, false))) return rc;
    if ((rc = make_tmap_2d(&ma2, ws.hq, dr, PL.R, dr, 128, 128, true))) return rc;
    if ((rc = make_tmap_2d(&msa2, ws.hsf, ds, PL.R, ds, 16, 128, false))) return rc;
    if ((rc = make_tmap_2d(&mb2, p->slots, dr, pool_bytes / dr, dr, 128, 128, true))) return rc;
    if ((rc = make_tmap_2d(&msb2, p->slots, ds, pool_bytes / ds, ds, 16, 128, false))) return rc;

    GemmArgs g{};
    g.ws = ws;
    g.tscale = p->tscale;
    g.w = w;
    g.y = y;
    g.status = status;
    g.layer = layer;
    g.E = c.E;
    g.k = c.k;
    g.H = c.H;
    g.I = c.I;
    g.limit_ns = 2000000000ull;
    g.b_rows_per_slot = B.bytes / gr;
    g.b_sf_rows_per_slot = B.bytes / gs;
    g.b_gate_row = B.off[0] / gr;
    g.b_up_row = B.off[2] / gr;
    g.b_gsf_row = B.off[1] / gs;
    g.b_usf_row = B.off[3] / gs;
    const int smem = PSmem::total + 1024;   // the limit was raised when the pool was created
    g.NT = c.I / 64;
    const int grid1 = std::min(PL.MT * g.NT, p->num_sms);
    grouped_gemm_kernel<1><<<grid1, kPThreads, smem, s>>>(ma1, msa1, mb1, msb1, g);
    MOE_CUDA_TRY(cudaGetLastError());
    // GEMM2 reads the down rows of the slot with its own pitch
    g.b_rows_per_slot = B.bytes / dr;
    g.b_sf_rows_per_slot = B.bytes / ds;
    g.d_row = B.off[4] / dr;
    g.d_sf_row = B.off[5] / ds;
    g.NT = c.H / 128;
    const int grid2 = std::min(PL.MT * g.NT, p->num_sms);
    grouped_gemm_kernel<2><<<grid2, kPThreads, smem, s>>>(ma2, msa2, mb2, msb2, g);
    MOE_CUDA_TRY(cudaGetLastError());
    return MOE_OK;
}
