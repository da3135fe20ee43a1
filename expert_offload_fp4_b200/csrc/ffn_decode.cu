// K4 decode expert FFN, K5 combine, and the slot dequantiser.
//
// K4 is one persistent kernel over the unique experts ("groups") of a decode
// call.  Work items, in a fixed order that every CTA derives alike:
//   A(g, rb): RA rows of gate and the same RA rows of up of group g -> h rows
//   B(g, rb): RB rows of down of group g -> weighted outputs y_part
// all A items first, then all B items; CTA c takes items c, c + grid, ...
// Groups are ordered by the ticket their slot must show, so resident experts
// come first and missed ones in the order the copy engine delivers them.
//
// Warp specialisation: warp NC (the producer) streams each item's FP4 codes and
// block scales with 1-D TMA bulk copies into a ring of shared-memory stages
// (mbarrier full/empty pairs); for a missed expert it first waits (bounded) for
// the slot's ready flag written by the copy stream.  Warps 0..NC-1 (consumers)
// decode E2M1 pairs with cvt.rn.f16x2.e2m1x2 and accumulate with the mixed
// fma.rn.f32.f16 (exact products, fp32 sums) against activations held in f16
// after a per-token power-of-two scale (bf16 x is exact in f16 that way; h is
// rounded to f16's 11 significant bits).  A block's partial sum is scaled by
// its E8M0 / E4M3 scale in fp32; the NVFP4 tensor scale and the activation
// scale are applied per row.  A items publish h rows and bump a per-group
// counter; B items wait (bounded) until all I rows of h exist.
#include <math.h>

#include "common.cuh"

namespace moe {

constexpr int kNC = 8;                       // consumer warps
constexpr int kFfnThreads = (kNC + 1) * 32;  // + one producer warp
// Register cap: with 9 warps one SM sub-partition holds 3 of them, and it must
// keep room (2 x 32 x 32 registers) for warps of the miss-copy kernel the FFN
// waits for: 3 * 32 * 144 + 2048 <= 16384.
constexpr int kFfnMaxRegs = 144;
constexpr int kAbortIdx = kMaxDecodePairs;   // ctr[kAbortIdx] = abort flag
constexpr int kDoneIdx = kMaxDecodePairs + 1;

struct Group {
    int expert, slot, M, pos;
    int ready;                 // the slot already showed the ticket this call needs
    float ts[3];
    float wt[kMaxDecodeT];     // routing weight of each member (token, rank)
    uint8_t tok[kMaxDecodeT];
    uint8_t rank[kMaxDecodeT];
};

struct FfnArgs {
    const uint16_t* x;
    const int32_t* idx;
    const float* w;
    const int32_t* slot_of;
    float* y_part;
    int* status;
    const uint8_t* slots;
    unsigned long long block_bytes;
    unsigned long long off[6];
    const float* tscale;
    const uint32_t* need;
    const uint32_t* ready;
    float* hbuf;
    unsigned int* hamax;
    unsigned int* ctr;
    int T, k, H, I, E, S, layer, fmt;
    int RA, RB, stage_bytes, nstage;
    unsigned long long ready_ns, dep_ns, pipe_ns;
    unsigned long long* trace;   // optional [gridDim][64] phase timestamps (ns), or null
};

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
    return e == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23);
}

// two E4M3 bytes (lo = first block) -> two floats
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two) {
    uint32_t h2;
    asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; cvt.rn.f16x2.e4m3x2 %0, lo; }"
        : "=r"(h2) : "r"(two));
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF))),
                       __half2float(__ushort_as_half((unsigned short)(h2 >> 16))));
}

// Power-of-two scale putting amax in [2^13, 2^14): bf16 values stay exact in f16,
// and a product with a weight (|e2m1 * 2^-14| <= 6 * 2^-14) is at most 6, so a
// 16-product f16 block sum stays below 100.
__device__ __forceinline__ float act_scale(float amax) {
    if (!(amax > 0.0f)) return 1.0f;
    int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
    int se = 127 + 13 - e;
    se = se < 1 ? 1 : (se > 254 ? 254 : se);
    return __uint_as_float((uint32_t)se << 23);
}

// Activations in shared memory are f16 rows stored piece-major: the 32 elements
// of chunk c (16 code bytes) are four 16-byte pieces, piece q of chunk c at
// uint4 index q*cpr + c (cpr = chunks per row), so lanes reading consecutive
// chunks touch consecutive 16-byte words (no bank conflicts).  Inside a piece
// the 8 elements are ordered 0,4,2,6,1,5,3,7: the f16x2 words hold the element
// pairs (0,4), (2,6), (1,5), (3,7), the pairing the E2M1 decode below produces.
__device__ __forceinline__ int act_index(int h, int cpr) {
    const int c = h >> 5, o = h & 31, e = o & 7;
    return (((o >> 3) * cpr + c) << 3) + (((e & 1) << 2) | (e & 2) | (e >> 2));
}

// Eight values of one piece (elements 0..7) as the four f16x2 words of that order.
__device__ __forceinline__ uint4 pack_piece(const float (&f)[8]) {
    const __half2 w0 = __floats2half2_rn(f[0], f[4]), w1 = __floats2half2_rn(f[2], f[6]);
    const __half2 w2 = __floats2half2_rn(f[1], f[5]), w3 = __floats2half2_rn(f[3], f[7]);
    return make_uint4(*reinterpret_cast<const uint32_t*>(&w0), *reinterpret_cast<const uint32_t*>(&w1),
                      *reinterpret_cast<const uint32_t*>(&w2), *reinterpret_cast<const uint32_t*>(&w3));
}

// 32 E2M1 codes (16 bytes; element n of a 32-bit word in bits 4n..4n+3) to 16
// f16x2 words, each value e2m1 * 2^-14 exactly: a code's magnitude bits go to
// f16 bits 11..9 (exponent low bits and the top mantissa bit) and its sign to
// bit 15, so 2^-14 scales every value, the E2M1 subnormal 0.5 included.  Per
// 32-bit word the f16 high bytes of the even elements (low nibbles) and of the
// odd elements (high nibbles) are formed in place, four bytes at a time; byte
// moves then give the words (e0,e4), (e2,e6), (e1,e5), (e3,e7).
__device__ __forceinline__ void decode_e2m1_x2(const uint4 c, uint32_t (&w)[16]) {
    const uint32_t v[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const uint32_t x = v[q];
        const uint32_t ev = ((x << 1) & 0x0E0E0E0Eu) | ((x << 4) & 0x80808080u);   // bytes: e0 e2 e4 e6
        const uint32_t od = ((x >> 3) & 0x0E0E0E0Eu) | (x & 0x80808080u);          // bytes: e1 e3 e5 e7
        w[4 * q + 0] = __byte_perm(ev, 0u, 0x2404);
        w[4 * q + 1] = ev & 0xFF00FF00u;
        w[4 * q + 2] = __byte_perm(od, 0u, 0x2404);
        w[4 * q + 3] = od & 0xFF00FF00u;
    }
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t hadd2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// acc + (v.lo + v.hi) * s, with s an f16 (an E4M3 scale is exact in f16): two
// mixed fmas, each product exact, each sum rounded once to fp32.
__device__ __forceinline__ float fma2_f16(uint32_t v, uint16_t s, float acc) {
    asm("{ .reg .f16 lo, hi, sc; mov.b32 {lo, hi}, %1; mov.b16 sc, %2;"
        " fma.rn.f32.f16 %0, lo, sc, %0; fma.rn.f32.f16 %0, hi, sc, %0; }"
        : "+f"(acc) : "r"(v), "h"(s));
    return acc;
}

__device__ __forceinline__ float f16x2_sum(uint32_t v) {
    const __half2 h = *reinterpret_cast<const __half2*>(&v);
    const float2 f = __half22float2(h);
    return f.x + f.y;
}

// two E4M3 bytes (lo = first block) -> two f16 scales in one word
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t h2;
    asm("{ .reg .b16 lo; cvt.u16.u32 lo, %1; cvt.rn.f16x2.e4m3x2 %0, lo; }" : "=r"(h2) : "r"(two));
    return h2;
}

// Dot products of one row chunk (16 code bytes = 32 elements) with MT activation
// rows.  Within a scale block the exact f16 products are summed in f16x2 (8 per
// half for NVFP4, 16 for MXFP4); each block sum is scaled and added in fp32.
// Weights carry 2^-14 (see decode_e2m1_x2); the caller multiplies it back.
template <int FMT, int MT>
__device__ __forceinline__ void chunk_dot(const uint8_t* code, const uint8_t* scl, int c, int cpr,
                                          const __half* const* act, int M, float (&acc)[MT]) {
    uint32_t wv[16];
    decode_e2m1_x2(*reinterpret_cast<const uint4*>(code + 16 * c), wv);
    uint32_t s2 = 0u;
    float sm = 0.0f;
    if (FMT == MOE_NVFP4) s2 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(scl + 2 * c));
    else sm = e8m0_to_f32(scl[c]);
#pragma unroll
    for (int m = 0; m < MT; m++) {
        if (m >= M) break;
        const uint4* xp = reinterpret_cast<const uint4*>(act[m]) + c;
        const uint4 x0 = xp[0], x1 = xp[cpr], x2 = xp[2 * cpr], x3 = xp[3 * cpr];
        const uint32_t xv[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                 x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
        uint32_t pa = 0u, pb = 0u, pc = 0u, pd = 0u;   // two chains per 16-element block
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            pa = hfma2_u32(wv[i], xv[i], pa);
            pb = hfma2_u32(wv[i + 1], xv[i + 1], pb);
            pc = hfma2_u32(wv[8 + i], xv[8 + i], pc);
            pd = hfma2_u32(wv[9 + i], xv[9 + i], pd);
        }
        if (FMT == MOE_NVFP4) {
            acc[m] = fma2_f16(hadd2_u32(pa, pb), (uint16_t)(s2 & 0xFFFFu), acc[m]);
            acc[m] = fma2_f16(hadd2_u32(pc, pd), (uint16_t)(s2 >> 16), acc[m]);
        } else {
            acc[m] = fmaf(f16x2_sum(hadd2_u32(hadd2_u32(pa, pb), hadd2_u32(pc, pd))), sm, acc[m]);
        }
    }
}

// Gate and up rows of one chunk together: the activation chunk of each token is
// loaded once and the eight f16x2 chains (4 per row) run interleaved.
template <int FMT, int MT>
__device__ __forceinline__ void chunk_dot_pair(const uint8_t* gcode, const uint8_t* gscl, const uint8_t* ucode,
                                               const uint8_t* uscl, int c, int cpr, const __half* const* act,
                                               int M, float (&ag)[MT], float (&au)[MT]) {
    uint32_t wg[16], wu[16];
    decode_e2m1_x2(*reinterpret_cast<const uint4*>(gcode + 16 * c), wg);
    decode_e2m1_x2(*reinterpret_cast<const uint4*>(ucode + 16 * c), wu);
    uint32_t sg2 = 0u, su2 = 0u;
    float sgm = 0.0f, sum_ = 0.0f;
    if (FMT == MOE_NVFP4) {
        sg2 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(gscl + 2 * c));
        su2 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(uscl + 2 * c));
    } else {
        sgm = e8m0_to_f32(gscl[c]);
        sum_ = e8m0_to_f32(uscl[c]);
    }
#pragma unroll
    for (int m = 0; m < MT; m++) {
        if (m >= M) break;
        const uint4* xp = reinterpret_cast<const uint4*>(act[m]) + c;
        const uint4 x0 = xp[0], x1 = xp[cpr], x2 = xp[2 * cpr], x3 = xp[3 * cpr];
        const uint32_t xv[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                                 x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
        uint32_t ga = 0u, gb = 0u, gc = 0u, gd = 0u, ua = 0u, ub = 0u, uc = 0u, ud = 0u;
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            ga = hfma2_u32(wg[i], xv[i], ga);
            ua = hfma2_u32(wu[i], xv[i], ua);
            gb = hfma2_u32(wg[i + 1], xv[i + 1], gb);
            ub = hfma2_u32(wu[i + 1], xv[i + 1], ub);
            gc = hfma2_u32(wg[8 + i], xv[8 + i], gc);
            uc = hfma2_u32(wu[8 + i], xv[8 + i], uc);
            gd = hfma2_u32(wg[9 + i], xv[9 + i], gd);
            ud = hfma2_u32(wu[9 + i], xv[9 + i], ud);
        }
        if (FMT == MOE_NVFP4) {
            ag[m] = fma2_f16(hadd2_u32(ga, gb), (uint16_t)(sg2 & 0xFFFFu), ag[m]);
            ag[m] = fma2_f16(hadd2_u32(gc, gd), (uint16_t)(sg2 >> 16), ag[m]);
            au[m] = fma2_f16(hadd2_u32(ua, ub), (uint16_t)(su2 & 0xFFFFu), au[m]);
            au[m] = fma2_f16(hadd2_u32(uc, ud), (uint16_t)(su2 >> 16), au[m]);
        } else {
            ag[m] = fmaf(f16x2_sum(hadd2_u32(hadd2_u32(ga, gb), hadd2_u32(gc, gd))), sgm, ag[m]);
            au[m] = fmaf(f16x2_sum(hadd2_u32(hadd2_u32(ua, ub), hadd2_u32(uc, ud))), sum_, au[m]);
        }
    }
}

// Sum over the G lanes of each lane group (G a power of two <= 32, warp-uniform);
// the offsets are unrolled and the MT sums interleaved.
template <int MT>
__device__ __forceinline__ void group_reduce(float (&acc)[MT], int G) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (off < G) {
#pragma unroll
            for (int m = 0; m < MT; m++) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
        }
    }
}

template <int MT>
__device__ __forceinline__ void group_reduce4(float (&x0)[MT], float (&y0)[MT], float (&x1)[MT], float (&y1)[MT],
                                              int G, bool two) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (off < G) {
#pragma unroll
            for (int m = 0; m < MT; m++) {
                x0[m] += __shfl_xor_sync(0xffffffffu, x0[m], off);
                y0[m] += __shfl_xor_sync(0xffffffffu, y0[m], off);
                if (two) {
                    x1[m] += __shfl_xor_sync(0xffffffffu, x1[m], off);
                    y1[m] += __shfl_xor_sync(0xffffffffu, y1[m], off);
                }
            }
        }
    }
}

template <int MT>
__device__ __forceinline__ void group_reduce2(float (&x)[MT], float (&y)[MT], int G) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        if (off < G) {
#pragma unroll
            for (int m = 0; m < MT; m++) {
                x[m] += __shfl_xor_sync(0xffffffffu, x[m], off);
                y[m] += __shfl_xor_sync(0xffffffffu, y[m], off);
            }
        }
    }
}

__host__ __device__ __forceinline__ int lanes_per_row(int K) {
    const int cpr = K / 32;  // 16-byte chunks per row
    int g = 32;
    while (g > 1 && cpr % g) g >>= 1;
    return g;
}

__device__ __forceinline__ bool wait_ready(const FfnArgs& a, int slot, volatile unsigned int* abort_flag) {
    const uint32_t want = a.need[slot];
    if (ld_acquire_sys_u32(a.ready + slot) == want) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (ld_acquire_sys_u32(a.ready + slot) == want) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > a.ready_ns) return false;
        __nanosleep(64);
    }
}

template <int FMT, int MT>
__global__ void __maxnreg__(kFfnMaxRegs) ffn_decode_kernel(const FfnArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + a.nstage;
    Group* groups = reinterpret_cast<Group*>(smem + 16 * a.nstage);
    float* xinv = reinterpret_cast<float*>(groups + kMaxDecodePairs);   // [16]
    float* hinv = xinv + kMaxDecodeT;                                   // [16]
    int* s_misc = reinterpret_cast<int*>(hinv + kMaxDecodeT);           // [4]
    __half* xs = reinterpret_cast<__half*>(
        (reinterpret_cast<uintptr_t>(s_misc + 4) + 15) & ~uintptr_t(15));  // [T][H]
    __half* hs = xs + a.T * a.H;                                        // [MT][I]
    uint8_t* stages = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(hs + MT * a.I) + 127) & ~uintptr_t(127));

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    volatile unsigned int* abort_flag = a.ctr + kAbortIdx;
    unsigned long long* trace = a.trace ? a.trace + (size_t)blockIdx.x * 64 : nullptr;
    if (trace && tid == 0) trace[0] = globaltimer();
    const int bs = FMT == MOE_MXFP4 ? 32 : 16;
    const unsigned long long codeA = (unsigned long long)a.H / 2, sclA = (unsigned long long)a.H / bs;
    const unsigned long long codeB = (unsigned long long)a.I / 2, sclB = (unsigned long long)a.I / bs;

    // ---- prologue 1 (before the previous kernel of the stream finishes): barriers
    // and the activations, which predate the router: per-token power-of-two
    // scale, f16, piece-major rows, 16-byte loads (8 bf16), a shared per-token max
    // first (in hinv, free until the down projection)
    const int cprA = a.H / 32, cprB = a.I / 32;
    {
        unsigned* tok_amax = reinterpret_cast<unsigned*>(hinv);
        if (tid < a.T) tok_amax[tid] = 0u;
        __syncthreads();
        const int nvec = a.T * a.H / 8;
        for (int v = tid; v < nvec; v += blockDim.x) {
            const uint4 q = __ldg(reinterpret_cast<const uint4*>(a.x) + v);
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
            float mx = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; i++)
                mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(u[i] << 16)), fabsf(__uint_as_float(u[i] & 0xFFFF0000u))));
            atomicMax(tok_amax + (v * 8) / a.H, __float_as_uint(mx));
        }
        __syncthreads();
        for (int v = tid; v < nvec; v += blockDim.x) {
            const int t = (v * 8) / a.H, h = v * 8 - t * a.H;
            const float sc = act_scale(__uint_as_float(tok_amax[t]));
            const uint4 q = __ldg(reinterpret_cast<const uint4*>(a.x) + v);
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                f[2 * i] = __uint_as_float(u[i] << 16) * sc;
                f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u) * sc;
            }
            *reinterpret_cast<uint4*>(xs + t * a.H + act_index(h, cprA)) = pack_piece(f);
            if (h == 0) xinv[t] = 1.0f / sc;
        }
    }
    // ---- the slot lookup's outputs (slot_of, tickets) are needed from here on
    pdl_wait();
    pdl_trigger();   // the combine may launch; it waits for this grid to finish
    if (trace && tid == 0) trace[1] = globaltimer();
    // ---- prologue: barriers, groups, activations (parallel; the stage ring is
    // still unused, so its first bytes hold the per-(token, rank) scratch)
    int* e_s = reinterpret_cast<int*>(stages);            // [n] expert or -1
    int* s_s = e_s + kMaxDecodePairs;                      // [n] slot
    unsigned* need_s = reinterpret_cast<unsigned*>(s_s + kMaxDecodePairs);
    int* lead_s = reinterpret_cast<int*>(need_s + kMaxDecodePairs);   // first entry of my expert
    int* mi_s = lead_s + kMaxDecodePairs;                  // my index inside the group
    int* grank_s = mi_s + kMaxDecodePairs;                 // group rank of a leader
    int* rdy_s = grank_s + kMaxDecodePairs;                // slot shows the needed ticket
    float* ts_s = reinterpret_cast<float*>(rdy_s + kMaxDecodePairs);   // [n][3] tensor scales
    const int n = a.T * a.k;
    if (tid == 0) {
        for (int i = 0; i < a.nstage; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kNC);
        }
        fence_mbar_init();
    }
    __syncthreads();   // activation staging above used hinv; the table below uses the stage ring
    if (tid < n) {
        // one dependent round of loads: the slot's tickets and the tensor scales
        const int e = a.idx[tid], sl = a.slot_of[tid];
        int bad = 0;
        if (e < 0 || e >= a.E) bad |= MOE_STATUS_BAD_EXPERT;
        if (sl < 0 || sl >= a.S) bad |= MOE_STATUS_BAD_SLOT;
        uint32_t nd = 0u, rd = 1u;
        float t0 = 0.0f, t1 = 0.0f, t2 = 0.0f;
        if (!bad) {
            nd = a.need[sl];
            rd = ld_acquire_sys_u32(a.ready + sl);
            const float* ts = a.tscale + ((size_t)a.layer * a.E + e) * 3;
            t0 = ts[0];
            t1 = ts[1];
            t2 = ts[2];
        }
        e_s[tid] = bad ? -1 : e;
        s_s[tid] = sl;
        need_s[tid] = nd;
        rdy_s[tid] = (rd == nd);
        ts_s[3 * tid] = t0;
        ts_s[3 * tid + 1] = t1;
        ts_s[3 * tid + 2] = t2;
        if (bad && blockIdx.x == 0) atomicOr(a.status, bad);
    }
    __syncthreads();
    if (tid < n && e_s[tid] >= 0) {
        const int e = e_s[tid];
        int lead = tid, mi = 0;
        for (int j = 0; j < tid; j++)
            if (e_s[j] == e) {
                if (lead == tid) lead = j;
                mi++;
            }
        lead_s[tid] = lead;
        mi_s[tid] = mi;
    }
    __syncthreads();
    // leaders: rank by (ticket the slot must show, expert) so resident experts come
    // first and missed ones in the order the copy engine delivers them
    if (tid < n && e_s[tid] >= 0 && lead_s[tid] == tid) {
        const int e = e_s[tid];
        const unsigned kt = need_s[tid];
        int rank = 0, M = 0, pos = 0;
        for (int j = 0; j < n; j++) {
            const int ej = e_s[j];
            if (ej < 0) continue;
            if (ej == e) M++;
            const bool before = need_s[j] < kt || (need_s[j] == kt && ej < e);
            if (lead_s[j] == j && before) rank++;
            if (before) pos++;       // members of groups ranked before mine
        }
        grank_s[tid] = rank;
        Group& G = groups[rank];
        G.expert = e;
        G.slot = s_s[tid];
        G.M = M;
        G.pos = pos;
        G.ready = rdy_s[tid];
        G.ts[0] = ts_s[3 * tid];
        G.ts[1] = ts_s[3 * tid + 1];
        G.ts[2] = ts_s[3 * tid + 2];
    }
    __syncthreads();
    if (tid < n && e_s[tid] >= 0) {
        Group& G = groups[grank_s[lead_s[tid]]];
        G.tok[mi_s[tid]] = (uint8_t)(tid / a.k);
        G.rank[mi_s[tid]] = (uint8_t)(tid % a.k);
        G.wt[mi_s[tid]] = a.w[tid];
    }
    if (warp == 0) {
        int c = 0;
        for (int i = lane; i < n; i += 32) c += (e_s[i] >= 0 && lead_s[i] == i);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
        if (lane == 0) s_misc[0] = c;
    }
    __syncthreads();
    if (trace && tid == 0) trace[2] = globaltimer();
    const int ng = s_misc[0];
    const int nA_per = a.I / a.RA, nB_per = a.H / a.RB;
    const int NA = ng * nA_per, NB = ng * nB_per;
    // contiguous item ranges per CTA (consecutive items mostly share an expert):
    // this CTA's A items, then its B items
    const int a0 = (int)((long long)blockIdx.x * NA / gridDim.x);
    const int a1 = (int)((long long)(blockIdx.x + 1) * NA / gridDim.x);
    const int b0 = (int)((long long)blockIdx.x * NB / gridDim.x);
    const int b1 = (int)((long long)(blockIdx.x + 1) * NB / gridDim.x);
    const int nmine = (a1 - a0) + (b1 - b0);
    // Stage layouts are the same for every item of a kind: A = gate codes, gate
    // scales, up codes, up scales of RA rows; B = down codes, down scales of RB
    // rows.  Every piece starts 16-byte aligned (H, I multiples of 256 and RA, RB
    // powers of two >= 8, checked on the host), so each is one bulk copy.
    const uint32_t lcA = (uint32_t)(a.RA * codeA), lsA = (uint32_t)(a.RA * sclA);
    const uint32_t lcB = (uint32_t)(a.RB * codeB), lsB = (uint32_t)(a.RB * sclB);
    const uint32_t bytesA = 2 * (lcA + lsA), bytesB = lcB + lsB;
    // this CTA's items in order: (kind, group, row block), advanced without division
    struct Cursor {
        int j, isB, g, rb;
    };
    auto cursor_start = [&]() {
        Cursor c{0, a1 == a0, 0, 0};
        const int first = c.isB ? b0 : a0, per = c.isB ? nB_per : nA_per;
        c.g = first / per;
        c.rb = first - c.g * per;
        return c;
    };
    auto cursor_next = [&](Cursor& c) {
        c.j++;
        if (!c.isB && c.j == a1 - a0) {
            c.isB = 1;
            c.g = b0 / nB_per;
            c.rb = b0 - c.g * nB_per;
            return;
        }
        if (++c.rb == (c.isB ? nB_per : nA_per)) {
            c.rb = 0;
            c.g++;
        }
    };

    if (warp == kNC) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            // experts whose slot showed the needed ticket when the table was built
            // (acquired there, ordered before this thread by the block barrier) are
            // read behind one proxy fence; the others are waited for when their
            // first item comes up
            uint32_t ready_mask[kMaxDecodePairs / 32] = {0, 0, 0, 0};
            for (int g = 0; g < ng; g++)
                if (groups[g].ready) ready_mask[g >> 5] |= 1u << (g & 31);
            fence_proxy_async_global();
            int st = 0, round = 0;
            for (Cursor cu = cursor_start(); cu.j < nmine; cursor_next(cu)) {
                const int j = cu.j, g = cu.g;
                if (!mbar_wait(&empty[st], (round & 1) ^ 1, a.pipe_ns)) {
                    atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
                    *abort_flag = 1;
                }
                if (!(ready_mask[g >> 5] & (1u << (g & 31)))) {
                    if (!wait_ready(a, groups[g].slot, abort_flag)) {
                        atomicOr(a.status, MOE_STATUS_READY_TIMEOUT);
                        *abort_flag = 1;
                    }
                    ready_mask[g >> 5] |= 1u << (g & 31);
                    fence_proxy_async_global();
                }
                uint8_t* dst = stages + (size_t)st * a.stage_bytes;
                const uint8_t* blk = a.slots + (unsigned long long)groups[g].slot * a.block_bytes;
                if (trace && j < 16) trace[40 + j] = globaltimer();
                if (!cu.isB) {
                    const unsigned long long r0 = (unsigned long long)cu.rb * a.RA;
                    mbar_arrive_expect_tx(&full[st], bytesA);
                    bulk_g2s(dst, blk + a.off[0] + r0 * codeA, lcA, &full[st]);
                    bulk_g2s(dst + lcA, blk + a.off[1] + r0 * sclA, lsA, &full[st]);
                    bulk_g2s(dst + lcA + lsA, blk + a.off[2] + r0 * codeA, lcA, &full[st]);
                    bulk_g2s(dst + 2 * lcA + lsA, blk + a.off[3] + r0 * sclA, lsA, &full[st]);
                } else {
                    const unsigned long long r0 = (unsigned long long)cu.rb * a.RB;
                    mbar_arrive_expect_tx(&full[st], bytesB);
                    bulk_g2s(dst, blk + a.off[4] + r0 * codeB, lcB, &full[st]);
                    bulk_g2s(dst + lcB, blk + a.off[5] + r0 * sclB, lsB, &full[st]);
                }
                if (++st == a.nstage) {
                    st = 0;
                    round++;
                }
            }
            // no copy may still be in flight when the CTA exits: wait (bounded) for
            // the last phase of every stage used
            for (int j = (nmine > a.nstage ? nmine - a.nstage : 0); j < nmine; j++)
                if (!mbar_wait(&full[j % a.nstage], (j / a.nstage) & 1, a.pipe_ns))
                    atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
        }
    } else {
        // ---------------------------------------------------------------- consumers
        const int GA = lanes_per_row(a.H), GB = lanes_per_row(a.I);
        int pend_g = -1, pend_n = 0;   // h rows written by this warp, not yet published
        auto publish = [&]() {
            __syncwarp();
            if (lane == 0 && pend_n > 0) {
                __threadfence();
                atomicAdd(a.ctr + pend_g, (unsigned int)pend_n);
            }
            pend_n = 0;
        };
        int staged_g = -1;             // group whose h sits in hs (same on every consumer warp)
        int st = 0, round = 0;
        for (Cursor cu = cursor_start(); cu.j < nmine; cursor_next(cu)) {
            const int j = cu.j, g = cu.g, rb = cu.rb;
            const bool isB = cu.isB;
            const bool ok = mbar_wait(&full[st], round & 1, a.pipe_ns);
            if (!ok) {
                if (lane == 0) atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
                *abort_flag = 1;
            }
            if (trace && tid == 0 && j == 0) trace[3] = globaltimer();
            if (trace && tid == 0 && j < 16) trace[8 + 2 * j] = globaltimer();
            if (trace && tid == 0 && j == 1) trace[62] = clock64();
            const uint8_t* sb = stages + (size_t)st * a.stage_bytes;
            const Group& G = groups[g];
            const int M = G.M;
            if (!isB) {
                // A: gate row p and up row p per lane group, of this item and (when
                // the next item is also a gate/up item) of the next one together:
                // two independent chains per warp hide each other's latency
                // (pairs only for up to 2 tokens per expert: more tokens already give
                // each warp independent chains, and the registers of two would spill)
                const int np = (MT <= 2 && j + 1 < a1 - a0) ? 2 : 1;
                Cursor cn = cu;
                int st2 = st, round2 = round;
                bool ok2 = true;
                if (np == 2) {
                    cursor_next(cn);
                    if (++st2 == a.nstage) {
                        st2 = 0;
                        round2++;
                    }
                    ok2 = mbar_wait(&full[st2], round2 & 1, a.pipe_ns);
                    if (!ok2) {
                        if (lane == 0) atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
                        *abort_flag = 1;
                    }
                }
                const Group* GG[2] = {&G, &groups[cn.g]};
                const int gg[2] = {g, cn.g}, rbs[2] = {rb, cn.rb};
                const uint8_t* sbs[2] = {sb, stages + (size_t)st2 * a.stage_bytes};
                const int MM[2] = {M, GG[1]->M};
                const int RW = 32 / GA, sub = lane / GA, gl = lane % GA;
                const __half* act[2][MT];
#pragma unroll
                for (int u = 0; u < 2; u++)
#pragma unroll
                    for (int q = 0; q < MT; q++) act[u][q] = xs + (size_t)GG[u]->tok[q < MM[u] ? q : 0] * a.H;
                for (int base = 0; base < a.RA; base += kNC * RW) {
                    const int p = base + warp * RW + sub;
                    float ag[2][MT], au[2][MT];
#pragma unroll
                    for (int u = 0; u < 2; u++)
#pragma unroll
                        for (int q = 0; q < MT; q++) ag[u][q] = au[u][q] = 0.0f;
                    if (p < a.RA && ok && ok2) {
                        const uint8_t *gc[2], *gs[2], *uc[2], *us[2];
#pragma unroll
                        for (int u = 0; u < 2; u++) {
                            gc[u] = sbs[u] + (size_t)p * codeA;
                            gs[u] = sbs[u] + lcA + (size_t)p * sclA;
                            uc[u] = sbs[u] + lcA + lsA + (size_t)p * codeA;
                            us[u] = sbs[u] + 2 * lcA + lsA + (size_t)p * sclA;
                        }
                        if (trace && tid == 0 && j == 1) trace[58] = clock64();
                        if (np == 2) {
                            for (int c = gl; c < cprA; c += GA) {
                                chunk_dot_pair<FMT, MT>(gc[0], gs[0], uc[0], us[0], c, cprA, act[0], MM[0], ag[0], au[0]);
                                chunk_dot_pair<FMT, MT>(gc[1], gs[1], uc[1], us[1], c, cprA, act[1], MM[1], ag[1], au[1]);
                            }
                        } else {
#pragma unroll 2
                            for (int c = gl; c < cprA; c += GA)
                                chunk_dot_pair<FMT, MT>(gc[0], gs[0], uc[0], us[0], c, cprA, act[0], MM[0], ag[0], au[0]);
                        }
                    }
                    if (trace && tid == 0 && j == 1) trace[59] = clock64();
                    group_reduce4<MT>(ag[0], au[0], ag[1], au[1], GA, np == 2);
                    if (trace && tid == 0 && j == 1) trace[60] = clock64();
#pragma unroll
                    for (int u = 0; u < 2; u++) {
                        if (u >= np) break;
                        const Group& Gu = *GG[u];
                        if (gg[u] != pend_g) {     // rows of the previous group are all written
                            publish();
                            pend_g = gg[u];
                        }
                        if (p < a.RA && gl == 0) {
                            const int i = rbs[u] * a.RA + p;
#pragma unroll
                            for (int q = 0; q < MT; q++) {
                                if (q >= MM[u]) break;
                                const float xi = xinv[Gu.tok[q]] * 16384.0f;   // undo the decode's 2^-14
                                const float gv = ag[u][q] * xi * Gu.ts[0];
                                const float uv = au[u][q] * xi * Gu.ts[1];
                                const float hv = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
                                a.hbuf[(size_t)(Gu.pos + q) * a.I + i] = hv;
                                atomicMax(a.hamax + Gu.pos + q, __float_as_uint(fabsf(hv)));
                            }
                        }
                        // rows this warp finished in this pass (the same count on every lane)
                        const int left = a.RA - (base + warp * RW);
                        pend_n += left <= 0 ? 0 : (left < RW ? left : RW);
                    }
                    if (trace && tid == 0 && j == 1) trace[61] = clock64();
                }
                if (np == 2) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[st2]);
                }
                if (j + np == a1 - a0) {            // last A item of this CTA
                    publish();
                    if (trace && tid == 0) trace[4] = globaltimer();
                }
                if (np == 2) {
                    // release the first stage and step over both items (the loop's
                    // increment takes the second)
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[st]);
                    if (trace && tid == 0 && j < 16) trace[9 + 2 * j] = globaltimer();
                    cursor_next(cu);
                    st = st2;
                    round = round2;
                    if (++st == a.nstage) {
                        st = 0;
                        round++;
                    }
                    continue;
                }
            } else {
                // B: h of the group staged once per run of its items, then RB rows of down
                if (g != staged_g) {
                    if (warp == 0 && lane == 0) {
                        const unsigned int want = (unsigned int)a.I;
                        if (ld_acquire_u32(a.ctr + g) < want) {
                            const unsigned long long t0 = globaltimer();
                            while (ld_acquire_u32(a.ctr + g) < want) {
                                if (*abort_flag || globaltimer() - t0 > a.dep_ns) {
                                    atomicOr(a.status, MOE_STATUS_DEP_TIMEOUT);
                                    *abort_flag = 1;
                                    break;
                                }
                            }
                        }
                    }
                    if (trace && tid == 0 && staged_g < 0) trace[5] = globaltimer();
                    named_sync(1, kNC * 32);   // also: every warp is done with the old hs
                    for (int q = warp; q < M; q += kNC) {
                        const float amax = __uint_as_float(__ldcg(a.hamax + G.pos + q));
                        const float sc = act_scale(amax);
                        if (lane == 0) hinv[q] = 1.0f / sc;
                        const float4* hrow = reinterpret_cast<const float4*>(a.hbuf + (size_t)(G.pos + q) * a.I);
                        for (int v = lane; v < a.I / 8; v += 32) {
                            const float4 f0 = __ldcg(hrow + 2 * v), f1 = __ldcg(hrow + 2 * v + 1);
                            const float f[8] = {f0.x * sc, f0.y * sc, f0.z * sc, f0.w * sc,
                                                f1.x * sc, f1.y * sc, f1.z * sc, f1.w * sc};
                            *reinterpret_cast<uint4*>(hs + (size_t)q * a.I + act_index(8 * v, cprB)) = pack_piece(f);
                        }
                    }
                    named_sync(1, kNC * 32);
                    staged_g = g;
                }
                const int RW = 32 / GB, sub = lane / GB, gl = lane % GB;
                const __half* act[MT];
#pragma unroll
                for (int q = 0; q < MT; q++) act[q] = hs + (size_t)(q < M ? q : 0) * a.I;
                for (int base = 0; base < a.RB; base += kNC * RW) {
                    const int r = base + warp * RW + sub;
                    float ay[MT];
#pragma unroll
                    for (int q = 0; q < MT; q++) ay[q] = 0.0f;
                    if (r < a.RB && ok) {
                        const uint8_t* dc = sb + (size_t)r * codeB;
                        const uint8_t* ds = sb + lcB + (size_t)r * sclB;
#pragma unroll 2
                        for (int c = gl; c < cprB; c += GB) chunk_dot<FMT, MT>(dc, ds, c, cprB, act, M, ay);
                    }
                    group_reduce<MT>(ay, GB);
                    if (r < a.RB && gl == 0) {
                        const int row = rb * a.RB + r;
#pragma unroll
                        for (int q = 0; q < MT; q++) {
                            if (q >= M) break;
                            const int t = G.tok[q], jr = G.rank[q];
                            a.y_part[((size_t)t * a.k + jr) * a.H + row] =
                                G.wt[q] * (ay[q] * (hinv[q] * 16384.0f) * G.ts[2]);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
            if (trace && tid == 0 && j < 16) trace[9 + 2 * j] = globaltimer();
            if (trace && tid == 0 && j == 1) trace[63] = clock64();
            if (++st == a.nstage) {
                st = 0;
                round++;
            }
        }
        publish();
        if (trace && tid == 0) trace[6] = globaltimer();
    }

    // ---- epilogue: the last CTA clears the per-call counters
    __syncthreads();
    if (trace && tid == 0) {
        trace[7] = globaltimer();
        trace[56] = (unsigned long long)nmine;
        trace[57] = (unsigned long long)(a1 - a0);
    }
    if (tid == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(a.ctr + kDoneIdx, 1u);
        if (prev == gridDim.x - 1) {
            __threadfence();
            for (int g = 0; g < ng; g++) a.ctr[g] = 0;
            for (int i = 0; i < a.T * a.k; i++) a.hamax[i] = 0;
            a.ctr[kAbortIdx] = 0;
            a.ctr[kDoneIdx] = 0;
            __threadfence();
        }
    }
}

// ------------------------------------------------------------------ combine

__global__ void combine_kernel(const float* __restrict__ y_part, int T, int k, int H, uint16_t* __restrict__ y) {
    pdl_wait();      // y_part comes from the expert FFN
    pdl_trigger();   // the next layer's router may launch and fetch its weights
    const size_t n4 = (size_t)T * H / 4;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i * 4;
        const size_t t = e / H, h = e % H;
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; j++) {
            const float4 v = *reinterpret_cast<const float4*>(y_part + (t * k + j) * H + h);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        const float f[4] = {s.x, s.y, s.z, s.w};
        uint16_t o[4];
#pragma unroll
        for (int q = 0; q < 4; q++) o[q] = __bfloat16_as_ushort(__float2bfloat16_rn(f[q]));
        *reinterpret_cast<uint2*>(y + e) = make_uint2(o[0] | ((uint32_t)o[1] << 16), o[2] | ((uint32_t)o[3] << 16));
    }
}

// ------------------------------------------------------------------ dequant

template <int FMT>
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                               float ts, int rows, int K, float* __restrict__ out) {
    const int bs = FMT == MOE_MXFP4 ? 32 : 16;
    const size_t nbytes = (size_t)rows * K / 2;
    for (size_t b = blockIdx.x * (size_t)blockDim.x + threadIdx.x; b < nbytes; b += (size_t)gridDim.x * blockDim.x) {
        const size_t r = b / (K / 2), c = (b % (K / 2)) * 2;
        uint32_t h2;
        asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"((uint32_t)codes[b]));
        const uint8_t s = scales[r * (K / bs) + c / bs];
        float sv;
        if (FMT == MOE_NVFP4) sv = e4m3x2_to_f32((uint32_t)s).x;
        else sv = e8m0_to_f32(s);
        float v0 = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF))) * sv;
        float v1 = __half2float(__ushort_as_half((unsigned short)(h2 >> 16))) * sv;
        if (FMT == MOE_NVFP4) {
            v0 *= ts;
            v1 *= ts;
        }
        out[r * K + c] = v0;
        out[r * K + c + 1] = v1;
    }
}

// ------------------------------------------------------------------ host side

struct FfnPlan {
    int RA, RB, stage_bytes, nstage, smem, grid;
};

static int pick_pow2_rows(int limit_rows, int rows_total, int cap) {
    int r = 1;
    while (r * 2 <= cap && r * 2 <= limit_rows && rows_total % (r * 2) == 0) r *= 2;
    return r;
}

template <int FMT, int MT>
static int launch_ffn(moe_pool* p, FfnArgs& a, cudaStream_t s) {
    const moe_config& c = p->cfg;
    const int bs = p->bs;
    const size_t rowA = (size_t)c.H / 2 + (size_t)c.H / bs;   // one gate (or up) row
    const size_t rowB = (size_t)c.I / 2 + (size_t)c.I / bs;
    // items of about 20 KB, but at least one row (pair) per consumer lane group
    const size_t target = 20 * 1024;
    const int minA = kNC * (32 / lanes_per_row(c.H)), minB = kNC * (32 / lanes_per_row(c.I));
    a.RA = pick_pow2_rows(std::max((int)(target / (2 * rowA)), minA), c.I, 64);
    a.RB = pick_pow2_rows(std::max((int)(target / rowB), minB), c.H, 256);
    // every piece of a stage (codes or scales of an item's rows) must be a whole
    // number of 16-byte units so that each is one bulk copy at an aligned offset
    if (((size_t)a.RA * c.H / bs) % 16 || ((size_t)a.RB * c.I / bs) % 16)
        return fail(MOE_EINVAL, "decode FFN: item scale rows not a multiple of 16 bytes");
    const size_t bytesA = 2 * ((size_t)a.RA * c.H / 2 + (size_t)a.RA * c.H / bs);
    const size_t bytesB = (size_t)a.RB * c.I / 2 + (size_t)a.RB * c.I / bs;
    a.stage_bytes = (int)((std::max(bytesA, bytesB) + 127) / 128 * 128);
    const size_t fixed = 16 * 16 + sizeof(Group) * kMaxDecodePairs + 4 * (2 * kMaxDecodeT + 4) + 16 +
                        (size_t)a.T * c.H * 2 + (size_t)MT * c.I * 2 + 128;
    const size_t budget = (size_t)p->ffn_smem;
    if (fixed + 2 * (size_t)a.stage_bytes > budget) return fail(MOE_EINVAL, "decode FFN: shapes exceed shared memory");
    a.nstage = (int)std::min<size_t>(12, (budget - fixed) / a.stage_bytes);
    // the prologue keeps its per-(token, rank) table (7 ints + 3 floats each) in the ring
    if ((size_t)a.nstage * a.stage_bytes < 10 * 4 * (size_t)kMaxDecodePairs)
        return fail(MOE_EINVAL, "decode FFN: stage ring smaller than the prologue table");
    const size_t smem = 16 * (size_t)a.nstage + sizeof(Group) * kMaxDecodePairs + 4 * (2 * kMaxDecodeT + 4) + 16 +
                        (size_t)a.T * c.H * 2 + (size_t)MT * c.I * 2 + 128 + (size_t)a.nstage * a.stage_bytes;
    auto kern = ffn_decode_kernel<FMT, MT>;
    const int fi = FMT == MOE_NVFP4 ? 1 : 0, mi = MT == 1 ? 0 : MT == 2 ? 1 : MT == 4 ? 2 : MT == 8 ? 3 : 4;
    if (!p->ffn_attr_set[fi][mi]) {
        // once per pool and template: the largest shared-memory carve-out, and the
        // number of co-resident CTAs per SM at that size (1: the kernel is persistent)
        MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)budget));
        MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                          cudaSharedmemCarveoutMaxShared));
        int per_sm = 0;
        MOE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFfnThreads, budget));
        p->ffn_per_sm[fi][mi] = per_sm;
        p->ffn_attr_set[fi][mi] = 1;
    }
    const int per_sm = p->ffn_per_sm[fi][mi];
    if (per_sm < 1) return fail(MOE_EINVAL, "decode FFN kernel does not fit on an SM");
    const int items_max = a.T * a.k * (c.I / a.RA + c.H / a.RB);
    const int grid = std::max(1, std::min(p->num_sms * per_sm, items_max));
    // CTAs wait on one another (down rows wait for every gate/up row of their
    // expert), so all of them must be resident together: one CTA per SM fits
    // (the shared-memory ring takes the SM) and the grid is at most the SM
    // count, so they are, once the kernels ahead of this one in the stream have
    // left.  A plain launch (not a cooperative one) lets the slot lookup before
    // it hand over through programmatic serialisation and lets the miss copies
    // of the copy stream run beside it; every wait is bounded in any case.
    MOE_CUDA_TRY(launch_pdl(kern, dim3(grid), dim3(kFfnThreads), smem, s, a));
    return MOE_OK;
}

int preload_ffn_kernels() {
    cudaFuncAttributes fa;
#define PRELOAD(F)                                                           \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, ffn_decode_kernel<F, 1>));       \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, ffn_decode_kernel<F, 2>));       \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, ffn_decode_kernel<F, 4>));       \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, ffn_decode_kernel<F, 8>));       \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, ffn_decode_kernel<F, 16>));      \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, dequant_kernel<F>));
    PRELOAD(MOE_NVFP4)
    PRELOAD(MOE_MXFP4)
#undef PRELOAD
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, combine_kernel));
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

static unsigned long long g_ready_ns = 5000000000ull, g_dep_ns = 5000000000ull, g_pipe_ns = 10000000000ull;
static unsigned long long* g_trace = nullptr;

extern "C" int moe_set_ffn_trace(void* buf) {
    g_trace = (unsigned long long*)buf;
    return MOE_OK;
}

extern "C" int moe_set_wait_limits(double ready_ms, double dep_ms, double pipe_ms) {
    if (!(ready_ms > 0) || !(dep_ms > 0) || !(pipe_ms > 0)) return fail(MOE_EINVAL, "wait limits must be positive");
    g_ready_ns = (unsigned long long)(ready_ms * 1e6);
    g_dep_ns = (unsigned long long)(dep_ms * 1e6);
    g_pipe_ns = (unsigned long long)(pipe_ms * 1e6);
    return MOE_OK;
}

extern "C" int moe_expert_ffn(moe_pool* p, int layer, const void* x_bf16, int T, const int32_t* idx,
                              const float* w, const int32_t* slot_of, float* y_part, int* status,
                              void* stream) {
    if (!p || !x_bf16 || !idx || !w || !slot_of || !y_part || !status) return fail(MOE_EINVAL, "null argument");
    const moe_config& c = p->cfg;
    if (layer < 0 || layer >= c.L) return fail(MOE_EBOUNDS, "layer outside the pool");
    if (T <= 0 || T > c.max_tokens) return fail(MOE_EINVAL, "decode FFN: T must be in [1, max_tokens]");
    FfnArgs a{};
    a.x = (const uint16_t*)x_bf16;
    a.idx = idx;
    a.w = w;
    a.slot_of = slot_of;
    a.y_part = y_part;
    a.status = status;
    a.slots = p->slots;
    a.block_bytes = p->lay.bytes;
    for (int i = 0; i < 6; i++) a.off[i] = p->lay.off[i];
    a.tscale = p->tscale;
    a.need = p->need;
    a.ready = p->ready;
    a.hbuf = p->hbuf;
    a.hamax = p->hamax;
    a.ctr = p->ctr;
    a.T = T;
    a.k = c.k;
    a.H = c.H;
    a.I = c.I;
    a.E = c.E;
    a.S = c.n_slots;
    a.layer = layer;
    a.fmt = c.fmt;
    a.ready_ns = g_ready_ns;
    a.dep_ns = g_dep_ns;
    a.pipe_ns = g_pipe_ns;
    a.trace = g_trace;
    cudaStream_t s = (cudaStream_t)stream;
    const int MT = T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : 16;
#define DISPATCH(F)                                              \
    switch (MT) {                                                \
        case 1: return launch_ffn<F, 1>(p, a, s);                \
        case 2: return launch_ffn<F, 2>(p, a, s);                \
        case 4: return launch_ffn<F, 4>(p, a, s);                \
        case 8: return launch_ffn<F, 8>(p, a, s);                \
        default: return launch_ffn<F, 16>(p, a, s);              \
    }
    if (c.fmt == MOE_NVFP4) { DISPATCH(MOE_NVFP4) } else { DISPATCH(MOE_MXFP4) }
#undef DISPATCH
}

extern "C" int moe_combine(const float* y_part, int T, int k, int H, void* y_bf16, void* stream) {
    if (!y_part || !y_bf16) return fail(MOE_EINVAL, "null argument");
    if (T <= 0 || k <= 0 || H <= 0 || H % 4) return fail(MOE_EINVAL, "combine: bad shape");
    const size_t n4 = (size_t)T * H / 4;
    const int threads = 256;
    const int blocks = (int)std::min<size_t>((n4 + threads - 1) / threads, 148 * 8);
    MOE_CUDA_TRY(launch_pdl(combine_kernel, dim3(blocks), dim3(threads), 0, (cudaStream_t)stream, y_part, T, k, H,
                            (uint16_t*)y_bf16));
    return MOE_OK;
}

extern "C" int moe_dequant_slot(moe_pool* p, int slot, int key, int which, float* out, void* stream) {
    if (!p || !out) return fail(MOE_EINVAL, "null argument");
    const moe_config& c = p->cfg;
    if (slot < 0 || slot >= c.n_slots || key < 0 || key >= c.L * c.E || which < 0 || which > 2)
        return fail(MOE_EBOUNDS, "dequant: slot/key/which out of range");
    const int rows = which == 2 ? c.H : c.I, K = which == 2 ? c.I : c.H;
    const uint8_t* base = p->slots + (size_t)slot * p->lay.bytes;
    const uint8_t* codes = base + p->lay.off[2 * which];
    const uint8_t* scales = base + p->lay.off[2 * which + 1];
    float ts = 1.0f;
    if (c.fmt == MOE_NVFP4) MOE_CUDA_TRY(cudaMemcpy(&ts, p->tscale + (size_t)key * 3 + which, 4, cudaMemcpyDeviceToHost));
    const size_t nbytes = (size_t)rows * K / 2;
    const int blocks = (int)std::min<size_t>((nbytes + 255) / 256, 148 * 16);
    if (c.fmt == MOE_NVFP4)
        dequant_kernel<MOE_NVFP4><<<blocks, 256, 0, (cudaStream_t)stream>>>(codes, scales, ts, rows, K, out);
    else
        dequant_kernel<MOE_MXFP4><<<blocks, 256, 0, (cudaStream_t)stream>>>(codes, scales, ts, rows, K, out);
    MOE_CUDA_TRY(cudaGetLastError());
    return MOE_OK;
}
