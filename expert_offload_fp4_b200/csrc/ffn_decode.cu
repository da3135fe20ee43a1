// K4 decode expert FFN with the K5 combine fused in, and the slot dequantiser.
//
// Work split over the whole GPU, one CTA per SM.  The call's unique experts
// ("groups", in ticket order: resident experts first, missed ones in the order
// the copy engine delivers them) give two lists of equal-sized work items:
//   A items: 16 rows of gate and the same 16 rows of up of one group; their dot
//      products with the x of every member token give 16 rows of
//      h = silu(gate x) * (up x), stored in fp32 to a global buffer (one row of I
//      values per (token, rank)) and counted per group;
//   B tiles: 16 rows of down of one group; once the group's whole h is counted,
//      y_e = down h for each member, times its routing weight, goes to y_part.
// CTA c takes the c-th contiguous share of each list (A first, then B), so every
// SM streams the same number of weight bytes whatever the number of groups.  B
// waits (bounded) for A items of other CTAs; all CTAs are resident at once (one
// per SM), and A items wait for nothing but their own copies and tickets, so the
// waits always end.  Every B tile counts its 16-row tile of H (an atomic count
// per tile); afterwards CTA c waits for the full counts of tiles c, c + grid, ...
// and sums y_part over the ranks in rank order into their bf16 output rows (K5).
//
// Warp specialisation: warp 16 (the producer) streams the FP4 code rows and
// block scales of each work stage with 1-D bulk copies (a tile of rows is one
// contiguous range of the slot) into a ring of shared-memory stages (mbarrier
// full/empty pairs); for a missed expert it first waits (bounded) for the
// slot's ready ticket written by the copy stream.  B stages are prefetched
// while h is still being produced elsewhere.
// Warps 0..15 (consumers) run the dot products on the tensor cores with
// mma.sync m16n8k16, f16 inputs and fp32 accumulation:
//  - weights: E2M1 code pairs converted to f16 pairs (cvt.rn.f16x2.e2m1x2),
//    multiplied (exactly) by their block scale in f16: the E4M3 scale itself
//    (NVFP4), or 2^(e - E) with E the largest E8M0 exponent of the row's
//    128-element segment (MXFP4; 2^(E-127) is applied to the segment's fp32 sum);
//  - activations: x of each token times a power of two (bf16 is exact in f16
//    that way); h of each (token, expert) times a power of two and split into
//    an f16 high part and an f16 remainder, so down h is carried to ~22 bits;
//  - products are exact, sums fp32 in a fixed order, so results are reproducible.
#include <math.h>

#include "common.cuh"
#include "router_topk.cuh"

namespace moe {

constexpr int kNC = 16;                      // consumer warps
constexpr int kFfnThreads = (kNC + 1) * 32;  // + one producer warp
constexpr int kConsThreads = kNC * 32;
// Register cap.  The 17 warps of a CTA spread over the SM's 4 sub-partitions, 5 on
// one of them, whose register file holds 16384 registers; one warp of the SM copy
// kernel (128 threads, at most 32 registers), which a waiting FFN may depend on,
// must fit beside them: 5 * 32 * 96 + 32 * 32 <= 16384.
constexpr int kFfnMaxRegs = 96;
constexpr int kSeg = 128;                    // K elements per segment (64 code bytes)
// SMs left free for the SM copy kernel (MOE_COPY_SM), which a waiting FFN depends on
constexpr int kCopySMs = 16;

struct Group {
    int expert, slot, M;
    int ready_a, ready_b;      // the slot showed gate/up (a) or the whole block (b) at table time
    unsigned need;
    float ts[3];
    float wt[kMaxDecodeT];     // routing weight of each member (token, rank)
    uint8_t tok[kMaxDecodeT];
    uint8_t rank[kMaxDecodeT];
};

struct FfnArgs {
    const uint16_t* x;
    const int32_t* idx;
    const float* w;
    int32_t* idx_out;          // fused router: the caller's idx and w, written by CTA 0
    float* w_out;
    int32_t* slot_of;          // read; written by CTA 0 in resident mode
    float* y_part;
    uint16_t* y;               // bf16 output [T, H] (the fused combine), or null
    int* status;
    const uint8_t* slots;
    unsigned long long block_bytes;
    unsigned long long off[6];
    const float* tscale;
    const uint32_t* need;
    const uint32_t* ready;
    float* hbuf;               // [T * k][I] h of each (token, rank), fp32
    // resident mode (no lookup kernel before this one): slots come from key_slot;
    // CTA 0 touches the hits' LRU clocks the way the lookup does and writes slot_of
    const int32_t* key_slot;
    unsigned long long* slot_clock;
    unsigned long long* clock;
    int resident;
    // fused router (resident mode only), or wr = null: idx and w come from the caller.
    // Each of the first E consumer warps of the grid computes one expert's logits for
    // every token in the router kernel's order; every CTA then selects the top-k of
    // every token; CTA 0 writes idx and w for the caller.
    const uint16_t* wr;        // [E][H] bf16
    const float* rbias;        // [E] or null
    int renorm;
    float* rlogits;            // [T][E] fp32 scratch
    unsigned int* ctr;         // [H/16] row tiles, [kMaxDecodePairs] groups, [kMaxDecodePairs] pair maxima,
                               // abort flag, done count
    int T, k, H, I, E, S, layer;
    int TRB;                   // 16-row down tiles per B stage: 1, 2, 4 or 8
    int stage_bytes, nstage;
    // byte offsets in dynamic shared memory
    int o_groups, o_misc, o_ts, o_red, o_frag, o_stage;
    unsigned long long ready_ns, dep_ns, pipe_ns;
    unsigned long long* trace;   // optional [gridDim][32] phase stamps (ns), or null
};

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
    return e == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(e << 23);
}

// two E4M3 bytes (lo = first block) -> two f16 values in one word
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    uint32_t h2;
    asm("{ .reg .b16 lo; cvt.u16.u32 lo, %1; cvt.rn.f16x2.e4m3x2 %0, lo; }" : "=r"(h2) : "r"(two));
    return h2;
}

// two E4M3 bytes (lo = first block) -> two floats
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two) {
    const uint32_t h2 = e4m3x2_to_f16x2(two);
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF))),
                       __half2float(__ushort_as_half((unsigned short)(h2 >> 16))));
}

// Power-of-two scale putting amax in [2^13, 2^14): bf16 values stay exact in f16.
__device__ __forceinline__ float act_scale(float amax) {
    if (!(amax > 0.0f)) return 1.0f;
    int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
    int se = 127 + 13 - e;
    se = se < 1 ? 1 : (se > 254 ? 254 : se);
    return __uint_as_float((uint32_t)se << 23);
}

// 2^d as an f16 bit pattern for d <= 0 (0 below the smallest subnormal).
__device__ __forceinline__ uint32_t f16_pow2(int d) {
    if (d >= -14) return (uint32_t)(d + 15) << 10;
    if (d >= -24) return 1u << (d + 24);
    return 0u;
}

// Eight values of one 16-byte piece (elements 0..7) as the f16x2 words (0,1),
// (2,3), (4,5), (6,7): the pairs a code word's four bytes decode to.
__device__ __forceinline__ uint4 pack_piece(const float (&f)[8]) {
    const __half2 w0 = __floats2half2_rn(f[0], f[1]), w1 = __floats2half2_rn(f[2], f[3]);
    const __half2 w2 = __floats2half2_rn(f[4], f[5]), w3 = __floats2half2_rn(f[6], f[7]);
    return make_uint4(*reinterpret_cast<const uint32_t*>(&w0), *reinterpret_cast<const uint32_t*>(&w1),
                      *reinterpret_cast<const uint32_t*>(&w2), *reinterpret_cast<const uint32_t*>(&w3));
}

// Two E2M1 codes (the low nibble of v's low byte first) -> their f16 values.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t v) {
    uint32_t h2;
    asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"(v));
    return h2;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// D += A * B for one 16x8x16 tile: A row-major f16 (4 words), B col-major f16
// (2 words), D fp32 (4 values).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    // no side effects: the compiler may interleave independent MMAs
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bounded wait on an mbarrier phase that also gives up as soon as another wait
// of the launch has raised the abort flag.
__device__ __forceinline__ bool mbar_wait_abort(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                                volatile unsigned int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (unsigned it = 0;; it++) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 15) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) return false;
        }
    }
}

// Acquire at GPU scope.  The ready tickets and the slot bytes they publish are
// this GPU's memory, written by its SM copy kernel or by its copy engine ahead of
// a stream write of the ticket; the slot bytes are read by bulk copies through L2.
__device__ __forceinline__ unsigned ld_acquire_gpu_u32(const unsigned int* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait until (*ready & mask) == want: mask ~kTicketPartA for the gate/up
// part of a copy, all ones for the whole block.
__device__ __forceinline__ bool wait_ready(const uint32_t* ready, uint32_t want, uint32_t mask,
                                           unsigned long long limit_ns, volatile unsigned int* abort_flag) {
    if ((ld_acquire_gpu_u32(ready) & mask) == want) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if ((ld_acquire_gpu_u32(ready) & mask) == want) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) return false;
        __nanosleep(64);
    }
}

// Bounded wait (acquire) until a counter of this launch reaches `want`.
__device__ __forceinline__ bool wait_count(const unsigned int* ctr, unsigned want, unsigned long long limit_ns,
                                           volatile unsigned int* abort_flag) {
    if (ld_acquire_gpu_u32(ctr) >= want) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (ld_acquire_gpu_u32(ctr) >= want) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) return false;
        __nanosleep(32);
    }
}

// ------------------------------------------------------------------ tile math
//
// The dot products of one 16-row tile with NB B operands of NT 8-column tiles,
// over the nseg 128-element K segments seg0 .. seg0+nseg-1.  Thread (g = lane/4,
// q = lane%4) reads the 16 code bytes [64 s + 16 q, +16) of rows g and g+8 of
// segment s (its elements 32q .. 32q+31): word j of them holds elements
// 8j .. 8j+7, whose four byte pairs become the A fragments of two MMA k-tiles
// (k slots 2q, 2q+1 take pair 0 / 2 of the word, slots 2q+8, 2q+9 pair 1 / 3).
// The B operands are stored in the same order.
// B operand layout (16-byte pieces): piece (s, j, n, q) holds column n's
// elements 128 s + 32 q + 8 j + 0..7 at index ((4 s + j) * N + n) * 4 + q;
// bcol[b][n] points at (0, 0, n, q) (null past the group's columns) and
// bstride = 4 N pieces separates consecutive j.
// The two k-tiles of a word and the NB operands go to 2 NB separate fp32
// accumulators (independent MMA chains), summed in a fixed order at the end;
// the next segment's codes and scales are loaded before this one is decoded.
template <int FMT, int NT, int NB>
__device__ __forceinline__ void tile_mma(const uint8_t* code, uint32_t row8_code, const uint8_t* scl,
                                         uint32_t row8_scl, int q, int seg0, int nseg,
                                         const uint4* const (&bcol)[NB][NT], int bstride,
                                         float (&out)[NT][4]) {
    constexpr int NA = 2 * NB;
    constexpr uint32_t sstep = FMT == MOE_NVFP4 ? 8u : 4u;     // scale bytes of a row's segment
    float acc[NA][NT][4];
#pragma unroll
    for (int i = 0; i < NA; i++)
#pragma unroll
        for (int n = 0; n < NT; n++)
#pragma unroll
            for (int e = 0; e < 4; e++) acc[i][n][e] = 0.0f;
    auto ld_scale = [](const uint8_t* p) -> uint32_t {
        return FMT == MOE_NVFP4 ? (uint32_t)*reinterpret_cast<const uint16_t*>(p)
                                : *reinterpret_cast<const uint32_t*>(p);
    };
    code += (size_t)seg0 * 64;
    scl += (size_t)seg0 * sstep;
    uint4 c = *reinterpret_cast<const uint4*>(code), c8 = *reinterpret_cast<const uint4*>(code + row8_code);
    uint32_t u = ld_scale(scl), u8 = ld_scale(scl + row8_scl);
    for (int i = 0; i < nseg; i++) {
        const int seg = seg0 + i;
        // the next segment's words (this one's again on the last, in bounds)
        const uint8_t* cn = code + (i + 1 < nseg ? 64 : 0);
        const uint8_t* sn = scl + (i + 1 < nseg ? sstep : 0u);
        const uint4 c_n = *reinterpret_cast<const uint4*>(cn), c8_n = *reinterpret_cast<const uint4*>(cn + row8_code);
        const uint32_t u_n = ld_scale(sn), u8_n = ld_scale(sn + row8_scl);
        uint32_t fa, fb, fa8, fb8;
        float post = 1.0f, post8 = 1.0f;
        if (FMT == MOE_NVFP4) {
            // the thread's two scales per row (blocks 2q, 2q+1 of the segment), exact in f16
            const uint32_t s2 = e4m3x2_to_f16x2(u), s28 = e4m3x2_to_f16x2(u8);
            fa = __byte_perm(s2, 0u, 0x1010);
            fb = __byte_perm(s2, 0u, 0x3232);
            fa8 = __byte_perm(s28, 0u, 0x1010);
            fb8 = __byte_perm(s28, 0u, 0x3232);
        } else {
            // the 4 E8M0 exponents of the segment; the thread's block (q) relative to their max
            uint32_t m = __vmaxu4(u, u >> 8), m8 = __vmaxu4(u8, u8 >> 8);
            m = __vmaxu4(m, m >> 16) & 0xFFu;
            m8 = __vmaxu4(m8, m8 >> 16) & 0xFFu;
            const uint32_t f = f16_pow2((int)((u >> (8 * q)) & 0xFFu) - (int)m);
            const uint32_t f8 = f16_pow2((int)((u8 >> (8 * q)) & 0xFFu) - (int)m8);
            fa = fb = f | (f << 16);
            fa8 = fb8 = f8 | (f8 << 16);
            post = e8m0_to_f32(m);
            post8 = e8m0_to_f32(m8);
        }
        float sacc[NA][NT][4];     // MXFP4: this segment's sums, before 2^(E-127)
        if (FMT == MOE_MXFP4) {
#pragma unroll
            for (int a = 0; a < NA; a++)
#pragma unroll
                for (int n = 0; n < NT; n++)
#pragma unroll
                    for (int e = 0; e < 4; e++) sacc[a][n][e] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 4; j++) {
            uint4 bv[NB][NT];
#pragma unroll
            for (int b = 0; b < NB; b++)
#pragma unroll
                for (int n = 0; n < NT; n++)
                    bv[b][n] = bcol[b][n] ? bcol[b][n][(seg * 4 + j) * bstride] : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t cw = j == 0 ? c.x : j == 1 ? c.y : j == 2 ? c.z : c.w;
            const uint32_t cw8 = j == 0 ? c8.x : j == 1 ? c8.y : j == 2 ? c8.z : c8.w;
            const uint32_t f = j < 2 ? fa : fb, f8 = j < 2 ? fa8 : fb8;
            const uint32_t p0 = hmul2_u32(e2m1x2_to_f16x2(cw), f), p1 = hmul2_u32(e2m1x2_to_f16x2(cw >> 8), f);
            const uint32_t p2 = hmul2_u32(e2m1x2_to_f16x2(cw >> 16), f), p3 = hmul2_u32(e2m1x2_to_f16x2(cw >> 24), f);
            const uint32_t t0 = hmul2_u32(e2m1x2_to_f16x2(cw8), f8), t1 = hmul2_u32(e2m1x2_to_f16x2(cw8 >> 8), f8);
            const uint32_t t2 = hmul2_u32(e2m1x2_to_f16x2(cw8 >> 16), f8), t3 = hmul2_u32(e2m1x2_to_f16x2(cw8 >> 24), f8);
#pragma unroll
            for (int n = 0; n < NT; n++)
#pragma unroll
                for (int b = 0; b < NB; b++) {
                    float (&d0)[4] = FMT == MOE_MXFP4 ? sacc[b][n] : acc[b][n];
                    float (&d1)[4] = FMT == MOE_MXFP4 ? sacc[NB + b][n] : acc[NB + b][n];
                    mma16816(d0, p0, t0, p1, t1, bv[b][n].x, bv[b][n].y);
                    mma16816(d1, p2, t2, p3, t3, bv[b][n].z, bv[b][n].w);
                }
        }
        if (FMT == MOE_MXFP4) {
#pragma unroll
            for (int a = 0; a < NA; a++)
#pragma unroll
                for (int n = 0; n < NT; n++) {
                    acc[a][n][0] = fmaf(sacc[a][n][0], post, acc[a][n][0]);
                    acc[a][n][1] = fmaf(sacc[a][n][1], post, acc[a][n][1]);
                    acc[a][n][2] = fmaf(sacc[a][n][2], post8, acc[a][n][2]);
                    acc[a][n][3] = fmaf(sacc[a][n][3], post8, acc[a][n][3]);
                }
        }
        c = c_n;
        c8 = c8_n;
        u = u_n;
        u8 = u8_n;
        code = cn;
        scl = sn;
    }
#pragma unroll
    for (int n = 0; n < NT; n++)
#pragma unroll
        for (int e = 0; e < 4; e++) {
            float v = acc[0][n][e];
#pragma unroll
            for (int i = 1; i < NA; i++) v += acc[i][n][e];
            out[n][e] = v;
        }
}

// Index (16-byte pieces) of the B-operand piece holding elements k0 .. k0+7
// (k0 a multiple of 8) of column n, for N columns.
__device__ __forceinline__ int piece_index(int k0, int n, int N) {
    const int s = k0 >> 7, q = (k0 >> 5) & 3, j = (k0 >> 3) & 3;
    return ((s * 4 + j) * N + n) * 4 + q;
}

// ------------------------------------------------------------------ the kernel

template <int FMT, int NT>
__global__ void __maxnreg__(kFfnMaxRegs) ffn_decode_kernel(const FfnArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + a.nstage;
    Group* groups = reinterpret_cast<Group*>(smem + a.o_groups);
    float* xinv = reinterpret_cast<float*>(smem + a.o_misc);           // [16] per token
    float* hinv = xinv + kMaxDecodeT;                                  // [16] per member
    unsigned* hmx = reinterpret_cast<unsigned*>(hinv + kMaxDecodeT);   // [16] per token (x staging)
    int* s_misc = reinterpret_cast<int*>(hmx + kMaxDecodeT);           // [8]
    int32_t* ridx = reinterpret_cast<int32_t*>(s_misc + 8);            // [T*k] fused router's choices
    float* rw = reinterpret_cast<float*>(ridx + kMaxDecodePairs);      // [T*k] and weights
    float* ts_row = reinterpret_cast<float*>(smem + a.o_ts);           // [E][3] this layer's tensor scales
    float* unitbuf = reinterpret_cast<float*>(smem + a.o_red);         // [unit][2][2 (gate, up)][ks][16][T]
    uint4* xf = reinterpret_cast<uint4*>(smem + a.o_frag);             // x fragments (A), N = T
    uint4* hf_hi = reinterpret_cast<uint4*>(smem + a.o_frag);          // h fragments (B), same bytes
    uint4* hf_lo = hf_hi + (size_t)a.T * a.I / 8;
    uint8_t* stages = smem + a.o_stage;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = a.T, H = a.H, I = a.I;
    unsigned int* rowcnt = a.ctr;                                      // [H/16] groups done per row tile
    unsigned int* gcnt = a.ctr + H / 16;                               // [kMaxDecodePairs] h values published
    unsigned int* pmax = gcnt + kMaxDecodePairs;                       // [kMaxDecodePairs] max |h| bits per pair
    volatile unsigned int* abort_flag = pmax + kMaxDecodePairs;
    unsigned int* done_ctr = pmax + kMaxDecodePairs + 1;
    unsigned int* route_ctr = pmax + kMaxDecodePairs + 2;              // experts whose logits are out
    const int bs = FMT == MOE_MXFP4 ? 32 : 16;
    const int nTA = I / 16, nTB = H / 16;                              // A items, B tiles per group
    const int nsegA = H / kSeg, nsegB = I / kSeg;
    const uint32_t SA = H / bs, SB = I / bs;                           // scale bytes of a gate/up row, a down row
    const uint32_t CA = 16 * (H / 2);                                  // code bytes of 16 gate (or up) rows
    unsigned long long* trace = a.trace ? a.trace + (size_t)blockIdx.x * 32 : nullptr;
    if (trace && tid == 0) trace[0] = globaltimer();

    // ---- prologue 1 (may overlap the kernel before this one in the stream):
    // barriers, the layer's tensor scales (written only when experts are loaded
    // into the host store), and the activations, which predate the router:
    // per-token power-of-two scale, f16 B fragments
    if (tid == 0) {
        for (int i = 0; i < a.nstage; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kNC);
        }
        fence_mbar_init();
    }
    for (int i = tid; i < a.E * 3; i += blockDim.x) ts_row[i] = a.tscale[(size_t)a.layer * a.E * 3 + i];
    {
        if (tid < T) hmx[tid] = 0u;
        __syncthreads();
        const int nvec = T * H / 8;
        for (int v = tid; v < nvec; v += blockDim.x) {
            const uint4 qv = __ldg(reinterpret_cast<const uint4*>(a.x) + v);
            const uint32_t u[4] = {qv.x, qv.y, qv.z, qv.w};
            float mx = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; i++)
                mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(u[i] << 16)), fabsf(__uint_as_float(u[i] & 0xFFFF0000u))));
            atomicMax(hmx + (v * 8) / H, __float_as_uint(mx));
        }
        __syncthreads();
        for (int v = tid; v < nvec; v += blockDim.x) {
            const int t = (v * 8) / H, h = v * 8 - t * H;
            const float sc = act_scale(__uint_as_float(hmx[t]));
            const uint4 qv = __ldg(reinterpret_cast<const uint4*>(a.x) + v);
            const uint32_t u[4] = {qv.x, qv.y, qv.z, qv.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                f[2 * i] = __uint_as_float(u[i] << 16) * sc;
                f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u) * sc;
            }
            xf[piece_index(h, t, T)] = pack_piece(f);
            if (h == 0) xinv[t] = 1.0f / sc;
        }
    }
    // fused router: this warp's expert's router row on its way to L2, and the raw
    // bf16 x in the (still unused) stage ring after the top-k scratch
    const int r_e = blockIdx.x * kNC + warp;
    uint4* rx = reinterpret_cast<uint4*>(stages + (size_t)kNC * a.E * 5 + 15 - ((size_t)kNC * a.E * 5 + 15) % 16);
    if (a.wr) {
        if (warp < kNC && r_e < a.E)
            for (int l = lane; l < H * 2 / 128; l += 32)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(a.wr + (size_t)r_e * H) + 128 * l));
        for (int v = tid; v < T * H / 8; v += blockDim.x) rx[v] = __ldg(reinterpret_cast<const uint4*>(a.x) + v);
    }
    __syncthreads();
    if (trace && tid == 0) trace[1] = globaltimer();

    // ---- the slot lookup's outputs (slot_of, tickets) are needed from here on
    pdl_wait();
    pdl_trigger();   // the next kernel may launch; it waits for this grid to finish
    if (trace && tid == 0) trace[2] = globaltimer();

    // ---- fused router: fp32 logits in the router kernel's order (lane j sums, by
    // fmaf in ascending h, the 8-element chunks c with c % 32 == j; then a xor
    // butterfly 16 .. 1; the bias last), exchanged through global memory
    if (a.wr) {
        if (warp < kNC && r_e < a.E) {
            float acc[kMaxDecodeT];
#pragma unroll
            for (int t = 0; t < kMaxDecodeT; t++) acc[t] = 0.0f;
            const uint4* wrow = reinterpret_cast<const uint4*>(a.wr + (size_t)r_e * H);
            // chunks c = lane + 32 q in ascending q, four loads of W in flight at a time
            for (int q0 = 0; q0 < H / 256; q0 += 4) {
                uint4 wq[4];
#pragma unroll
                for (int i = 0; i < 4; i++) wq[i] = q0 + i < H / 256 ? __ldg(wrow + lane + 32 * (q0 + i)) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    if (q0 + i >= H / 256) break;
                    const int c = lane + 32 * (q0 + i);
                    const uint32_t wu[4] = {wq[i].x, wq[i].y, wq[i].z, wq[i].w};
#pragma unroll
                    for (int t = 0; t < kMaxDecodeT; t++) {
                        if (t >= T) break;
                        const uint4 xq = rx[(size_t)t * (H / 8) + c];
                        const uint32_t xu[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
                        for (int r = 0; r < 4; r++) {
                            acc[t] = fmaf(__uint_as_float(xu[r] << 16), __uint_as_float(wu[r] << 16), acc[t]);
                            acc[t] = fmaf(__uint_as_float(xu[r] & 0xFFFF0000u), __uint_as_float(wu[r] & 0xFFFF0000u),
                                          acc[t]);
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < kMaxDecodeT; t++) {
                if (t >= T) break;
                float v = acc[t];
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) v = v + __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) a.rlogits[(size_t)t * a.E + r_e] = v + (a.rbias ? a.rbias[r_e] : 0.0f);
            }
            __syncwarp();
            if (lane == 0) red_release_add(route_ctr, 1u);
        }
        if (tid == 0 && !wait_count(route_ctr, (unsigned)a.E, a.dep_ns, abort_flag)) {
            atomicOr(a.status, MOE_STATUS_DEP_TIMEOUT);
            *abort_flag = 1;
        }
        __syncthreads();
        // top-k of token t by warp t (the stage ring is still unused: its first
        // bytes hold the logits rows and the taken flags)
        float* s_l = reinterpret_cast<float*>(stages) + (size_t)warp * a.E;
        unsigned char* s_taken = stages + (size_t)kNC * a.E * 4 + (size_t)warp * a.E;
        if (warp < T) {
            for (int e = lane; e < a.E; e += 32) s_l[e] = __ldcg(a.rlogits + (size_t)warp * a.E + e);
            __syncwarp();
            router_topk_warp(s_l, s_taken, a.E, a.k, a.renorm, lane, ridx + warp * a.k, rw + warp * a.k);
            if (blockIdx.x == 0 && lane < a.k) {
                a.idx_out[warp * a.k + lane] = ridx[warp * a.k + lane];
                a.w_out[warp * a.k + lane] = rw[warp * a.k + lane];
            }
        }
        __syncthreads();
    }

    // ---- prologue 2: the groups (unique experts) of the call, in ticket order.
    // The stage ring is still unused, so its first bytes hold the per-(token, rank)
    // scratch.
    int* e_s = reinterpret_cast<int*>(stages);            // [n] expert or -1
    int* s_s = e_s + kMaxDecodePairs;                      // [n] slot
    unsigned* need_s = reinterpret_cast<unsigned*>(s_s + kMaxDecodePairs);
    int* lead_s = reinterpret_cast<int*>(need_s + kMaxDecodePairs);   // first entry of my expert
    int* mi_s = lead_s + kMaxDecodePairs;                  // my index inside the group
    int* gm_s = mi_s + kMaxDecodePairs;                    // members of a leader's group
    int* rdy_s = gm_s + kMaxDecodePairs;                   // slot shows the needed ticket
    int* lpos_s = rdy_s + kMaxDecodePairs;                 // [leaders] entry of each leader
    int* grank_s = lpos_s + kMaxDecodePairs;               // group rank of a leader
    unsigned long long* lkey_s = reinterpret_cast<unsigned long long*>(grank_s + kMaxDecodePairs);  // [leaders]
    const int n = T * a.k;
    if (tid == 0) s_misc[0] = 0;
    if (tid < n) {
        const int e = a.wr ? ridx[tid] : a.idx[tid];
        int bad = 0;
        if (e < 0 || e >= a.E) bad |= MOE_STATUS_BAD_EXPERT;
        int sl = -1;
        if (!a.resident) sl = a.slot_of[tid];
        else if (!bad) sl = a.key_slot[(size_t)a.layer * a.E + e];
        if (a.resident && !bad && sl < 0) bad |= MOE_STATUS_NOT_RESIDENT;
        if (sl < 0 || sl >= a.S) bad |= MOE_STATUS_BAD_SLOT;
        if (a.resident && blockIdx.x == 0) a.slot_of[tid] = sl;
        uint32_t nd = 0u, rd = 1u;
        if (!bad) {
            nd = a.need[sl];
            rd = ld_acquire_gpu_u32(a.ready + sl);
        }
        e_s[tid] = bad ? -1 : e;
        s_s[tid] = sl;
        need_s[tid] = nd;
        rdy_s[tid] = ((rd & ~kTicketPartA) == nd) | ((rd == nd) << 1);
        gm_s[tid] = 0;
        if (bad && blockIdx.x == 0) atomicOr(a.status, bad);
    }
    __syncthreads();
    // the producer's bulk (async proxy) reads of slots acquired above come after
    // this fence; issued here, it overlaps the rest of the table
    if (warp == kNC) fence_proxy_async_global();
    // leader (first entry of the same expert) and index among the expert's
    // entries, by one scan of the earlier entries (broadcast loads)
    if (tid < n && e_s[tid] >= 0) {
        const int e = e_s[tid];
        int lead = tid, mi = 0;
#pragma unroll 8
        for (int j = 0; j < tid; j++) {
            const bool same = e_s[j] == e;
            lead = same && j < lead ? j : lead;
            mi += same;
        }
        lead_s[tid] = lead;
        mi_s[tid] = mi;
        atomicAdd(gm_s + lead, 1);
        if (lead == tid) {
            const int li = atomicAdd(s_misc, 1);
            lkey_s[li] = ((unsigned long long)need_s[tid] << 32) | (unsigned)e;
            lpos_s[li] = tid;
        }
    }
    __syncthreads();
    // groups ranked by (ticket the slot must show, expert): resident experts come
    // first and missed ones in the order the copy engine delivers them
    const int nl = s_misc[0];
    if (tid < nl) {
        const unsigned long long key = lkey_s[tid];
        int rank = 0, erank = 0;
#pragma unroll 8
        for (int j = 0; j < nl; j++) {
            rank += lkey_s[j] < key;
            erank += (unsigned)lkey_s[j] < (unsigned)key;
        }
        if (a.resident && blockIdx.x == 0) {
            // the lookup's touch of the hits: ascending expert id, clock = G0 + 1 + rank
            a.slot_clock[s_s[lpos_s[tid]]] = *a.clock + 1 + erank;
        }
        const int ld = lpos_s[tid], e = e_s[ld];
        grank_s[ld] = rank;
        Group& G = groups[rank];
        G.expert = e;
        G.slot = s_s[ld];
        G.M = gm_s[ld];
        G.ready_a = rdy_s[ld] & 1;
        G.ready_b = rdy_s[ld] >> 1;
        G.need = need_s[ld];
        G.ts[0] = ts_row[3 * e];
        G.ts[1] = ts_row[3 * e + 1];
        G.ts[2] = ts_row[3 * e + 2];
    }
    __syncthreads();
    if (tid < n && e_s[tid] >= 0) {
        Group& G = groups[grank_s[lead_s[tid]]];
        G.tok[mi_s[tid]] = (uint8_t)(tid / a.k);
        G.rank[mi_s[tid]] = (uint8_t)(tid % a.k);
        G.wt[mi_s[tid]] = a.wr ? rw[tid] : a.w[tid];
    }
    __syncthreads();
    const int ng = s_misc[0];
    if (a.resident && blockIdx.x == 0 && tid == 0) *a.clock += (unsigned long long)ng;
    if (trace && tid == 0) trace[3] = globaltimer();

    // ---- this CTA's work: A items [a0, a1) and B tiles [b0, b1) of the call's
    // lists (group-major, in ticket order); B stages are runs of up to TRB tiles
    // of one group
    const int P = gridDim.x, cta = blockIdx.x;
    const int NAi = ng * nTA, NBt = ng * nTB;
    const int a0 = (int)((long long)cta * NAi / P), a1 = (int)((long long)(cta + 1) * NAi / P);
    const int b0 = (int)((long long)cta * NBt / P), b1 = (int)((long long)(cta + 1) * NBt / P);
    const int nA = a1 - a0;
    auto bstage = [&](int i, int& g, int& r, int& nt) {
        g = i / nTB;
        r = i - g * nTB;
        nt = min(a.TRB, min(b1 - i, nTB - r));
    };

    if (warp == kNC) {
        // ---------------------------------------------------------------- producer
        int st = 0, issued = 0, lastg = -1, lastpart = 0;
        uint32_t round = 0;
        const uint8_t* blk = nullptr;
        // first use of a group's slot for gate/up (part 0) or down (part 1): a slot
        // that showed that part when the table was built was acquired then (the
        // CTA barrier and the proxy fence after it order the bulk reads); for a
        // pending one, wait (bounded) for the part's ticket, acquire it and fence
        // here.
        if (trace && lane == 0) trace[9] = globaltimer();
        auto use_group = [&](int g, int part) {
            if (g == lastg && part == lastpart) return;
            lastg = g;
            lastpart = part;
            const Group& G = groups[g];
            if (!(part ? G.ready_b : G.ready_a)) {
                bool ok = true;
                if (lane == 0)
                    ok = wait_ready(a.ready + G.slot, G.need, part ? 0xFFFFFFFFu : ~kTicketPartA, a.ready_ns,
                                    abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok && lane == 0) {
                    atomicOr(a.status, MOE_STATUS_READY_TIMEOUT);
                    *abort_flag = 1;
                }
                (void)ld_acquire_gpu_u32(a.ready + G.slot);
                fence_proxy_async_global();
            }
            blk = a.slots + (unsigned long long)G.slot * a.block_bytes;
        };
        auto take_slot = [&](uint32_t tx) -> uint8_t* {
            bool ok = true;
            if (lane == 0) ok = mbar_wait_abort(&empty[st], (round & 1) ^ 1, a.pipe_ns, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok && lane == 0) {
                atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
                *abort_flag = 1;
            }
            if (lane == 0) mbar_arrive_expect_tx(&full[st], tx);
            __syncwarp();
            return stages + (size_t)st * a.stage_bytes;
        };
        auto advance = [&]() {
            if (trace && lane == 0 && issued < 8) trace[24 + issued] = globaltimer();
            issued++;
            if (++st == a.nstage) {
                st = 0;
                round++;
            }
        };
        // A item: 16 rows of gate and the same rows of up, codes then scales
        for (int i = a0; i < a1; i++) {
            const int g = i / nTA, t = i - g * nTA;
            use_group(g, 0);
            uint8_t* dst = take_slot(2 * CA + 2 * 16 * SA);
            const unsigned long long r0 = (unsigned long long)t * 16;
            if (lane == 0) bulk_g2s(dst, blk + a.off[0] + r0 * (H / 2), CA, &full[st]);
            if (lane == 1) bulk_g2s(dst + CA, blk + a.off[2] + r0 * (H / 2), CA, &full[st]);
            if (lane == 2) bulk_g2s(dst + 2 * CA, blk + a.off[1] + r0 * SA, 16 * SA, &full[st]);
            if (lane == 3) bulk_g2s(dst + 2 * CA + 16 * SA, blk + a.off[3] + r0 * SA, 16 * SA, &full[st]);
            advance();
        }
        // B stage: nt * 16 rows of down, codes then scales
        for (int i = b0; i < b1;) {
            int g, r, nt;
            bstage(i, g, r, nt);
            i += nt;
            use_group(g, 1);
            const uint32_t cb = (uint32_t)nt * 16 * (I / 2), sbb = (uint32_t)nt * 16 * SB;
            uint8_t* dst = take_slot(cb + sbb);
            const unsigned long long r0 = (unsigned long long)r * 16;
            if (lane == 0) bulk_g2s(dst, blk + a.off[4] + r0 * (I / 2), cb, &full[st]);
            if (lane == 1) bulk_g2s(dst + cb, blk + a.off[5] + r0 * SB, sbb, &full[st]);
            advance();
        }
        if (trace && lane == 0) trace[11] = globaltimer();
        // no copy may still be in flight when the CTA exits: wait (bounded) for
        // the last phase of every stage used
        if (lane == 0)
            for (int j = (issued > a.nstage ? issued - a.nstage : 0); j < issued; j++)
                if (!mbar_wait(&full[j % a.nstage], (uint32_t)(j / a.nstage) & 1, a.pipe_ns))
                    atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
    } else {
        // ---------------------------------------------------------------- consumers
        // A item = 16 rows of gate and the same 16 rows of up.  Unit u = warp /
        // (2 ks) takes the CTA's A items u, u + nAU, ...: its even warps the gate
        // tile, its odd ones the up tile, each over 1/ks of K (part kp); the unit
        // then sums the parts in order, forms h and stores it to global memory,
        // counting the values it publishes per group.
        // B stage = up to TRB tiles of 16 down rows: a group of TRB * kb warps takes
        // B stages group, group + nBU, ..., each tile over 1/kb of K per warp (the
        // kb parts summed in order), once every h value of the stage's group is
        // published.
        // nAU and nBU divide the ring size, so within a phase every slot is filled
        // and emptied for one unit (or group) only, in order: a wait never meets a
        // slot whose earlier fill is still pending (whose phase parity would
        // alias).  Consumer barriers separate the phases.
        const int g8 = lane >> 2, q = lane & 3;
        const uint32_t qs = FMT == MOE_NVFP4 ? 2 * q : 0;   // the thread's scale bytes in a row's segment
        const int bstride = 4 * T;                         // pieces between the words j of a segment
        // the K split with the fewest rounds for this CTA's A items (one round =
        // an item's full-K dot products / ks), a little weight against more warps
        // meeting at every item
        int ks = 1, nAU = 1;
        {
            float best = 1e30f;
            for (int c = 1; c <= kNC / 2; c *= 2) {
                if (nsegA % c) continue;
                int u = min(kNC / (2 * c), a.nstage);
                while (a.nstage % u) u--;
                const float cost = (float)((nA + u - 1) / u) / (float)c + 0.05f * (float)c;
                if (cost < best) {
                    best = cost;
                    ks = c;
                    nAU = u;
                }
            }
        }
        const int uw = 2 * ks, unit = warp / uw, widx = warp - unit * uw;
        const int role = widx & 1, kp = widx >> 1, segsA = nsegA / ks;
        // B: the K split kb (1, 2, 4) with the fewest rounds for this CTA's stages
        const int TRB = a.TRB;
        int nbst = 0;
        for (int i = b0; i < b1; nbst++) {
            int g, r, nt;
            bstage(i, g, r, nt);
            i += nt;
        }
        int kb = 1, nBU = 1;
        {
            float best = 1e30f;
            for (int c = 1; c <= 4 && TRB * c <= kNC; c *= 2) {
                if (nsegB % c) continue;
                int u = min(kNC / (TRB * c), a.nstage);
                while (a.nstage % u) u--;
                const float cost = (float)((nbst + u - 1) / u) / (float)c + 0.05f * (float)c;
                if (cost < best) {
                    best = cost;
                    kb = c;
                    nBU = u;
                }
            }
        }
        const int gw = TRB * kb, grp = warp / gw, bw = warp - grp * gw;
        const int tile = bw % TRB, bkp = bw / TRB, segsB = nsegB / kb;
        if (trace && tid == 0) {
            trace[12] = (unsigned long long)nA;
            trace[13] = (unsigned long long)(b1 - b0);
            trace[14] = (unsigned long long)ks;
            trace[15] = (unsigned long long)kb;
        }
        auto slot_wait = [&](int k) {
            if (!mbar_wait_abort(&full[k % a.nstage], (uint32_t)(k / a.nstage) & 1, a.pipe_ns, abort_flag)) {
                if (lane == 0) atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
                *abort_flag = 1;
            }
        };
        // the empty barrier counts kNC arrivals per stage: each of the n warps of a stage gives kNC / n
        auto slot_release = [&](int k, int n) {
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0], %1;"
                             ::"r"(smem_addr(&empty[k % a.nstage])), "r"(kNC / n) : "memory");
        };
        int k = 0, pst = 0;                                // stage index, unit stages done

        // ---- A
        for (int s = 0; s < nA; s++, k++) {
            if (unit >= nAU || s % nAU != unit) continue;
            const int i = a0 + s, g = i / nTA, t = i - g * nTA;
            const Group& G = groups[g];
            const int M = G.M;
            slot_wait(k);
            if (trace && tid == 0 && s == 0) trace[4] = globaltimer();
            if (trace && lane == 0 && widx == 0 && s < 8) trace[16 + s] = globaltimer();
            const uint8_t* sb = stages + (size_t)(k % a.nstage) * a.stage_bytes;
            const uint8_t* tb = sb + role * CA;                       // gate or up codes
            const uint8_t* tsc = sb + 2 * CA + role * 16 * SA;        // their scale rows
            const uint4* xb[1][NT];                                   // x of the member's token
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                const int m = g8 + 8 * nt;
                xb[0][nt] = m < M ? xf + (size_t)G.tok[m] * 4 + q : nullptr;
            }
            float part[NT][4];
            tile_mma<FMT, NT, 1>(tb + g8 * (H / 2) + 16 * q, 8 * (H / 2), tsc + g8 * SA + qs, 8 * SA, q,
                                 kp * segsA, segsA, xb, bstride, part);
            slot_release(k, uw);
            // the unit's parts: [parity][role][kp][16][T]
            float* ub = unitbuf + (size_t)unit * 2 * 2 * ks * 16 * T + (size_t)(pst & 1) * 2 * ks * 16 * T;
            float* pb = ub + (size_t)(role * ks + kp) * 16 * T;
#pragma unroll
            for (int nt = 0; nt < NT; nt++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int rr = g8 + (e >> 1) * 8, m = 8 * nt + 2 * q + (e & 1);
                    if (m < M) pb[rr * T + m] = part[nt][e];
                }
            named_sync(2 + unit, 32 * uw);
            int cnt = 0;
            // o = 16 m + row: each half-warp holds the 16 rows of one member
            for (int base = widx * 32; base < 16 * M; base += 32 * uw) {
                const int o = base + lane, rr = o & 15, m = o >> 4;
                float hv = 0.0f;
                int pair = 0;
                if (o < 16 * M) {
                    float gs = ub[rr * T + m], us = ub[(size_t)ks * 16 * T + rr * T + m];
                    for (int p = 1; p < ks; p++) {
                        gs += ub[(size_t)p * 16 * T + rr * T + m];
                        us += ub[(size_t)(ks + p) * 16 * T + rr * T + m];
                    }
                    const float xs = xinv[G.tok[m]];               // undo x's scale
                    const float gv = gs * xs * G.ts[0], uv = us * xs * G.ts[1];
                    hv = gv / (1.0f + expf(-gv)) * uv;
                    pair = G.tok[m] * a.k + G.rank[m];
                    a.hbuf[(size_t)pair * I + t * 16 + rr] = hv;
                    cnt++;
                }
                float mx = fabsf(hv);
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                if ((lane & 15) == 0 && o < 16 * M) atomicMax(pmax + pair, __float_as_uint(mx));
            }
            // publish: the warp's h values and maxima are visible before the group's
            // count grows (the warp barrier orders the lanes' writes before lane 0's
            // release add)
            cnt = __reduce_add_sync(0xffffffffu, cnt);
            __syncwarp();
            if (lane == 0 && cnt) red_release_add(gcnt + g, (unsigned)cnt);
            pst++;
        }
        named_sync(1, kConsThreads);      // x fragments are dead from here on
        if (trace && tid == 0) trace[5] = globaltimer();

        // ---- B
        int curg = -1, nbs = 0, bps = 0;
        const uint4* hb2[2][NT] = {};     // h of the member: high parts, remainders
        for (int i = b0; i < b1; nbs++, k++) {
            int g, r, nt;
            bstage(i, g, r, nt);
            i += nt;
            const Group& G = groups[g];
            const int M = G.M;
            if (g != curg) {
                // a new group: every warp is done with the previous fragments; wait
                // (bounded) until all I * M values of its h (and their maxima) are
                // published, then scale each member's h by a power of two and split
                // it into f16 high parts and remainders
                curg = g;
                named_sync(1, kConsThreads);
                if (tid == 0) {
                    if (!wait_count(gcnt + g, (unsigned)(I * M), a.dep_ns, abort_flag)) {
                        atomicOr(a.status, MOE_STATUS_DEP_TIMEOUT);
                        *abort_flag = 1;
                    }
                    if (trace && nbs == 0) trace[6] = globaltimer();
                }
                named_sync(1, kConsThreads);
                if (tid < M) hinv[tid] = 1.0f / act_scale(__uint_as_float(__ldcg(pmax + G.tok[tid] * a.k + G.rank[tid])));
                for (int v = tid; v < M * (I / 8); v += kConsThreads) {
                    const int m = v / (I / 8), k0 = (v - m * (I / 8)) * 8;
                    const int pair = G.tok[m] * a.k + G.rank[m];
                    const float4* src = reinterpret_cast<const float4*>(a.hbuf + (size_t)pair * I + k0);
                    const float4 u0 = __ldcg(src), u1 = __ldcg(src + 1);
                    const float sc = act_scale(__uint_as_float(__ldcg(pmax + pair)));
                    const float hv[8] = {u0.x * sc, u0.y * sc, u0.z * sc, u0.w * sc,
                                         u1.x * sc, u1.y * sc, u1.z * sc, u1.w * sc};
                    float hi[8], lo[8];
#pragma unroll
                    for (int j = 0; j < 8; j++) {
                        hi[j] = __half2float(__float2half_rn(hv[j]));
                        lo[j] = hv[j] - hi[j];                 // exact in fp32
                    }
                    const int pi = piece_index(k0, m, T);
                    hf_hi[pi] = pack_piece(hi);
                    hf_lo[pi] = pack_piece(lo);
                }
                named_sync(1, kConsThreads);
                if (trace && tid == 0 && nbs == 0) trace[7] = globaltimer();
#pragma unroll
                for (int n8 = 0; n8 < NT; n8++) {
                    const int m = g8 + 8 * n8;
                    hb2[0][n8] = m < M ? hf_hi + (size_t)m * 4 + q : nullptr;
                    hb2[1][n8] = m < M ? hf_lo + (size_t)m * 4 + q : nullptr;
                }
            }
            if (grp >= nBU || nbs % nBU != grp) continue;
            slot_wait(k);
            if (trace && lane == 0 && bw == 0 && nA + nbs < 8) trace[16 + nA + nbs] = globaltimer();
            float acc[NT][4];
            if (tile < nt) {
                const uint8_t* sb = stages + (size_t)(k % a.nstage) * a.stage_bytes;
                const uint32_t cb = (uint32_t)nt * 16 * (I / 2);
                const int row = tile * 16 + g8;
                tile_mma<FMT, NT, 2>(sb + row * (I / 2) + 16 * q, 8 * (I / 2), sb + cb + row * SB + qs, 8 * SB, q,
                                     bkp * segsB, segsB, hb2, bstride, acc);
            }
            slot_release(k, gw);    // every warp of the group arrives, with a tile or without
            if (kb > 1) {
                // the group's parts: [parity][tile][kp][16][T]; part 0's warp sums them
                float* gb = unitbuf + ((size_t)grp * 2 + (bps & 1)) * TRB * kb * 16 * T;
                if (tile < nt) {
#pragma unroll
                    for (int n8 = 0; n8 < NT; n8++)
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            const int rr = g8 + (e >> 1) * 8, m = 8 * n8 + 2 * q + (e & 1);
                            if (m < M) gb[((size_t)(tile * kb + bkp) * 16 + rr) * T + m] = acc[n8][e];
                        }
                }
                named_sync(2 + grp, 32 * gw);
                bps++;
                if (bkp != 0 || tile >= nt) continue;
#pragma unroll
                for (int n8 = 0; n8 < NT; n8++)
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int rr = g8 + (e >> 1) * 8, m = 8 * n8 + 2 * q + (e & 1);
                        if (m < M) {
                            float v = gb[((size_t)(tile * kb) * 16 + rr) * T + m];
                            for (int p2 = 1; p2 < kb; p2++) v += gb[((size_t)(tile * kb + p2) * 16 + rr) * T + m];
                            acc[n8][e] = v;
                        }
                    }
            } else if (tile >= nt) {
                continue;
            }
            const int rt = r + tile;                                   // row tile of H
#pragma unroll
            for (int n8 = 0; n8 < NT; n8++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    const int rr = g8 + (e >> 1) * 8, m = 8 * n8 + 2 * q + (e & 1);
                    if (m < M)
                        a.y_part[((size_t)G.tok[m] * a.k + G.rank[m]) * H + rt * 16 + rr] =
                            G.wt[m] * (acc[n8][e] * hinv[m] * G.ts[2]);
                }
            if (!a.y) continue;
            // the row tile's part from this group is in y_part: count it (release)
            __syncwarp();
            if (lane == 0) red_release_add(rowcnt + rt, 1u);
        }
        if (trace && tid == 0) trace[8] = globaltimer();

        // ---- K5: CTA c sums the 16-row tiles rt = c, c + grid, ... of H over the
        // ranks in rank order and writes their bf16 rows, once every group has
        // counted them (bounded wait, acquire); the work is spread over the grid
        if (a.y) {
            for (int rt = blockIdx.x; rt < H / 16; rt += gridDim.x) {
                if (tid == 0 && !wait_count(rowcnt + rt, (unsigned)ng, a.dep_ns, abort_flag)) {
                    atomicOr(a.status, MOE_STATUS_DEP_TIMEOUT);
                    *abort_flag = 1;
                }
                named_sync(1, kConsThreads);
                for (int v = tid; v < T * 16; v += kConsThreads) {
                    const int t = v >> 4, row = rt * 16 + (v & 15);
                    float sum = 0.0f;
                    for (int j = 0; j < a.k; j++) sum += __ldcg(a.y_part + ((size_t)t * a.k + j) * H + row);
                    a.y[(size_t)t * H + row] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
                }
            }
        }
    }

    // ---- epilogue: the last CTA to finish clears the launch's counters and the
    // abort flag for the next launch (every other CTA is done with them)
    __syncthreads();
    if (trace && tid == 0) trace[10] = globaltimer();
    if (tid == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(done_ctr, 1u);
        s_misc[2] = prev == gridDim.x - 1;
        if (s_misc[2]) __threadfence();
    }
    __syncthreads();
    if (s_misc[2]) {
        for (int i = tid; i < H / 16; i += blockDim.x) rowcnt[i] = 0u;
        for (int i = tid; i < 2 * kMaxDecodePairs; i += blockDim.x) gcnt[i] = 0u;   // counts and maxima
        if (tid == 0) *route_ctr = 0u;
        __syncthreads();
        if (tid == 0) {
            *abort_flag = 0u;
            *done_ctr = 0u;
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

static size_t up(size_t n, size_t a) { return (n + a - 1) / a * a; }

// Shared-memory layout, ring and B stage shape of a launch with T tokens.
static int plan_ffn(const moe_pool* p, int T, FfnArgs& a, size_t& smem, bool fused_router) {
    const moe_config& c = p->cfg;
    const int bs = p->bs;
    const size_t SA = c.H / bs, SB = c.I / bs;
    const size_t budget = (size_t)p->ffn_smem;
    const size_t stA = 2 * (size_t)16 * (c.H / 2) + 2 * (size_t)16 * SA;
    const size_t rowB = c.I / 2 + SB;
    // B stages: the most 16-row tiles (8, 4, 2 or 1) that fit an A stage (or one tile)
    a.TRB = 1;
    for (int t = 8; t >= 1; t >>= 1)
        if ((size_t)t * 16 * rowB <= std::max(stA, 16 * rowB)) {
            a.TRB = t;
            break;
        }
    a.stage_bytes = (int)up(std::max(stA, (size_t)a.TRB * 16 * rowB), 128);
    size_t o = up((2 * 8) * sizeof(uint64_t), 128);
    a.o_groups = (int)o;
    o += sizeof(Group) * std::min(kMaxDecodePairs, c.max_tokens * c.k);
    a.o_misc = (int)up(o, 16);
    o = a.o_misc + 3 * kMaxDecodeT * sizeof(float) + 8 * sizeof(int) + 2 * kMaxDecodePairs * 4;
    a.o_ts = (int)up(o, 16);
    o = a.o_ts + (size_t)c.E * 3 * sizeof(float);
    a.o_red = (int)up(o, 16);
    o = a.o_red + (size_t)(kNC / 2) * 2 * 2 * 16 * T * sizeof(float);   // units * ks <= kNC / 2
    a.o_frag = (int)up(o, 16);
    o = a.o_frag + std::max((size_t)T * c.H * 2, (size_t)2 * T * c.I * 2);
    a.o_stage = (int)up(o, 128);
    // the prologue keeps its per-(token, rank) table (9 ints + a u64 each) in the ring
    // (and the fused router its logits rows and flags, kNC * E * 5 bytes, then x)
    const size_t need_ring = std::max({(size_t)2 * a.stage_bytes, (size_t)11 * 4 * kMaxDecodePairs,
                                       fused_router ? up((size_t)kNC * c.E * 5, 16) + (size_t)T * c.H * 2 : 0});
    if (a.o_stage + need_ring > budget)
        return fail(MOE_EINVAL, "decode FFN: T * H too large for shared memory (lower max_tokens)");
    // a power of two (at most 8), so that 2, 4 or 8 consumer units can share the ring
    const int fit = (int)std::min<size_t>(8, (budget - a.o_stage) / a.stage_bytes);
    a.nstage = 1;
    while (a.nstage * 2 <= fit) a.nstage *= 2;
    smem = a.o_stage + (size_t)a.nstage * a.stage_bytes;
    return MOE_OK;
}

// One CTA per SM; every CTA must be resident at once (B tiles wait for A items
// of other CTAs), so the grid is what the occupancy calculator allows.
template <int FMT, int NT>
static int ffn_grid(moe_pool* p, int& grid) {
    auto kern = ffn_decode_kernel<FMT, NT>;
    const int fi = FMT == MOE_NVFP4, ni = NT - 1;
    if (!p->ffn_grid[fi][ni]) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p->ffn_smem));
        int per_sm = 0;
        MOE_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFfnThreads, p->ffn_smem));
        if (per_sm < 1) return fail(MOE_ECUDA, "decode FFN: no CTA fits on an SM");
        p->ffn_grid[fi][ni] = p->num_sms;   // one per SM: more would only wait
    }
    grid = p->ffn_grid[fi][ni];
    // the SM copy kernel streams misses the FFN waits for: leave it SMs of its own
    if (p->copy_mode == MOE_COPY_SM) grid = std::max(1, grid - kCopySMs);
    return MOE_OK;
}

template <int FMT, int NT>
static int launch_ffn(moe_pool* p, FfnArgs& a, cudaStream_t s) {
    size_t smem = 0;
    int grid = 0;
    int rc = ffn_grid<FMT, NT>(p, grid);
    if (rc) return rc;
    rc = plan_ffn(p, a.T, a, smem, a.wr != nullptr);
    if (rc) return rc;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(grid);
    lc.blockDim = dim3(kFfnThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    // programmatic serialisation: the activations are staged while the slot
    // lookup before this kernel finishes (the kernel waits for it before reading
    // slot_of, the tickets and the tensor scales)
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    MOE_CUDA_TRY(cudaLaunchKernelEx(&lc, ffn_decode_kernel<FMT, NT>, a));
    return MOE_OK;
}

int preload_ffn_kernels() {
    cudaFuncAttributes fa;
#define PRELOAD(F)                                                           \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, ffn_decode_kernel<F, 1>));       \
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, ffn_decode_kernel<F, 2>));       \
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

extern "C" int moe_ffn_launch_info(moe_pool* p, int T, int* ctas, int* nstage, int* stage_bytes, int* smem_bytes) {
    if (!p || !ctas || !nstage || !stage_bytes || !smem_bytes) return fail(MOE_EINVAL, "null argument");
    if (T <= 0 || T > p->cfg.max_tokens) return fail(MOE_EINVAL, "T must be in [1, max_tokens]");
    FfnArgs a{};
    size_t smem = 0;
    int grid = 0, rc;
    if (p->cfg.fmt == MOE_NVFP4)
        rc = T <= 8 ? ffn_grid<MOE_NVFP4, 1>(p, grid) : ffn_grid<MOE_NVFP4, 2>(p, grid);
    else
        rc = T <= 8 ? ffn_grid<MOE_MXFP4, 1>(p, grid) : ffn_grid<MOE_MXFP4, 2>(p, grid);
    if (rc) return rc;
    rc = plan_ffn(p, T, a, smem, false);
    if (rc) return rc;
    *ctas = grid;
    *nstage = a.nstage;
    *stage_bytes = a.stage_bytes;
    *smem_bytes = (int)smem;
    return MOE_OK;
}

extern "C" int moe_set_wait_limits(double ready_ms, double dep_ms, double pipe_ms) {
    if (!(ready_ms > 0) || !(dep_ms > 0) || !(pipe_ms > 0)) return fail(MOE_EINVAL, "wait limits must be positive");
    g_ready_ns = (unsigned long long)(ready_ms * 1e6);
    g_dep_ns = (unsigned long long)(dep_ms * 1e6);
    g_pipe_ns = (unsigned long long)(pipe_ms * 1e6);
    return MOE_OK;
}

namespace moe {

int expert_ffn(moe_pool* p, int layer, const void* x_bf16, int T, const int32_t* idx, const float* w,
               const int32_t* slot_of, float* y_part, void* y_bf16, int* status, void* stream, int resident,
               const FfnRoute* route) {
    if (route && !resident) return fail(MOE_EINVAL, "decode FFN: the fused router needs resident mode");
    if (route && (!route->wr || !route->idx || !route->w)) return fail(MOE_EINVAL, "null argument");
    if (!p || !x_bf16 || !idx || !w || !slot_of || !y_part || !status) return fail(MOE_EINVAL, "null argument");
    const moe_config& c = p->cfg;
    if (layer < 0 || layer >= c.L) return fail(MOE_EBOUNDS, "layer outside the pool");
    if (T <= 0 || T > c.max_tokens) return fail(MOE_EINVAL, "decode FFN: T must be in [1, max_tokens]");
    if (((uintptr_t)x_bf16 | (uintptr_t)y_part | (uintptr_t)y_bf16) & 15)
        return fail(MOE_EINVAL, "decode FFN: x, y_part and y must be 16-byte aligned");
    FfnArgs a{};
    a.x = (const uint16_t*)x_bf16;
    a.idx = idx;
    a.w = w;
    a.slot_of = const_cast<int32_t*>(slot_of);   // written only in resident mode, whose caller owns it
    a.y_part = y_part;
    a.y = (uint16_t*)y_bf16;
    a.status = status;
    a.slots = p->slots;
    a.block_bytes = p->lay.bytes;
    for (int i = 0; i < 6; i++) a.off[i] = p->lay.off[i];
    a.tscale = p->tscale;
    a.need = p->need;
    a.ready = p->ready;
    a.ctr = p->ctr;
    a.hbuf = p->hbuf;
    a.resident = resident;
    if (route) {
        a.wr = (const uint16_t*)route->wr;
        a.rbias = route->bias;
        a.renorm = route->renormalize;
        a.rlogits = p->rlogits;
        a.idx_out = route->idx;
        a.w_out = route->w;
    }
    a.key_slot = p->key_slot;
    a.slot_clock = p->slot_clock;
    a.clock = p->clock;
    a.T = T;
    a.k = c.k;
    a.H = c.H;
    a.I = c.I;
    a.E = c.E;
    a.S = c.n_slots;
    a.layer = layer;
    a.ready_ns = g_ready_ns;
    a.dep_ns = g_dep_ns;
    a.pipe_ns = g_pipe_ns;
    a.trace = g_trace;
    cudaStream_t s = (cudaStream_t)stream;
    if (c.fmt == MOE_NVFP4) return T <= 8 ? launch_ffn<MOE_NVFP4, 1>(p, a, s) : launch_ffn<MOE_NVFP4, 2>(p, a, s);
    return T <= 8 ? launch_ffn<MOE_MXFP4, 1>(p, a, s) : launch_ffn<MOE_MXFP4, 2>(p, a, s);
}

}  // namespace moe

extern "C" int moe_expert_ffn(moe_pool* p, int layer, const void* x_bf16, int T, const int32_t* idx,
                              const float* w, const int32_t* slot_of, float* y_part, void* y_bf16, int* status,
                              void* stream) {
    return expert_ffn(p, layer, x_bf16, T, idx, w, slot_of, y_part, y_bf16, status, stream, 0, nullptr);
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
