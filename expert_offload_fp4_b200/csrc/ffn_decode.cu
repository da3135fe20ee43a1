// K4 decode expert FFN with the K5 combine fused in, and the slot dequantiser.
//
// Work split: one thread-block cluster of C CTAs (C = 16 where the GPU can
// co-schedule it) per unique expert ("group") of the call; clusters loop over
// the groups in ticket order (resident experts first, missed ones in the order
// the copy engine delivers them).  CTA rho of a cluster
//   A: computes rows [rho*I/C, (rho+1)*I/C) of gate and up for every token of the
//      group and its slice of h = silu(gate x) * (up x);
//   X: publishes the slice to the other CTAs of the cluster (an mbarrier arrive
//      in each peer's shared memory) and gathers the whole h from theirs
//      (distributed shared memory);
//   B: computes rows [rho*H/C, (rho+1)*H/C) of y_e = down h, weighted by the
//      routing weight of each (token, rank), into y_part.
// Every dependency stays inside the cluster, whose CTAs the hardware runs
// together, so no CTA ever waits for one that may not be resident.  The last
// CTA to finish a block of H/C rows (an atomic count over all groups) sums
// y_part over the ranks in rank order and writes the bf16 output rows (K5).
//
// Warp specialisation: warp 8 (the producer) streams the FP4 code rows and
// block scales of each work stage with 1-D bulk copies into a ring of
// shared-memory stages (mbarrier full/empty pairs; code rows padded so that the
// consumers' 16-byte reads are bank-conflict free); for a missed expert it first
// waits (bounded) for the slot's ready ticket written by the copy stream.
// Warps 0..7 (consumers) run the dot products on the tensor cores with
// mma.sync m16n8k16, f16 inputs and fp32 accumulation:
//  - weights: E2M1 codes decoded by integer ops to exact f16 values e2m1*2^-14,
//    multiplied (exactly) by their block scale in f16: the E4M3 scale itself
//    (NVFP4), or 2^(e - E) with E the largest E8M0 exponent of the row's
//    128-element segment (MXFP4; 2^(E-127) is applied to the segment's fp32 sum);
//  - activations: x of each token times a power of two (bf16 is exact in f16
//    that way); h of each (token, expert) times a power of two and split into
//    an f16 high part and an f16 remainder, so down h is carried to ~22 bits;
//  - products are exact, sums fp32; the K ranges of the 8 warps are added in
//    warp order, so results are reproducible.
#include <math.h>

#include "tcgen05.cuh"

namespace moe {

constexpr int kNC = 8;                       // consumer warps
constexpr int kFfnThreads = (kNC + 1) * 32;  // + one producer warp
constexpr int kConsThreads = kNC * 32;
// Register cap.  The 9 warps of a CTA spread over the SM's 4 sub-partitions, 3 on
// one of them, whose register file holds 16384 registers; one warp of the SM copy
// kernel (128 threads, at most 32 registers), which a waiting FFN may depend on,
// must fit beside them: 3 * 32 * 160 + 32 * 32 <= 16384.
constexpr int kFfnMaxRegs = 160;
constexpr int kAbortIdx = kMaxDecodePairs;   // ctr[kAbortIdx] = abort flag
constexpr int kDoneIdx = kMaxDecodePairs + 1;
constexpr int kMaxCluster = 16;
constexpr int kSeg = 128;                    // K elements per segment (64 code bytes)

struct Group {
    int expert, slot, M, ready;
    unsigned need;
    float ts[3];
    float wt[kMaxDecodeT];     // routing weight of each member (token, rank)
    uint8_t tok[kMaxDecodeT];
    uint8_t rank[kMaxDecodeT];
};

struct FfnArgs {
    // the pool's FP4 code rows as 2-D byte tensors (gate/up rows of H/2 bytes, down
    // rows of I/2), read in boxes 128 bytes wide with the 128-byte swizzle
    CUtensorMap map_a, map_b;
    const uint16_t* x;
    const int32_t* idx;
    const float* w;
    const int32_t* slot_of;
    float* y_part;
    uint16_t* y;               // bf16 output [T, H] (the fused combine), or null
    int* status;
    const uint8_t* slots;
    unsigned long long block_bytes;
    unsigned long long off[6];
    const float* tscale;
    const uint32_t* need;
    const uint32_t* ready;
    unsigned int* ctr;         // [0, C): per row-block group counts; abort, done
    int T, k, H, I, E, S, layer;
    int C;                     // CTAs per cluster
    int RA;                    // gate (and up) rows per A stage: 16 or 32
    int RB;                    // down rows per B stage: 16, 32, 64 or 128
    int rows_a, rows_b;        // map rows per slot block (block bytes / row bytes)
    int row_gate, row_up, row_down;   // map row of each tensor's first row inside a block
    int stage_bytes, nstage;
    // byte offsets in dynamic shared memory
    int o_groups, o_misc, o_red, o_hloc, o_x, o_h, o_stage;
    unsigned long long ready_ns, dep_ns, pipe_ns;
    unsigned long long* trace;   // optional [gridDim][16] phase stamps (ns), or null
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

// Eight values of one 16-byte piece (elements 0..7) as the f16x2 words of the
// fragment order (0,4), (2,6), (1,5), (3,7): the pairing decode_e2m1_x2 makes.
__device__ __forceinline__ uint4 pack_piece(const float (&f)[8]) {
    const __half2 w0 = __floats2half2_rn(f[0], f[4]), w1 = __floats2half2_rn(f[2], f[6]);
    const __half2 w2 = __floats2half2_rn(f[1], f[5]), w3 = __floats2half2_rn(f[3], f[7]);
    return make_uint4(*reinterpret_cast<const uint32_t*>(&w0), *reinterpret_cast<const uint32_t*>(&w1),
                      *reinterpret_cast<const uint32_t*>(&w2), *reinterpret_cast<const uint32_t*>(&w3));
}

// 8 E2M1 codes (one 32-bit word, element n in bits 4n..4n+3) to 4 f16x2 words,
// each value e2m1 * 2^-14 exactly: a code's magnitude bits go to f16 bits 11..9
// (exponent low bits and the top mantissa bit) and its sign to bit 15, so 2^-14
// scales every value, the E2M1 subnormal 0.5 included.  The f16 high bytes of
// the even elements (low nibbles) and of the odd ones are formed four at a time;
// byte moves then give the words (e0,e4), (e2,e6), (e1,e5), (e3,e7).
__device__ __forceinline__ void decode_word(uint32_t x, uint32_t& w0, uint32_t& w1, uint32_t& w2, uint32_t& w3) {
    const uint32_t ev = ((x << 1) & 0x0E0E0E0Eu) | ((x << 4) & 0x80808080u);   // bytes: e0 e2 e4 e6
    const uint32_t od = ((x >> 3) & 0x0E0E0E0Eu) | (x & 0x80808080u);          // bytes: e1 e3 e5 e7
    w0 = __byte_perm(ev, 0u, 0x2404);
    w1 = ev & 0xFF00FF00u;
    w2 = __byte_perm(od, 0u, 0x2404);
    w3 = od & 0xFF00FF00u;
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
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------- cluster plumbing

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t ncluster_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// All threads of all CTAs of the cluster (release / acquire at cluster scope).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_peer(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t peer_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(peer_bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;"
        " selp.u32 %0, 1, 0, p; }"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint4 ld_peer_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float ld_peer_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// Bounded wait on an mbarrier phase that also gives up as soon as another wait
// of the launch has raised the abort flag.
__device__ __forceinline__ bool mbar_wait_abort(uint64_t* bar, uint32_t parity, unsigned long long limit_ns,
                                                volatile unsigned int* abort_flag, bool cluster_scope = false) {
    if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (unsigned it = 0;; it++) {
        if (cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if ((it & 15) == 15) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit_ns) return false;
        }
    }
}

__device__ __forceinline__ bool wait_ready(const uint32_t* ready, uint32_t want, unsigned long long limit_ns,
                                           volatile unsigned int* abort_flag) {
    if (ld_acquire_sys_u32(ready) == want) return true;
    const unsigned long long t0 = globaltimer();
    while (true) {
        if (ld_acquire_sys_u32(ready) == want) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) return false;
        __nanosleep(64);
    }
}

// ------------------------------------------------------------------ tile math
//
// One 128-element K segment of TT 16-row tiles against NB B operands of NT
// 8-column tiles.  Thread (g = lane/4, q = lane%4) reads the 16 code bytes
// [64 s + 16 q, +16) of rows g and g+8 (elements 32q .. 32q+31 of the segment):
// word j of them feeds MMA k-tiles 2j and 2j+1.  Inside a k-tile the slots
// (2q, 2q+1, 2q+8, 2q+9) hold the elements (8j + p, 8j + 4 + p, 8j + 2 + p,
// 8j + 6 + p) of the thread's 32 (p = 0 for tile 2j, 1 for 2j+1): a fixed
// permutation of K that the B operands are stored in (see pack_piece), so the
// products and their sums are those of the plain dot product.
// B operand layout (16-byte pieces): piece (s, j, n, q) holds column n's
// elements 128 s + 32 q + 8 j + {0,4,2,6,1,5,3,7} at index ((4 s + j) * N + n) * 4 + q;
// bptr points at (s, 0, n, q) and bstride = 4 N pieces separates the j.
template <int FMT, int TT, int NT, int NB>
__device__ __forceinline__ void seg_mma(const uint8_t* const (&code)[TT], uint32_t row8_code,
                                        const uint8_t* const (&scl)[TT], uint32_t row8_scl, int q,
                                        const uint4* const (&bptr)[NB][NT], int bstride,
                                        float (&acc)[TT][NT][4]) {
    uint4 c[TT], c8[TT];
    uint32_t fa[TT], fb[TT], fa8[TT], fb8[TT];
    float post[TT], post8[TT];
#pragma unroll
    for (int t = 0; t < TT; t++) {
        c[t] = *reinterpret_cast<const uint4*>(code[t]);
        c8[t] = *reinterpret_cast<const uint4*>(code[t] + row8_code);
        if (FMT == MOE_NVFP4) {
            // the thread's two scales per row (blocks 2q, 2q+1 of the segment), exact in f16
            const uint32_t s = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(scl[t]));
            const uint32_t s8 = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(scl[t] + row8_scl));
            fa[t] = __byte_perm(s, 0u, 0x1010);
            fb[t] = __byte_perm(s, 0u, 0x3232);
            fa8[t] = __byte_perm(s8, 0u, 0x1010);
            fb8[t] = __byte_perm(s8, 0u, 0x3232);
        } else {
            // the 4 E8M0 exponents of the segment; the thread's block (q) relative to their max
            const uint32_t u = *reinterpret_cast<const uint32_t*>(scl[t]);
            const uint32_t u8 = *reinterpret_cast<const uint32_t*>(scl[t] + row8_scl);
            uint32_t m = __vmaxu4(u, u >> 8), m8 = __vmaxu4(u8, u8 >> 8);
            m = __vmaxu4(m, m >> 16) & 0xFFu;
            m8 = __vmaxu4(m8, m8 >> 16) & 0xFFu;
            const uint32_t f = f16_pow2((int)((u >> (8 * q)) & 0xFFu) - (int)m);
            const uint32_t f8 = f16_pow2((int)((u8 >> (8 * q)) & 0xFFu) - (int)m8);
            fa[t] = fb[t] = f | (f << 16);
            fa8[t] = fb8[t] = f8 | (f8 << 16);
            post[t] = e8m0_to_f32(m);
            post8[t] = e8m0_to_f32(m8);
        }
    }
    float sacc[TT][NT][4];
    if (FMT == MOE_MXFP4) {
#pragma unroll
        for (int t = 0; t < TT; t++)
#pragma unroll
            for (int n = 0; n < NT; n++)
#pragma unroll
                for (int e = 0; e < 4; e++) sacc[t][n][e] = 0.0f;
    }
#pragma unroll
    for (int j = 0; j < 4; j++) {
        uint4 bv[NB][NT];
#pragma unroll
        for (int b = 0; b < NB; b++)
#pragma unroll
            for (int n = 0; n < NT; n++)
                bv[b][n] = bptr[b][n] ? bptr[b][n][j * bstride] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int t = 0; t < TT; t++) {
            const uint32_t cw = j == 0 ? c[t].x : j == 1 ? c[t].y : j == 2 ? c[t].z : c[t].w;
            const uint32_t cw8 = j == 0 ? c8[t].x : j == 1 ? c8[t].y : j == 2 ? c8[t].z : c8[t].w;
            uint32_t r0, r1, r2, r3, s0, s1, s2, s3;
            decode_word(cw, r0, r1, r2, r3);
            decode_word(cw8, s0, s1, s2, s3);
            const uint32_t f = j < 2 ? fa[t] : fb[t], f8 = j < 2 ? fa8[t] : fb8[t];
            r0 = hmul2_u32(r0, f);
            r1 = hmul2_u32(r1, f);
            r2 = hmul2_u32(r2, f);
            r3 = hmul2_u32(r3, f);
            s0 = hmul2_u32(s0, f8);
            s1 = hmul2_u32(s1, f8);
            s2 = hmul2_u32(s2, f8);
            s3 = hmul2_u32(s3, f8);
#pragma unroll
            for (int n = 0; n < NT; n++)
#pragma unroll
                for (int b = 0; b < NB; b++) {
                    float (&d)[4] = FMT == MOE_MXFP4 ? sacc[t][n] : acc[t][n];
                    mma16816(d, r0, s0, r1, s1, bv[b][n].x, bv[b][n].y);
                    mma16816(d, r2, s2, r3, s3, bv[b][n].z, bv[b][n].w);
                }
        }
    }
    if (FMT == MOE_MXFP4) {
#pragma unroll
        for (int t = 0; t < TT; t++)
#pragma unroll
            for (int n = 0; n < NT; n++) {
                acc[t][n][0] = fmaf(sacc[t][n][0], post[t], acc[t][n][0]);
                acc[t][n][1] = fmaf(sacc[t][n][1], post[t], acc[t][n][1]);
                acc[t][n][2] = fmaf(sacc[t][n][2], post8[t], acc[t][n][2]);
                acc[t][n][3] = fmaf(sacc[t][n][3], post8[t], acc[t][n][3]);
            }
    }
}

// Index (16-byte pieces) of the B-operand piece holding elements k0 .. k0+7
// (k0 a multiple of 8) of column n, for N columns.
__device__ __forceinline__ int piece_index(int k0, int n, int N) {
    const int s = k0 >> 7, q = (k0 >> 5) & 3, j = (k0 >> 3) & 3;
    return ((s * 4 + j) * N + n) * 4 + q;
}

// Shared-memory byte offset of 16-byte chunk c (0..7) of row r in a box of 128-byte
// rows written with the 128-byte swizzle (the chunk index XOR the row's low 3 bits).
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// Row of a 16-row tile in shared memory that feeds MMA row i (0..15): rows 2p and
// 2p+1 of the MMA are read in the same shared-memory phase, so they go to rows p
// and p + 4, whose swizzled chunks sit in opposite halves of the banks.
__device__ __forceinline__ int tile_row(int i) { return (i & 8) | ((i & 1) << 2) | ((i & 7) >> 1); }

// Element e (0..3) of lane `lane`'s accumulator holding (row rr, column m) of a
// 16 x (8 NT) tile: rows g and g+8, columns 2q and 2q+1.
__device__ __forceinline__ int frag_slot(int rr, int m, int& lane) {
    const int ml = m & 7;
    lane = (rr & 7) * 4 + (ml >> 1);
    return (rr >> 3) * 2 + (ml & 1);
}

// ------------------------------------------------------------------ the kernel

template <int FMT, int NT>
__global__ void __maxnreg__(kFfnMaxRegs) ffn_decode_kernel(const __grid_constant__ FfnArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + a.nstage;
    uint64_t* hready = empty + a.nstage;                               // [2]
    Group* groups = reinterpret_cast<Group*>(smem + a.o_groups);
    float* xinv = reinterpret_cast<float*>(smem + a.o_misc);           // [16] per token
    float* hinv = xinv + kMaxDecodeT;                                  // [16] per member
    float* hsc = hinv + kMaxDecodeT;                                   // [16] per member
    int* s_misc = reinterpret_cast<int*>(hsc + kMaxDecodeT);           // [8]
    float* red = reinterpret_cast<float*>(smem + a.o_red);             // [2][kNC][2][NT][32][4]
    float* hloc = reinterpret_cast<float*>(smem + a.o_hloc);           // [2][T][I/C], then [2][T] maxima
    uint4* xf = reinterpret_cast<uint4*>(smem + a.o_x);                // x fragments, N = T
    uint4* hf_hi = reinterpret_cast<uint4*>(smem + a.o_h);             // h fragments, N = T
    uint4* hf_lo = hf_hi + (size_t)a.T * a.I / 8;
    // the 128-byte swizzle of the TMA boxes follows shared-memory address bits 7..9:
    // the stage ring starts on a 1024-byte boundary (the launch adds 1 KB of slack)
    uint8_t* stages = smem + a.o_stage;
    stages += (1024u - (smem_addr(stages) & 1023u)) & 1023u;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    volatile unsigned int* abort_flag = a.ctr + kAbortIdx;
    const int bs = FMT == MOE_MXFP4 ? 32 : 16;
    const int T = a.T, H = a.H, I = a.I, C = a.C;
    const int rho = (int)cluster_rank(), cid = (int)cluster_id_x(), ncl = (int)ncluster_x();
    const int IC = I / C, HC = H / C;
    const int nA = IC / a.RA, nB = HC / a.RB;               // stages per group
    const int nsegA = H / kSeg, nsegB = I / kSeg;
    const uint32_t SA = H / bs, SB = I / bs;                 // scale bytes of a gate/up row, a down row
    unsigned long long* trace = a.trace ? a.trace + (size_t)blockIdx.x * 32 : nullptr;
    if (trace && tid == 0) trace[0] = globaltimer();

    // ---- prologue 1 (may overlap the kernel before this one in the stream):
    // barriers, and the activations, which predate the router: per-token
    // power-of-two scale, f16 B fragments
    if (tid == 0) {
        for (int i = 0; i < a.nstage; i++) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kNC);
        }
        mbar_init(&hready[0], C);
        mbar_init(&hready[1], C);
        fence_mbar_init();
    }
    {
        unsigned* tok_amax = reinterpret_cast<unsigned*>(hsc);
        if (tid < T) tok_amax[tid] = 0u;
        __syncthreads();
        const int nvec = T * H / 8;
        for (int v = tid; v < nvec; v += blockDim.x) {
            const uint4 qv = __ldg(reinterpret_cast<const uint4*>(a.x) + v);
            const uint32_t u[4] = {qv.x, qv.y, qv.z, qv.w};
            float mx = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; i++)
                mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(u[i] << 16)), fabsf(__uint_as_float(u[i] & 0xFFFF0000u))));
            atomicMax(tok_amax + (v * 8) / H, __float_as_uint(mx));
        }
        __syncthreads();
        for (int v = tid; v < nvec; v += blockDim.x) {
            const int t = (v * 8) / H, h = v * 8 - t * H;
            const float sc = act_scale(__uint_as_float(tok_amax[t]));
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
    __syncthreads();
    // the cluster's barrier initialisations are visible before any peer arrives remotely
    cluster_sync_all();
    if (trace && tid == 0) trace[1] = globaltimer();

    // ---- the slot lookup's outputs (slot_of, tickets) are needed from here on
    pdl_wait();
    pdl_trigger();   // the next kernel may launch; it waits for this grid to finish
    if (trace && tid == 0) trace[2] = globaltimer();

    // ---- prologue 2: the groups (unique experts) of the call, in ticket order.
    // The stage ring is still unused, so its first bytes hold the per-(token, rank)
    // scratch.
    int* e_s = reinterpret_cast<int*>(stages);            // [n] expert or -1
    int* s_s = e_s + kMaxDecodePairs;                      // [n] slot
    unsigned* need_s = reinterpret_cast<unsigned*>(s_s + kMaxDecodePairs);
    int* lead_s = reinterpret_cast<int*>(need_s + kMaxDecodePairs);   // first entry of my expert
    int* mi_s = lead_s + kMaxDecodePairs;                  // my index inside the group
    int* grank_s = mi_s + kMaxDecodePairs;                 // group rank of a leader
    int* rdy_s = grank_s + kMaxDecodePairs;                // slot shows the needed ticket
    float* ts_s = reinterpret_cast<float*>(rdy_s + kMaxDecodePairs);   // [n][3] tensor scales
    const int n = T * a.k;
    if (tid < n) {
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
        int rank = 0, M = 0;
        for (int j = 0; j < n; j++) {
            const int ej = e_s[j];
            if (ej < 0) continue;
            if (ej == e) M++;
            if (lead_s[j] == j && (need_s[j] < kt || (need_s[j] == kt && ej < e))) rank++;
        }
        grank_s[tid] = rank;
        Group& G = groups[rank];
        G.expert = e;
        G.slot = s_s[tid];
        G.M = M;
        G.ready = rdy_s[tid];
        G.need = kt;
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
    const int ng = s_misc[0];
    if (trace && tid == 0) {
        trace[3] = globaltimer();
        trace[12] = (unsigned long long)((ng - cid + ncl - 1) / ncl);
        trace[13] = (unsigned long long)C;
        trace[14] = (unsigned long long)rho;
    }

    // Stage layouts.  A: gate codes [H/256 boxes][RA rows][128 B], then up codes the
    // same, then the RA scale rows of gate and of up; B: down codes [I/256 boxes]
    // [RB rows][128 B], then the RB scale rows.  Boxes are 1024-byte aligned.
    const int RA = a.RA, RB = a.RB;
    const uint32_t boxA = (uint32_t)RA * 128, boxB = (uint32_t)RB * 128;
    const int nboxA = H / 256, nboxB = I / 256;
    const uint32_t codesA = (uint32_t)nboxA * boxA;          // one tensor's codes in an A stage
    if (warp == kNC) {
        // ---------------------------------------------------------------- producer
        const uint32_t txA = 2u * RA * (uint32_t)(H / 2) + 2u * RA * SA;
        const uint32_t txB = (uint32_t)RB * (uint32_t)(I / 2) + (uint32_t)RB * SB;
        if (lane == 0) {
            prefetch_tmap(&a.map_a);
            prefetch_tmap(&a.map_b);
        }
        int st = 0;
        uint32_t round = 0;
        int issued = 0;
        for (int g = cid; g < ng; g += ncl) {
            const Group& G = groups[g];
            if (!G.ready) {
                bool ok = true;
                if (lane == 0) ok = wait_ready(a.ready + G.slot, G.need, a.ready_ns, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok && lane == 0) {
                    atomicOr(a.status, MOE_STATUS_READY_TIMEOUT);
                    *abort_flag = 1;
                }
            }
            // every lane acquires the ticket itself, then orders its TMA (async
            // proxy) reads of the slot after that acquire
            (void)ld_acquire_sys_u32(a.ready + G.slot);
            fence_proxy_async_global();
            const uint8_t* blk = a.slots + (unsigned long long)G.slot * a.block_bytes;
            const int ya = G.slot * a.rows_a, yb = G.slot * a.rows_b;
            for (int s = 0; s < nA + nB; s++) {
                bool ok = true;
                if (lane == 0) ok = mbar_wait_abort(&empty[st], (round & 1) ^ 1, a.pipe_ns, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok && lane == 0) {
                    atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
                    *abort_flag = 1;
                }
                uint8_t* dst = stages + (size_t)st * a.stage_bytes;
                if (lane == 0) mbar_arrive_expect_tx(&full[st], s < nA ? txA : txB);
                __syncwarp();
                if (s < nA) {
                    const int r0 = rho * IC + RA * s;
                    for (int bx = lane; bx < 2 * nboxA; bx += 32) {       // gate boxes, then up boxes
                        const int t = bx >= nboxA, b = bx - t * nboxA;
                        tma_load_2d(dst + t * codesA + b * boxA, &a.map_a, b * 128,
                                    ya + (t ? a.row_up : a.row_gate) + r0, &full[st]);
                    }
                    if (lane == 0) bulk_g2s(dst + 2 * codesA, blk + a.off[1] + (unsigned long long)r0 * SA, RA * SA, &full[st]);
                    if (lane == 1)
                        bulk_g2s(dst + 2 * codesA + RA * SA, blk + a.off[3] + (unsigned long long)r0 * SA, RA * SA, &full[st]);
                } else {
                    const int r0 = rho * HC + (s - nA) * RB;
                    for (int b = lane; b < nboxB; b += 32)
                        tma_load_2d(dst + b * boxB, &a.map_b, b * 128, yb + a.row_down + r0, &full[st]);
                    if (lane == 0)
                        bulk_g2s(dst + nboxB * boxB, blk + a.off[5] + (unsigned long long)r0 * SB, RB * SB, &full[st]);
                }
                if (trace && lane == 0 && issued < 8) trace[24 + issued] = globaltimer();
                issued++;
                if (++st == a.nstage) {
                    st = 0;
                    round++;
                }
            }
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
        const int g8 = lane >> 2, q = lane & 3;
        const int pr = tile_row(g8);                       // shared-memory row of MMA row g8 (g8 + 8: pr + 8)
        // A: tile pairs (gate tile, up tile) of the stage; warps per pair split K
        const int TA = RA / 16, WPA = kNC / TA, tpa = warp / WPA, kpa = warp % WPA;
        // B: RB/16 tiles; warps per tile split K
        const int TRB = RB / 16, wpt = kNC / TRB, tile = warp % TRB, kpart = warp / TRB;
        constexpr int kRedStage = kNC * 2 * NT * 32 * 4;   // floats of one red buffer
        const int bstride = 4 * T;                         // pieces between the words j of a segment
        int st = 0, rb = 0, it = 0;
        uint32_t round = 0;
        auto next_stage = [&]() {
            rb ^= 1;
            if (++st == a.nstage) {
                st = 0;
                round++;
            }
        };
        auto wait_full = [&]() {
            if (!mbar_wait_abort(&full[st], round & 1, a.pipe_ns, abort_flag)) {
                if (lane == 0) atomicOr(a.status, MOE_STATUS_PIPE_TIMEOUT);
                *abort_flag = 1;
            }
        };
        // (MMA row rr, member m) of tile slot t summed over the warps w0, w0 + dw, ...
        auto red_sum = [&](int t, int rr, int m, int w0, int dw, int nw) {
            int lx;
            const int e = frag_slot(rr, m, lx);
            const int nt = m >> 3;
            float s = 0.0f;
            for (int i = 0; i < nw; i++) {
                const int w = w0 + i * dw;
                s += red[(size_t)rb * kRedStage + ((((size_t)w * 2 + t) * NT + nt) * 32 + lx) * 4 + e];
            }
            return s;
        };
        for (int g = cid; g < ng; g += ncl, it++) {
            const Group& G = groups[g];
            const int M = G.M, hb = it & 1;
            float* hl = hloc + (size_t)hb * T * IC;                        // [M][IC] this CTA's slice of h
            unsigned* hmx = reinterpret_cast<unsigned*>(hloc + (size_t)2 * T * IC) + hb * T;   // [M] |h| max
            if (tid < T) hmx[tid] = 0u;
            // this lane's B columns: member m = g8 + 8 nt of the group (null past M)
            const uint4* xcol[NT];
            const uint4* hcol_hi[NT];
            const uint4* hcol_lo[NT];
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                const int m = g8 + 8 * nt;
                xcol[nt] = m < M ? xf + (size_t)G.tok[m] * 4 + q : nullptr;
                hcol_hi[nt] = m < M ? hf_hi + (size_t)m * 4 + q : nullptr;
                hcol_lo[nt] = m < M ? hf_lo + (size_t)m * 4 + q : nullptr;
            }

            // ---- A: RA rows of gate and the same RA rows of up per stage
            for (int s = 0; s < nA; s++) {
                wait_full();
                if (trace && tid == 0 && it == 0 && s == 0) trace[4] = globaltimer();
                if (trace && tid == 0 && it == 0 && s < 8) trace[16 + s] = globaltimer();
                const uint8_t* sb = stages + (size_t)st * a.stage_bytes;
                float acc[2][NT][4];
#pragma unroll
                for (int t = 0; t < 2; t++)
#pragma unroll
                    for (int nt = 0; nt < NT; nt++)
#pragma unroll
                        for (int e = 0; e < 4; e++) acc[t][nt][e] = 0.0f;
                const int row = tpa * 16 + pr;                   // shared-memory row of MMA row g8
                for (int seg = kpa; seg < nsegA; seg += WPA) {
                    const uint32_t so = FMT == MOE_NVFP4 ? seg * 8 + 2 * q : seg * 4;
                    const uint32_t co = (seg >> 1) * boxA + swz(row, ((seg & 1) << 2) | q);
                    const uint8_t* code[2] = {sb + co, sb + codesA + co};
                    const uint8_t* scl[2] = {sb + 2 * codesA + row * SA + so, sb + 2 * codesA + (RA + row) * SA + so};
                    const uint4* bp[1][NT];
#pragma unroll
                    for (int nt = 0; nt < NT; nt++)
                        bp[0][nt] = xcol[nt] ? xcol[nt] + (size_t)seg * 4 * bstride : nullptr;
                    seg_mma<FMT, 2, NT, 1>(code, 8 * 128, scl, 8 * SA, q, bp, bstride, acc);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                float4* rp = reinterpret_cast<float4*>(red + (size_t)rb * kRedStage);
#pragma unroll
                for (int t = 0; t < 2; t++)
#pragma unroll
                    for (int nt = 0; nt < NT; nt++)
                        rp[(((size_t)warp * 2 + t) * NT + nt) * 32 + lane] =
                            make_float4(acc[t][nt][0], acc[t][nt][1], acc[t][nt][2], acc[t][nt][3]);
                named_sync(1, kConsThreads);
                for (int o = tid; o < RA * M; o += kConsThreads) {
                    const int pair = o / (16 * M), rem = o - pair * 16 * M, rr = rem & 15, m = rem >> 4;
                    const int w0 = pair * WPA;
                    const float gs = red_sum(0, rr, m, w0, 1, WPA), us = red_sum(1, rr, m, w0, 1, WPA);
                    const float xs = xinv[G.tok[m]] * 16384.0f;     // undo x's scale and the decode's 2^-14
                    const float gv = gs * xs * G.ts[0], uv = us * xs * G.ts[1];
                    const float hv = gv / (1.0f + expf(-gv)) * uv;
                    hl[m * IC + s * RA + pair * 16 + tile_row(rr)] = hv;
                    atomicMax(hmx + m, __float_as_uint(fabsf(hv)));
                }
                next_stage();
            }
            named_sync(1, kConsThreads);     // every row of this CTA's slice of h is written
            if (trace && tid == 0 && it == 0) trace[5] = globaltimer();

            // ---- X: publish the slice to every CTA of the cluster (itself included),
            // wait until all have published, gather the whole h
            // lane p arrives on peer p's barrier (the release fences run side by side)
            if (tid < C) mbar_arrive_remote(map_peer(&hready[hb], (uint32_t)tid));
            if (!mbar_wait_abort(&hready[hb], (uint32_t)(it >> 1) & 1, a.dep_ns, abort_flag, true)) {
                if (lane == 0) atomicOr(a.status, MOE_STATUS_DEP_TIMEOUT);
                *abort_flag = 1;
            }
            if (trace && tid == 0 && it == 0) trace[6] = globaltimer();
            if (tid < M) {
                float mx = 0.0f;
                for (int p = 0; p < C; p++) mx = fmaxf(mx, ld_peer_f32(map_peer(hmx + tid, (uint32_t)p)));
                const float sc = act_scale(mx);
                hsc[tid] = sc;
                hinv[tid] = 1.0f / sc;
            }
            named_sync(1, kConsThreads);
            for (int v = tid; v < M * (I / 8); v += kConsThreads) {
                const int m = v / (I / 8), k0 = (v - m * (I / 8)) * 8;
                const int p = k0 / IC, il = k0 - p * IC;
                const uint32_t src = map_peer(hl + m * IC + il, (uint32_t)p);
                const uint4 u0 = ld_peer_v4(src), u1 = ld_peer_v4(src + 16);
                const float sc = hsc[m];
                const float hv[8] = {__uint_as_float(u0.x) * sc, __uint_as_float(u0.y) * sc,
                                     __uint_as_float(u0.z) * sc, __uint_as_float(u0.w) * sc,
                                     __uint_as_float(u1.x) * sc, __uint_as_float(u1.y) * sc,
                                     __uint_as_float(u1.z) * sc, __uint_as_float(u1.w) * sc};
                float hi[8], lo[8];
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    hi[i] = __half2float(__float2half_rn(hv[i]));
                    lo[i] = hv[i] - hi[i];                 // exact in fp32
                }
                const int pi = piece_index(k0, m, T);
                hf_hi[pi] = pack_piece(hi);
                hf_lo[pi] = pack_piece(lo);
            }
            named_sync(1, kConsThreads);
            if (trace && tid == 0 && it == 0) trace[7] = globaltimer();

            // ---- B: RB rows of down per stage; warps on tile (warp % TRB), K part warp / TRB
            for (int s = 0; s < nB; s++) {
                wait_full();
                if (trace && tid == 0 && it == 0 && nA + s < 8) trace[16 + nA + s] = globaltimer();
                const uint8_t* sb = stages + (size_t)st * a.stage_bytes;
                float acc[1][NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; nt++)
#pragma unroll
                    for (int e = 0; e < 4; e++) acc[0][nt][e] = 0.0f;
                const int row = tile * 16 + pr;
                for (int seg = kpart; seg < nsegB; seg += wpt) {
                    const uint32_t so = FMT == MOE_NVFP4 ? seg * 8 + 2 * q : seg * 4;
                    const uint8_t* code[1] = {sb + (seg >> 1) * boxB + swz(row, ((seg & 1) << 2) | q)};
                    const uint8_t* scl[1] = {sb + nboxB * boxB + row * SB + so};
                    const uint4* bp[2][NT];
#pragma unroll
                    for (int nt = 0; nt < NT; nt++) {
                        bp[0][nt] = hcol_hi[nt] ? hcol_hi[nt] + (size_t)seg * 4 * bstride : nullptr;
                        bp[1][nt] = hcol_lo[nt] ? hcol_lo[nt] + (size_t)seg * 4 * bstride : nullptr;
                    }
                    seg_mma<FMT, 1, NT, 2>(code, 8 * 128, scl, 8 * SB, q, bp, bstride, acc);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
                float4* rp = reinterpret_cast<float4*>(red + (size_t)rb * kRedStage);
#pragma unroll
                for (int nt = 0; nt < NT; nt++)
                    rp[(((size_t)warp * 2) * NT + nt) * 32 + lane] =
                        make_float4(acc[0][nt][0], acc[0][nt][1], acc[0][nt][2], acc[0][nt][3]);
                named_sync(1, kConsThreads);
                const int r0 = rho * HC + s * RB;
                for (int o = tid; o < TRB * 16 * M; o += kConsThreads) {
                    const int tl = o / (16 * M), rem = o - tl * 16 * M, rr = rem & 15, m = rem >> 4;
                    const float ys = red_sum(0, rr, m, tl, TRB, wpt);
                    const int yrow = r0 + tl * 16 + tile_row(rr);
                    a.y_part[((size_t)G.tok[m] * a.k + G.rank[m]) * H + yrow] =
                        G.wt[m] * (ys * (hinv[m] * 16384.0f) * G.ts[2]);
                }
                next_stage();
            }

            // ---- this group's rows of block rho are in y_part: count it; the last
            // group to finish the block sums it over the ranks (K5)
            named_sync(1, kConsThreads);
            if (trace && tid == 0 && it == 0) trace[8] = globaltimer();
            if (tid == 0) {
                __threadfence();
                const unsigned prev = atomicAdd(a.ctr + rho, 1u);
                s_misc[1] = (prev == (unsigned)ng - 1u);
                if (s_misc[1]) __threadfence();
            }
            named_sync(1, kConsThreads);
            if (s_misc[1]) {
                if (a.y) {
                    const int q4 = HC / 4;
                    for (int v = tid; v < T * q4; v += kConsThreads) {
                        const int t = v / q4, r = rho * HC + (v - t * q4) * 4;
                        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int j = 0; j < a.k; j++) {
                            const float4 pv = __ldcg(reinterpret_cast<const float4*>(a.y_part + ((size_t)t * a.k + j) * H + r));
                            sum.x += pv.x;
                            sum.y += pv.y;
                            sum.z += pv.z;
                            sum.w += pv.w;
                        }
                        const uint32_t b0 = __bfloat16_as_ushort(__float2bfloat16_rn(sum.x));
                        const uint32_t b1 = __bfloat16_as_ushort(__float2bfloat16_rn(sum.y));
                        const uint32_t b2 = __bfloat16_as_ushort(__float2bfloat16_rn(sum.z));
                        const uint32_t b3 = __bfloat16_as_ushort(__float2bfloat16_rn(sum.w));
                        *reinterpret_cast<uint2*>(a.y + (size_t)t * H + r) = make_uint2(b0 | (b1 << 16), b2 | (b3 << 16));
                    }
                }
                if (tid == 0) a.ctr[rho] = 0u;
            }
            if (trace && tid == 0) trace[9] = globaltimer();
        }
    }

    // ---- epilogue: no CTA leaves while a peer may still read its shared memory;
    // the last CTA clears the abort flag for the next launch
    __syncthreads();
    cluster_sync_all();
    if (trace && tid == 0) trace[10] = globaltimer();
    if (tid == 0) {
        __threadfence();
        const unsigned int prev = atomicAdd(a.ctr + kDoneIdx, 1u);
        if (prev == gridDim.x - 1) {
            __threadfence();
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

static size_t up(size_t n, size_t a) { return (n + a - 1) / a * a; }

int make_tmap_2d(CUtensorMap* map, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t pitch,
                 uint32_t box_bytes, uint32_t box_rows, bool swizzle128);

// Shared-memory layout and stage sizes of one launch: RA = 32 gate rows per A
// stage when two such stages fit, else 16; RB = the most down rows (128, 64, 32
// or 16, dividing H/C) whose stage is no larger than an A stage.  MOE_EINVAL if
// not even two stages fit.
static int plan_ffn(const moe_pool* p, int T, int C, int NT, FfnArgs& a, size_t& smem) {
    const moe_config& c = p->cfg;
    const int bs = p->bs;
    const int IC = c.I / C, HC = c.H / C;
    const size_t SA = c.H / bs, SB = c.I / bs;
    const size_t budget = (size_t)p->ffn_smem;
    for (int RA = 32; RA >= 16; RA >>= 1) {
        if (IC % RA) continue;
        const size_t stA = 2 * (size_t)RA * (c.H / 2) + 2 * (size_t)RA * SA;
        int RB = 16;
        for (int rb = 128; rb >= 16; rb >>= 1)
            if (HC % rb == 0 && (size_t)rb * (c.I / 2 + SB) <= std::max<size_t>(stA, (size_t)16 * (c.I / 2 + SB))) {
                RB = rb;
                break;
            }
        a.RA = RA;
        a.RB = RB;
        const size_t stB = (size_t)RB * (c.I / 2 + SB);
        a.stage_bytes = (int)up(std::max(stA, stB), 1024);
        size_t o = up((2 * 16 + 2) * sizeof(uint64_t), 128);
        a.o_groups = (int)o;
        o += sizeof(Group) * kMaxDecodePairs;
        a.o_misc = (int)up(o, 16);
        o = a.o_misc + 3 * kMaxDecodeT * sizeof(float) + 8 * sizeof(int);
        a.o_red = (int)up(o, 16);
        o = a.o_red + (size_t)2 * kNC * 2 * NT * 32 * 4 * sizeof(float);
        a.o_hloc = (int)up(o, 16);
        o = a.o_hloc + ((size_t)2 * T * IC + 2 * T) * sizeof(float);
        a.o_x = (int)up(o, 16);
        o = a.o_x + (size_t)T * c.H * 2;
        a.o_h = (int)up(o, 16);
        o = a.o_h + (size_t)2 * T * c.I * 2;
        a.o_stage = (int)up(o, 1024);
        // the prologue keeps its per-(token, rank) table (7 ints + 3 floats each) in the ring
        const size_t need_ring = std::max((size_t)2 * a.stage_bytes, (size_t)10 * 4 * kMaxDecodePairs);
        if (a.o_stage + need_ring + 1024 > budget) continue;
        a.nstage = (int)std::min<size_t>(8, (budget - a.o_stage - 1024) / a.stage_bytes);
        smem = a.o_stage + (size_t)a.nstage * a.stage_bytes + 1024;
        return MOE_OK;
    }
    return fail(MOE_EINVAL, "decode FFN: T * (H + 2 I) too large for shared memory (lower max_tokens)");
}

// The 2-D views of the pool's code rows (boxes 128 bytes x `rows`), built once
// per pool and box height.  The FP4 code rows of every slot must sit at whole
// rows of the view: block bytes and tensor offsets multiples of the row bytes.
static int ffn_maps(moe_pool* p, FfnArgs& a) {
    const moe_config& c = p->cfg;
    const uint64_t rwa = c.H / 2, rwb = c.I / 2, blk = p->lay.bytes;
    if (blk % rwa || p->lay.off[0] % rwa || p->lay.off[2] % rwa || blk % rwb || p->lay.off[4] % rwb)
        return fail(MOE_EINVAL, "decode FFN: the expert block does not divide into rows of H/2 and I/2 bytes");
    const uint64_t pool_bytes = (uint64_t)c.n_slots * blk;
    if (pool_bytes / rwa > 0x7fffffffull) return fail(MOE_EINVAL, "decode FFN: slot pool too large for a 2-D view");
    const int ia = a.RA == 32 ? 1 : 0;
    int ib = 0;
    while ((16 << ib) < a.RB) ib++;
    int rc;
    if (!p->ffn_map_a_ok[ia]) {
        if ((rc = make_tmap_2d(&p->ffn_map_a[ia], p->slots, rwa, pool_bytes / rwa, rwa, 128, a.RA, true))) return rc;
        p->ffn_map_a_ok[ia] = 1;
    }
    if (!p->ffn_map_b_ok[ib]) {
        if ((rc = make_tmap_2d(&p->ffn_map_b[ib], p->slots, rwb, pool_bytes / rwb, rwb, 128, a.RB, true))) return rc;
        p->ffn_map_b_ok[ib] = 1;
    }
    a.map_a = p->ffn_map_a[ia];
    a.map_b = p->ffn_map_b[ib];
    a.rows_a = (int)(blk / rwa);
    a.rows_b = (int)(blk / rwb);
    a.row_gate = (int)(p->lay.off[0] / rwa);
    a.row_up = (int)(p->lay.off[2] / rwa);
    a.row_down = (int)(p->lay.off[4] / rwb);
    return MOE_OK;
}

// For every cluster size C in {16, 8, 4, 2, 1} that splits I and H into 16-row
// tiles: how many clusters of C CTAs (with this kernel's shared memory) the GPU
// can hold at once (0 when C does not split the shapes or no cluster fits).
template <int FMT, int NT>
static int query_clusters(moe_pool* p, int (&ncl)[5]) {
    auto kern = ffn_decode_kernel<FMT, NT>;
    const moe_config& c = p->cfg;
    MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p->ffn_smem));
    MOE_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1));
    int any = 0;
    cudaError_t last = cudaSuccess;
    for (int ci = 0, C = kMaxCluster; ci < 5; ci++, C >>= 1) {
        ncl[ci] = 0;
        if (c.I % (16 * C) || c.H % (16 * C)) continue;
        int n = 0;
        if (C == 1) {
            // a "cluster" of one CTA: plain occupancy
            int per_sm = 0;
            last = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFfnThreads, p->ffn_smem);
            if (last == cudaSuccess) n = per_sm * p->num_sms;
        } else {
            cudaLaunchConfig_t lc = {};
            lc.gridDim = dim3(C);
            lc.blockDim = dim3(kFfnThreads);
            lc.dynamicSmemBytes = p->ffn_smem;
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = C;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            lc.attrs = at;
            lc.numAttrs = 1;
            last = cudaOccupancyMaxActiveClusters(&n, kern, &lc);
        }
        if (last != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;
        }
        ncl[ci] = n;
        any |= n > 0;
    }
    if (!any)
        return fail(MOE_EINVAL, std::string("decode FFN: no cluster size fits on this GPU (last query: ") +
                                    cudaGetErrorString(last) + ")");
    return MOE_OK;
}

// The cluster size of a launch with at most `groups` unique experts.  A CTA's
// share of a group is 1/C of it, and the clusters that fit at once take the
// groups in ceil(groups / clusters) rounds, so the time goes as rounds / C: pick
// the smallest, then the fewest rounds, then the larger C.
static int g_force_cluster = 0;   // moe_set_ffn_cluster: 0 = automatic

static void choose_cluster(const int (&ncl)[5], int groups, int& C, int& nclusters) {
    if (g_force_cluster > 0)
        for (int ci = 0, c = kMaxCluster; ci < 5; ci++, c >>= 1)
            if (c == g_force_cluster && ncl[ci] > 0) {
                C = c;
                nclusters = std::min(ncl[ci], groups);
                return;
            }
    double best = 1e30;
    int best_rounds = 1 << 30;
    C = 1;
    nclusters = 1;
    for (int ci = 0, c = kMaxCluster; ci < 5; ci++, c >>= 1) {
        if (ncl[ci] <= 0) continue;
        const int n = std::min(ncl[ci], groups);
        const int rounds = (groups + n - 1) / n;
        const double cost = (double)rounds / c;
        if (cost < best - 1e-12 || (cost < best + 1e-12 && rounds < best_rounds)) {
            best = cost;
            best_rounds = rounds;
            C = c;
            nclusters = n;
        }
    }
}

template <int FMT, int NT>
static int ffn_shape(moe_pool* p, FfnArgs& a, size_t& smem, int& nclusters) {
    const int fi = FMT == MOE_NVFP4 ? 1 : 0, ni = NT - 1;
    if (!p->ffn_attr_set[fi][ni]) {
        int rc = query_clusters<FMT, NT>(p, p->ffn_ncl[fi][ni]);
        if (rc) return rc;
        p->ffn_attr_set[fi][ni] = 1;
    }
    // a call has at most T * k unique experts, one cluster each
    choose_cluster(p->ffn_ncl[fi][ni], a.T * a.k, a.C, nclusters);
    int rc = plan_ffn(p, a.T, a.C, NT, a, smem);
    if (rc) return rc;
    return ffn_maps(p, a);
}

template <int FMT, int NT>
static int launch_ffn(moe_pool* p, FfnArgs& a, cudaStream_t s) {
    size_t smem = 0;
    int ncl = 0;
    int rc = ffn_shape<FMT, NT>(p, a, smem, ncl);
    if (rc) return rc;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(ncl * a.C);
    lc.blockDim = dim3(kFfnThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = a.C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    // programmatic serialisation: the activations are staged while the slot
    // lookup before this kernel finishes (the kernel waits for it before reading
    // slot_of, the tickets and the tensor scales)
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 2;
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

extern "C" int moe_set_ffn_cluster(int cluster) {
    if (cluster != 0 && cluster != 1 && cluster != 2 && cluster != 4 && cluster != 8 && cluster != 16)
        return fail(MOE_EINVAL, "cluster size must be 0 (automatic), 1, 2, 4, 8 or 16");
    g_force_cluster = cluster;
    return MOE_OK;
}

extern "C" int moe_ffn_launch_info(moe_pool* p, int T, int* cluster, int* clusters, int* nstage,
                                   int* smem_bytes) {
    if (!p || !cluster || !clusters || !nstage || !smem_bytes) return fail(MOE_EINVAL, "null argument");
    if (T <= 0 || T > p->cfg.max_tokens) return fail(MOE_EINVAL, "T must be in [1, max_tokens]");
    FfnArgs a{};
    a.T = T;
    a.k = p->cfg.k;
    size_t smem = 0;
    int ncl = 0, rc;
    if (p->cfg.fmt == MOE_NVFP4)
        rc = T <= 8 ? ffn_shape<MOE_NVFP4, 1>(p, a, smem, ncl) : ffn_shape<MOE_NVFP4, 2>(p, a, smem, ncl);
    else
        rc = T <= 8 ? ffn_shape<MOE_MXFP4, 1>(p, a, smem, ncl) : ffn_shape<MOE_MXFP4, 2>(p, a, smem, ncl);
    if (rc) return rc;
    *cluster = a.C;
    *clusters = ncl;
    *nstage = a.nstage;
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

extern "C" int moe_expert_ffn(moe_pool* p, int layer, const void* x_bf16, int T, const int32_t* idx,
                              const float* w, const int32_t* slot_of, float* y_part, void* y_bf16, int* status,
                              void* stream) {
    static_assert(offsetof(FfnArgs, map_a) % 64 == 0 && offsetof(FfnArgs, map_b) % 64 == 0,
                  "tensor maps must be 64-byte aligned in the kernel parameters");
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
    a.slot_of = slot_of;
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
