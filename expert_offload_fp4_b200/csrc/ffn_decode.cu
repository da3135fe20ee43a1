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
// block scales of each work stage with 1-D bulk copies (a whole tile of rows is
// one contiguous range of the slot) into a ring of shared-memory stages
// (mbarrier full/empty pairs); for a missed expert it first waits (bounded) for
// the slot's ready ticket written by the copy stream.
// Warps 0..7 (consumers) run the dot products on the tensor cores with
// mma.sync m16n8k16, f16 inputs and fp32 accumulation:
//  - weights: E2M1 code pairs converted to f16 pairs (cvt.rn.f16x2.e2m1x2),
//    multiplied (exactly) by their block scale in f16: the E4M3 scale itself
//    (NVFP4), or 2^(e - E) with E the largest E8M0 exponent of the row's
//    128-element segment (MXFP4; 2^(E-127) is applied to the segment's fp32 sum);
//  - activations: x of each token times a power of two (bf16 is exact in f16
//    that way); h of each (token, expert) times a power of two and split into
//    an f16 high part and an f16 remainder, so down h is carried to ~22 bits;
//  - products are exact, sums fp32; every output row is one warp's chain of
//    MMAs over the whole K, in a fixed order, so results are reproducible.
#include <math.h>

#include "common.cuh"

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
    int stage_bytes, nstage;
    int ks;                    // A: K split of a unit (1, 2, 4): 2 ks warps per unit
    int nAU;                   // A: units at work (divides nstage)
    int nBU;                   // B: warp groups at work (divides nstage)
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
    uint64_t* hready = empty + a.nstage;                               // [2]
    Group* groups = reinterpret_cast<Group*>(smem + a.o_groups);
    float* xinv = reinterpret_cast<float*>(smem + a.o_misc);           // [16] per token
    float* hinv = xinv + kMaxDecodeT;                                  // [16] per member
    float* hsc = hinv + kMaxDecodeT;                                   // [16] per member
    int* s_misc = reinterpret_cast<int*>(hsc + kMaxDecodeT);           // [8]
    float* pairbuf = reinterpret_cast<float*>(smem + a.o_red);         // [unit][2][2 (gate, up)][ks][16][T]
    float* hloc = reinterpret_cast<float*>(smem + a.o_hloc);           // [2][T][I/C], then [2][T] maxima
    uint4* xf = reinterpret_cast<uint4*>(smem + a.o_x);                // x fragments, N = T
    uint4* hf_hi = reinterpret_cast<uint4*>(smem + a.o_h);             // h fragments, N = T
    uint4* hf_lo = hf_hi + (size_t)a.T * a.I / 8;
    uint8_t* stages = smem + a.o_stage;

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

    // Stage layouts (row-major, as in the slot): A = RA code rows of gate, RA of up,
    // then their RA scale rows each; B = RB code rows of down, then their scale rows.
    const int RA = a.RA, RB = a.RB;
    const uint32_t CA = (uint32_t)RA * (H / 2);               // one tensor's code bytes in an A stage
    const uint32_t CB = (uint32_t)RB * (I / 2);
    if (warp == kNC) {
        // ---------------------------------------------------------------- producer
        const uint32_t txA = 2u * CA + 2u * RA * SA;
        const uint32_t txB = CB + (uint32_t)RB * SB;
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
            // every lane acquires the ticket itself, then orders its bulk (async
            // proxy) reads of the slot after that acquire
            (void)ld_acquire_sys_u32(a.ready + G.slot);
            fence_proxy_async_global();
            const uint8_t* blk = a.slots + (unsigned long long)G.slot * a.block_bytes;
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
                    const unsigned long long r0 = (unsigned long long)(rho * IC + RA * s);
                    if (lane == 0) bulk_g2s(dst, blk + a.off[0] + r0 * (H / 2), CA, &full[st]);
                    if (lane == 1) bulk_g2s(dst + CA, blk + a.off[2] + r0 * (H / 2), CA, &full[st]);
                    if (lane == 2) bulk_g2s(dst + 2 * CA, blk + a.off[1] + r0 * SA, RA * SA, &full[st]);
                    if (lane == 3) bulk_g2s(dst + 2 * CA + RA * SA, blk + a.off[3] + r0 * SA, RA * SA, &full[st]);
                } else {
                    const unsigned long long r0 = (unsigned long long)(rho * HC + (s - nA) * RB);
                    if (lane == 0) bulk_g2s(dst, blk + a.off[4] + r0 * (I / 2), CB, &full[st]);
                    if (lane == 1) bulk_g2s(dst + CB, blk + a.off[5] + r0 * SB, RB * SB, &full[st]);
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
        // A stage = 16 rows of gate and the same 16 rows of up.  Unit u = warp /
        // (2 ks) takes A stages u, u + nAU, ...: its even warps the gate tile, its
        // odd ones the up tile, each over 1/ks of K (part kp = (warp % 2ks) / 2);
        // the unit then sums the parts in order and forms h.
        // B stage = RB rows of down, TRB = RB / 16 tiles: warp group warp / TRB takes
        // B stages group, group + nBU, ..., one tile over the whole K per warp.
        // nAU and nBU divide the ring size, so within a phase every slot is filled
        // and emptied for one unit (or group) only, in order: a wait never meets a
        // slot whose earlier fill is still pending (whose phase parity would
        // alias).  Consumer barriers separate the phases.
        const int g8 = lane >> 2, q = lane & 3;
        const int ks = a.ks, uw = 2 * ks, unit = warp / uw, widx = warp - unit * uw;
        const int role = widx & 1, kp = widx >> 1, segsA = nsegA / ks;
        const int TRB = RB / 16, grp = warp / TRB, tile = warp % TRB;
        const int nAU = a.nAU, nBU = a.nBU;
        const uint32_t qs = FMT == MOE_NVFP4 ? 2 * q : 0;   // the thread's scale bytes in a row's segment
        const int bstride = 4 * T;                         // pieces between the words j of a segment
        int gi = 0, it = 0, pst = 0;                       // global stage index, group count, pair stages
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
        for (int g = cid; g < ng; g += ncl, it++) {
            const Group& G = groups[g];
            const int M = G.M, hb = it & 1;
            float* hl = hloc + (size_t)hb * T * IC;                        // [M][IC] this CTA's slice of h
            unsigned* hmx = reinterpret_cast<unsigned*>(hloc + (size_t)2 * T * IC) + hb * T;   // [M] |h| max
            if (tid < T) hmx[tid] = 0u;
            named_sync(1, kConsThreads);     // hmx is zero before any pair adds to it
            // this lane's B columns: member m = g8 + 8 nt of the group (null past M)
            const uint4* xb[1][NT];            // x of the member's token
            const uint4* hb2[2][NT];           // h of the member: high parts, remainders
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                const int m = g8 + 8 * nt;
                xb[0][nt] = m < M ? xf + (size_t)G.tok[m] * 4 + q : nullptr;
                hb2[0][nt] = m < M ? hf_hi + (size_t)m * 4 + q : nullptr;
                hb2[1][nt] = m < M ? hf_lo + (size_t)m * 4 + q : nullptr;
            }

            // ---- A: stage s = gate rows [rho*IC + 16 s, +16) and the same rows of up
            for (int s = 0; s < nA; s++) {
                const int k = gi + s;
                if (unit >= nAU || s % nAU != unit) continue;
                slot_wait(k);
                if (trace && tid == 0 && it == 0 && s == 0) trace[4] = globaltimer();
                if (trace && lane == 0 && widx == 0 && it == 0 && s < 8) trace[16 + s] = globaltimer();
                const uint8_t* sb = stages + (size_t)(k % a.nstage) * a.stage_bytes;
                const uint8_t* tb = sb + role * CA;                       // gate or up codes
                const uint8_t* tsc = sb + 2 * CA + role * RA * SA;        // their scale rows
                float part[NT][4];
                tile_mma<FMT, NT, 1>(tb + g8 * (H / 2) + 16 * q, 8 * (H / 2), tsc + g8 * SA + qs, 8 * SA, q,
                                     kp * segsA, segsA, xb, bstride, part);
                slot_release(k, uw);
                // the unit's parts: [parity][role][kp][16][T]
                float* ub = pairbuf + (size_t)unit * 2 * 2 * ks * 16 * T + (size_t)(pst & 1) * 2 * ks * 16 * T;
                float* pb = ub + (size_t)(role * ks + kp) * 16 * T;
#pragma unroll
                for (int nt = 0; nt < NT; nt++)
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int rr = g8 + (e >> 1) * 8, m = 8 * nt + 2 * q + (e & 1);
                        if (m < M) pb[rr * T + m] = part[nt][e];
                    }
                named_sync(2 + unit, 32 * uw);
                for (int o = widx * 32 + lane; o < 16 * M; o += 32 * uw) {
                    const int rr = o & 15, m = o >> 4;
                    float gs = ub[rr * T + m], us = ub[(size_t)ks * 16 * T + rr * T + m];
                    for (int p = 1; p < ks; p++) {
                        gs += ub[(size_t)p * 16 * T + rr * T + m];
                        us += ub[(size_t)(ks + p) * 16 * T + rr * T + m];
                    }
                    const float xs = xinv[G.tok[m]];                   // undo x's scale
                    const float gv = gs * xs * G.ts[0], uv = us * xs * G.ts[1];
                    const float hv = gv / (1.0f + expf(-gv)) * uv;
                    hl[m * IC + s * 16 + rr] = hv;
                    atomicMax(hmx + m, __float_as_uint(fabsf(hv)));
                }
                pst++;
            }
            gi += nA;
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

            // ---- B: stage b = down rows [rho*HC + RB b, +RB); warp `tile` of group b % ngrp
            for (int b = 0; b < nB; b++) {
                const int k = gi + b;
                if (b % nBU != grp) continue;
                slot_wait(k);
                if (trace && lane == 0 && tile == 0 && it == 0 && nA + b < 8) trace[16 + nA + b] = globaltimer();
                const uint8_t* sb = stages + (size_t)(k % a.nstage) * a.stage_bytes;
                const int row = tile * 16 + g8;
                float acc[NT][4];
                tile_mma<FMT, NT, 2>(sb + row * (I / 2) + 16 * q, 8 * (I / 2), sb + CB + row * SB + qs, 8 * SB, q,
                                     0, nsegB, hb2, bstride, acc);
                slot_release(k, TRB);
                const int r0 = rho * HC + b * RB + tile * 16;
#pragma unroll
                for (int nt = 0; nt < NT; nt++)
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int rr = g8 + (e >> 1) * 8, m = 8 * nt + 2 * q + (e & 1);
                        if (m < M)
                            a.y_part[((size_t)G.tok[m] * a.k + G.rank[m]) * H + r0 + rr] =
                                G.wt[m] * (acc[nt][e] * hinv[m] * G.ts[2]);
                    }
            }
            gi += nB;

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
                // y = the rank-ordered sum of y_part, rounded to bf16
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
                    if (a.y) {
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

// Shared-memory layout and stage sizes of one launch.  A CTA streams at HBM rate
// only with several stages in flight, so stages are small: RA = 16 gate (and up)
// rows per A stage (one 16-row tile of each); RB = the most down rows
// (128, 64, 32 or 16, dividing H/C) whose stage is no larger than an A stage.
// MOE_EINVAL if not even two stages fit.
static int plan_ffn(const moe_pool* p, int T, int C, int NT, FfnArgs& a, size_t& smem) {
    const moe_config& c = p->cfg;
    const int bs = p->bs;
    const int IC = c.I / C, HC = c.H / C;
    const size_t SA = c.H / bs, SB = c.I / bs;
    const size_t budget = (size_t)p->ffn_smem;
    {
        const int RA = 16;
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
        a.stage_bytes = (int)up(std::max(stA, stB), 128);
        size_t o = up((2 * 16 + 2) * sizeof(uint64_t), 128);
        a.o_groups = (int)o;
        o += sizeof(Group) * kMaxDecodePairs;
        a.o_misc = (int)up(o, 16);
        o = a.o_misc + 3 * kMaxDecodeT * sizeof(float) + 8 * sizeof(int);
        a.o_red = (int)up(o, 16);
        o = a.o_red + (size_t)(kNC / 2) * 2 * 2 * 16 * T * sizeof(float);   // units * ks <= 4
        a.o_hloc = (int)up(o, 16);
        o = a.o_hloc + ((size_t)2 * T * IC + 2 * T) * sizeof(float);
        a.o_x = (int)up(o, 16);
        o = a.o_x + (size_t)T * c.H * 2;
        a.o_h = (int)up(o, 16);
        o = a.o_h + (size_t)2 * T * c.I * 2;
        a.o_stage = (int)up(o, 128);
        // the prologue keeps its per-(token, rank) table (7 ints + 3 floats each) in the ring
        const size_t need_ring = std::max((size_t)2 * a.stage_bytes, (size_t)10 * 4 * kMaxDecodePairs);
        if (a.o_stage + need_ring > budget)
            return fail(MOE_EINVAL, "decode FFN: T * (H + 2 I) too large for shared memory (lower max_tokens)");
        a.nstage = (int)std::min<size_t>(8, (budget - a.o_stage) / a.stage_bytes);
        if (a.nstage >= kNC / 2) a.nstage = a.nstage / (kNC / 2) * (kNC / 2);
        smem = a.o_stage + (size_t)a.nstage * a.stage_bytes;
        // A: units of 2 ks warps, as many as divide the ring; the K split with the
        // fewest rounds (one round = one stage's full-K dot products / ks) wins,
        // a little weight against more warps meeting at every stage
        const int nA = IC / RA, nsegA = c.H / 128;
        double best = 1e30;
        for (int ks = 1; ks <= kNC / 2; ks *= 2) {
            if (nsegA % ks) continue;
            int u = std::min(kNC / (2 * ks), a.nstage);
            while (a.nstage % u) u--;
            const double cost = (double)((nA + u - 1) / u) / ks + 0.05 * ks;
            if (cost < best) {
                best = cost;
                a.ks = ks;
                a.nAU = u;
            }
        }
        // B: groups of RB / 16 warps, as many as divide the ring
        a.nBU = 1;
        for (int d = kNC / (a.RB / 16); d >= 1; d--)
            if (a.nstage % d == 0) {
                a.nBU = d;
                break;
            }
        return MOE_OK;
    }
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

// Cluster size C of a launch: the work of one expert is split over C CTAs, and
// the clusters that fit at once take the G unique experts in ceil(G / clusters)
// rounds, so the time goes as rounds * (1 / C + the fixed cost of a group, about
// 4 % of an expert on one CTA).  G is the expected number of unique experts,
// E (1 - (1 - k/E)^T) (at most T * k).
static void choose_cluster(const moe_pool* p, const int (&ncl)[5], int T, int& C, int& nclusters) {
    const moe_config& c = p->cfg;
    const double Gd = c.E * (1.0 - std::pow(1.0 - (double)c.k / c.E, (double)T));
    const int G = std::max(1, std::min(T * c.k, (int)(Gd + 0.5)));
    double best = 1e30;
    C = 1;
    nclusters = 1;
    for (int ci = 0, cc = kMaxCluster; ci < 5; ci++, cc >>= 1) {
        if (ncl[ci] <= 0) continue;
        if (g_force_cluster && cc != g_force_cluster) continue;
        const int n = std::min(ncl[ci], G);
        const int rounds = (G + n - 1) / n;
        const double cost = rounds * (1.0 / cc + 0.04);
        if (cost < best - 1e-12) {
            best = cost;
            C = cc;
            nclusters = std::min(ncl[ci], T * c.k);
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
    choose_cluster(p, p->ffn_ncl[fi][ni], a.T, a.C, nclusters);
    return plan_ffn(p, a.T, a.C, NT, a, smem);
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
