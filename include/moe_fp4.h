/*
 * moe_fp4.h -- C ABI of the B200 (sm_100a) hot path of one FreeToken-style MoE
 * layer with FP4 experts offloaded to pinned host memory.
 *
 * The layer, per decode step: route each token to k of E experts; look the
 * chosen experts up in an LRU pool of expert slots held in HBM; stream the
 * missed experts from pinned host memory into their slots on the copy engine
 * while the hits are already being computed; run the SwiGLU expert FFN on the
 * FP4 weights; merge the expert outputs by routing weight.  The q* bandwidth
 * split is a host function whose result is reported (every expert runs on the
 * GPU here).
 *
 * Conventions
 *  - Every call returns an int status (MOE_OK = 0 or an MOE_E* code); on error
 *    moe_last_error() returns a message for the calling thread.
 *  - Pointers are device pointers unless their name ends in _h (host memory).
 *    Device buffers and streams are owned by the caller; the pool (slot storage
 *    in HBM, pinned host expert store, slot metadata, scratch) is owned by the
 *    library and only created / destroyed through moe_pool_create/destroy.
 *  - A stream is a cudaStream_t passed as void* (NULL = the legacy stream).
 *  - Calls are asynchronous on their stream, except moe_slot_lookup, which
 *    waits (bounded) for the lookup kernel because the host must drive the copy
 *    engine with the miss list, and the pool create/load/state/stats calls.
 *  - Tensor layouts (row-major, "canonical"): bf16 activations x [T, H];
 *    router weight W_r [E, H] bf16; FP4 codes [rows, K/2] bytes with element c
 *    of a row in byte c/2, the lower element index in the low nibble; block
 *    scales [rows, K/bs] bytes, bs = 32 (MXFP4, E8M0) or 16 (NVFP4, E4M3).
 *    gate and up are [I, H] (K = H), down is [H, I] (K = I).
 */
#ifndef MOE_FP4_H
#define MOE_FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
    MOE_OK = 0,
    MOE_EINVAL = 1,   /* bad argument or shape outside the supported range */
    MOE_ENOMEM = 2,   /* device or pinned host allocation failed */
    MOE_ECUDA = 3,    /* a CUDA runtime call failed */
    MOE_ETIMEOUT = 4, /* a bounded wait (host or device) gave up */
    MOE_EBOUNDS = 5,  /* an index (layer, expert, slot) outside the pool */
    MOE_ESTATE = 6    /* call out of order (e.g. expert not loaded) */
};

/* FP4 expert formats named by the pages (post.smzdm.com/p/a825qpgl, section 一:
 * MXFP4 expert weights; an NVFP4 build of the 35B-A3B model).  Bit layouts from
 * the OCP MX v1.0 spec (E2M1 codes, E8M0 scale per 32) and NVIDIA's NVFP4
 * description (E2M1 codes, E4M3 scale per 16, FP32 tensor scale). */
enum { MOE_MXFP4 = 0, MOE_NVFP4 = 1 };

/* How moe_stream_misses moves a missed expert's block host -> slot. */
enum {
    MOE_COPY_SM = 0,   /* a kernel on the copy stream reads the mapped host block over
                          PCIe with 16-byte loads from every SM */
    MOE_COPY_DMA = 1   /* one cudaMemcpyAsync per miss on the copy engine (default) */
};

/* Bits of the device status word written by moe_expert_ffn. */
enum {
    MOE_STATUS_READY_TIMEOUT = 1,  /* a missed expert's ready flag never arrived */
    MOE_STATUS_DEP_TIMEOUT = 2,    /* waited too long for an expert's h (other CTAs) */
    MOE_STATUS_BAD_SLOT = 4,       /* slot index outside the pool */
    MOE_STATUS_BAD_EXPERT = 8,     /* expert index outside [0, E) */
    MOE_STATUS_PIPE_TIMEOUT = 16,  /* a shared-memory pipeline wait gave up */
    MOE_STATUS_NOT_RESIDENT = 32   /* moe_decode_resident: an expert was not resident */
};

typedef struct {
    int H;            /* hidden size, multiple of 256 */
    int I;            /* expert intermediate size, multiple of 256 */
    int E;            /* experts per layer, <= 1024 */
    int k;            /* experts chosen per token, <= 32 */
    int L;            /* MoE layers sharing the slot pool */
    int fmt;          /* MOE_MXFP4 or MOE_NVFP4 */
    int n_slots;      /* expert slots in HBM, >= the unique experts of one call */
    int max_tokens;   /* largest T of a decode call (moe_expert_ffn), <= 16 */
    int host_layers;  /* distinct host copies of the layers: layer l is stored at
                         l % host_layers (0 means L); lets a large model's host
                         store be folded when pinned RAM is short */
    int reserved[3];
} moe_config;

typedef struct moe_pool moe_pool;

/* One expert in the canonical layout (host memory).  tensor_scale[i] is the
 * NVFP4 FP32 tensor scale of gate/up/down (ignored for MXFP4). */
typedef struct {
    const uint8_t* codes_h[3];   /* gate [I, H/2], up [I, H/2], down [H, I/2] */
    const uint8_t* scales_h[3];  /* gate [I, H/bs], up [I, H/bs], down [H, I/bs] */
    float tensor_scale[3];
} moe_expert_src;

/* One missed expert of a lookup: copy the host block of (layer, expert) into
 * `slot`, then publish `ticket` in the slot's ready flag. */
typedef struct {
    int32_t expert;
    int32_t slot;
    uint32_t ticket;
    int32_t evicted_key;         /* layer*E + expert evicted from the slot, -1 if free */
} moe_miss;

typedef struct {
    int n_uniq;                  /* unique experts of the call, ascending id */
    int n_miss;
    int32_t* uniq_h;             /* caller array, capacity >= min(T*k, E) */
    int32_t* is_hit_h;           /* caller array, same capacity */
    moe_miss* miss_h;            /* caller array, same capacity */
} moe_lookup_result;

typedef struct {
    long long lookups, unique, hits, misses, evictions;
    long long h2d_bytes, h2d_copies;
} moe_stats;

const char* moe_last_error(void);

/* ---------------------------------------------------------------- the pool */

/* The expert store in the 4096-byte aligned per-expert layout ("FTW": every
 * tensor 4096-aligned so that a miss is one large DMA; "跑不快大模型，先别急着怪
 * 显卡", section 三) and the HBM slot pool.  Block = [gate codes][gate scales]
 * [up codes][up scales][down codes][down scales], each padded to 4096 bytes;
 * the FP32 tensor scales stay resident in a small HBM table.  Allocates
 * n_slots blocks of HBM (cudaMalloc) and host_layers*E blocks of pinned host
 * memory (cudaHostAlloc).  Errors: MOE_EINVAL (shape), MOE_ENOMEM. */
int moe_pool_create(const moe_config* cfg, moe_pool** out);
int moe_pool_destroy(moe_pool* pool);
size_t moe_expert_block_bytes(const moe_config* cfg);

/* Pack one expert from the canonical layout into its pinned host block.  The
 * expert is not resident until a lookup misses it.  Errors: MOE_EBOUNDS. */
int moe_pool_load_expert(moe_pool* pool, int layer, int expert, const moe_expert_src* src);

/* Empty the slot pool (every expert back to host-only, LRU clock and tickets
 * reset, statistics cleared) and let later lookups use only the first
 * n_active_slots slots (1 .. n_slots).  Synchronises the device.  For sweeps of
 * the pool size and for a cold restart; the host store is kept. */
int moe_pool_reset(moe_pool* pool, int n_active_slots);

/* Copy the LRU state to host arrays (synchronous; for checks and checkpoints):
 * slot_key_h[n_slots] (layer*E+expert or -1), slot_clock_h[n_slots],
 * key_slot_h[L*E] (slot or -1), *clock_h = global clock. */
/* Resize the slot pool to n_active_slots in [1, n_slots] at run time, keeping the
 * LRU state (to trade slot-pool HBM for other memory, e.g. a KV cache): shrinking
 * evicts the residents with the oldest clocks until at most n_active_slots remain
 * and moves every survivor sitting above the new end, in slot order, to the
 * lowest free slot below it (a device-to-device copy of its block; its clock and
 * ready ticket move with it); growing adds empty slots.  Entries whose copy never
 * landed (ready ticket != needed ticket) are dropped first.  The global clock is
 * unchanged, so later lookups continue the same LRU order.  Synchronises the
 * device: call between steps with no pool work in flight.  Errors: MOE_EINVAL,
 * MOE_ESTATE (a launched lookup not collected), MOE_ECUDA. */
int moe_pool_resize(moe_pool* pool, int n_active_slots);

/* The resize decision on host copies of the first n_old slots' state (for
 * checks): evict_slot_h receives the evicted slots (oldest clock first),
 * move_from_h / move_to_h the moves, in order.  Arrays hold n_old entries.
 * Errors: MOE_EINVAL, MOE_ESTATE (inconsistent state). */
int moe_lru_plan_resize(const int32_t* slot_key_h, const uint64_t* slot_clock_h, int n_old, int n_new,
                        int32_t* evict_slot_h, int* n_evict, int32_t* move_from_h, int32_t* move_to_h,
                        int* n_move);

int moe_pool_read_state(moe_pool* pool, int32_t* slot_key_h, uint64_t* slot_clock_h,
                        int32_t* key_slot_h, uint64_t* clock_h);
int moe_pool_stats(const moe_pool* pool, moe_stats* out);
/* Device pointer and byte size of one slot (for checks). */
int moe_pool_slot_ptr(moe_pool* pool, int slot, void** ptr, size_t* bytes);

/* ---------------------------------------------------------------- the path */

/* Router (mubeitech "游戏电脑如何跑动2840亿参数大模型": the gate picks a few
 * experts per token; post.smzdm.com/p/a825qpgl section 二: 256 experts, 6
 * active).  logits[t,e] = sum_h x[t,h]*W_r[e,h] + bias[e] in fp32 with a fixed
 * order (lane j of 32 accumulates, by fmaf in ascending h, the 8-element chunks
 * c with c%32 == j; lanes are added by a xor-butterfly 16,8,4,2,1; then +bias),
 * top-k by descending logit with ties to the lower index, and
 * w = softmax over the k chosen (renormalize=1) or the full softmax read at the
 * chosen experts (renormalize=0).  bias may be NULL.  Outputs idx [T,k] int32
 * and w [T,k] fp32 in rank order.  workspace: device scratch of
 * moe_route_workspace_bytes(T, E) bytes, its counters zero before the first
 * use (the call leaves them zero).  Limits: H % 256 == 0, E <= 1024,
 * k <= min(E, 32), x and W_r 16-byte aligned (both are read 16 bytes at a
 * time).  Errors: MOE_EINVAL. */
size_t moe_route_workspace_bytes(int T, int E);
int moe_route(const void* x_bf16, const void* wr_bf16, const float* bias, int T, int H, int E,
              int k, int renormalize, int32_t* idx, float* w, void* workspace,
              size_t workspace_bytes, void* stream);

/* Router without allocation (no counterpart in the paper).  The same router as
 * moe_route, for callers that cannot allocate device memory where they route
 * (HBM fully handed out at start-up, or no cudaMalloc allowed inside a decode
 * step): its scratch is a static device array inside the library, so the caller
 * passes only inputs and outputs.  Limits: T <= 4096 and T*E <= 65536 (256 KiB
 * of logits), else MOE_EINVAL.  The first call on a device looks the array's
 * address up; make that first call before any stream capture.  Every call
 * shares the array: calls that overlap on the GPU race, so serialise them on
 * one stream.  The array's memory is held on every GPU that loads the library
 * until the process exits.  Allocates nothing (no cudaMalloc / cudaFree). */
int moe_route_noalloc(const void* x_bf16, const void* wr_bf16, const float* bias, int T, int H,
                      int E, int k, int renormalize, int32_t* idx, float* w, void* stream);

/* LRU slot lookup (post.smzdm.com/p/aomxznrn, "FreeToken干的事": a global LRU
 * expert-slot pool).  One kernel, one CTA: the unique experts of idx in
 * ascending id; hits are touched first (clock = ++G), then each miss takes the
 * lowest free slot, else the occupied slot not used by this call with the
 * oldest clock; a miss gets clock = ++G and a ticket.  Writes slot_of [T,k]
 * (device) and, after a bounded wait for the kernel (MOE_ETIMEOUT), fills
 * *res (host).  The pool must hold at least the call's unique experts. */
int moe_slot_lookup(moe_pool* pool, int layer, const int32_t* idx, int T, int k, int32_t* slot_of,
                    moe_lookup_result* res, void* stream);

/* The two halves of moe_slot_lookup, so that the FFN of the same layer can be
 * enqueued before the host learns the misses: _launch enqueues the lookup kernel
 * (slot_of and the slot tickets are then final in stream order); _result waits
 * (bounded, MOE_ETIMEOUT after 10 s) for it and fills *res.  One lookup may be
 * outstanding per pool (MOE_ESTATE otherwise). */
int moe_slot_lookup_launch(moe_pool* pool, int layer, const int32_t* idx, int T, int k,
                           int32_t* slot_of, void* stream);
int moe_slot_lookup_result(moe_pool* pool, moe_lookup_result* res);

/* Miss streaming ("游戏电脑如何跑动2840亿参数大模型": prefetch with a double
 * buffer, copies in the background while computing).  For each miss, in order,
 * the expert's pinned host block is copied into its slot on copy_stream (one
 * cudaMemcpyAsync per part, or a copy kernel in MOE_COPY_SM mode).  A block of
 * 8 MiB or more goes in two parts: first the gate and up tensors (codes and
 * scales, the block's leading bytes), then a stream write of
 * ticket | 0x80000000 into the slot's ready word; then the down tensors, then
 * a stream write of the ticket itself.  A smaller block goes in one copy
 * followed by the ticket.  moe_expert_ffn starts at
 * once on another stream; its gate/up work on a missed expert waits (bounded)
 * for the first value and its down work for the second, so the copy of miss j+1
 * overlaps compute on the hits and on miss j, and a miss's gate/up rows are
 * consumed while its down rows are still crossing.  When the FFN is enqueued before the misses are streamed
 * (moe_slot_lookup_launch, moe_expert_ffn, moe_slot_lookup_result, then this
 * call), the host must not wait for the device in between (a synchronize, a
 * blocking allocation, a first launch of a lazily loaded kernel): the FFN would
 * wait for copies not yet issued until its bounded wait gives up.  The pool
 * loads all of the library's kernels when it is created.  Errors: MOE_EBOUNDS, MOE_ESTATE (expert never loaded). */
int moe_stream_misses(moe_pool* pool, int layer, const moe_miss* miss_h, int n_miss,
                      void* copy_stream);

/* Select how moe_stream_misses copies (MOE_COPY_SM or MOE_COPY_DMA) for later
 * calls on this pool.  Both write the same bytes and publish the same ready
 * tickets.  In MOE_COPY_SM mode the decode FFN runs on 16 SMs fewer, which the
 * copy kernel it waits for uses.  Errors: MOE_EINVAL. */
int moe_pool_set_copy_mode(moe_pool* pool, int mode);

/* Decode expert FFN (post.smzdm.com/p/aomxznrn, "FreeToken干的事": decode is
 * bandwidth-bound and scheduled apart from prefill; post.smzdm.com/p/a825qpgl
 * section 二: expert results merged by routing weight).  For every (t, j):
 * y_part[t, j, :] = w[t,j] * Wd (silu(Wg x_t) * (Wu x_t)) of expert idx[t,j] read
 * from slot slot_of[t,j]; FP4 weights dequantised on the fly (MXFP4: e2m1 *
 * 2^(s-127); NVFP4: e2m1 * e4m3(s) * S_tensor).  Arithmetic: every product of a
 * weight and an activation is exact and the sums are fp32 (tensor-core MMA with
 * fp32 accumulation); x enters as f16 after a per-token power of two (exact for
 * bf16 x down to 2^-24 of the token's largest element), h as the sum of two f16
 * values (about 22 significant bits).  If y_bf16 is not NULL the call also does
 * the combine: y_bf16[t, :] = bf16(sum over j = 0..k-1 of y_part[t, j, :]),
 * summed in fp32 in rank order, round to nearest even (the same as moe_combine).
 * One CTA per SM computes it: CTA c takes the c-th share of the call's 16-row
 * gate/up tiles (all unique experts, ticket order) and then of its 16-row down
 * tiles; h goes through a pool-owned global buffer with a count per expert, and
 * down tiles wait (bounded) for their expert's count.  All CTAs are resident at
 * once and gate/up tiles wait only for their own copies and for the ready
 * tickets of missed experts, so every wait ends.  Calls on one pool must not
 * run concurrently (they share the buffer and the counts).  It is a plain launch with programmatic
 * stream serialisation: it stages x while the kernel before it (the slot lookup)
 * finishes, so x must be complete before that kernel starts (it is, when the
 * router ran on x first).  Waits are bounded (moe_set_wait_limits); failures set
 * bits of *status (device int, caller-zeroed; MOE_STATUS_*).  y_part is [T, k, H]
 * fp32, y_bf16 [T, H]; x, y_part and y_bf16 16-byte aligned.  Limits: T <=
 * max_tokens of the pool, and max(T * H, 2 * T * I) * 2 bytes of activation
 * fragments must fit in shared memory beside two weight stages (MOE_EINVAL
 * otherwise).
 * Errors: MOE_EINVAL. */
int moe_expert_ffn(moe_pool* pool, int layer, const void* x_bf16, int T, const int32_t* idx,
                   const float* w, const int32_t* slot_of, float* y_part, void* y_bf16, int* status,
                   void* stream);

/* Limits of the device-side bounded waits of moe_expert_ffn, in milliseconds:
 * a missed expert's ready flag (default 5000), the wait for other CTAs to
 * publish an expert's h (default 5000), a shared-memory pipeline stage
 * (default 10000).
 * Process-wide; affects later launches.  Errors: MOE_EINVAL (non-positive). */
int moe_set_wait_limits(double ready_ms, double dep_ms, double pipe_ms);

/* Launch shape moe_expert_ffn uses on this pool for T tokens (for reports):
 * CTAs launched, shared-memory weight stages per CTA and bytes per stage,
 * dynamic shared memory per CTA in bytes.  Errors: MOE_EINVAL. */
int moe_ffn_launch_info(moe_pool* pool, int T, int* ctas, int* nstage, int* stage_bytes, int* smem_bytes);

/* Tracing (for profiling): when buf is a device buffer of at least 32 u64 per
 * CTA of the largest launch (32 * 296 covers every launch), each CTA of every
 * later moe_expert_ffn launch writes, at row blockIdx * 32, global-timer stamps
 * in ns: [0] start, [1] activations staged, [2] the preceding kernel (the slot
 * lookup) complete, [3] group table built, [4] first weights landed, [5] the
 * CTA's gate/up tiles done, [6] h of its first down tile's expert complete,
 * [7] that h in shared memory, [8] the CTA's down tiles done, [9] the producer
 * about to issue its first copy, [10] end, [11] the producer's last copy
 * issued, [16 + s] the CTA's stage s landed (consumer side, s < 8), [24 + s] the
 * producer's copies of stage s issued (s < 8); and counts: [12] gate/up tiles
 * of the CTA, [13] its down tiles, [14] the K split of its gate/up units, [15]
 * the K split of its down groups.
 * Unwritten entries keep their old value.  NULL turns tracing off. */
int moe_set_ffn_trace(void* buf);

/* Block-scaled NVFP4 GEMM on the tcgen05 tensor cores (the contraction of
 * the prefill expert FFN; post.smzdm.com/p/aomxznrn "FreeToken干的事":
 * compute-bound prefill scheduled apart from decode).  D[M, N] (fp32,
 * row-major) = sum_k dq(A)[m, k] * dq(B)[n, k], where A [M, K] and B [N, K] are
 * E2M1 codes (K-contiguous, K/2 bytes per row) with E4M3 scales per 16 elements
 * in the canonical layout [rows, K/16]; no tensor scale (apply it to D).
 * Limits: M, N multiples of 128, K a multiple of 256, operands 16-byte aligned.
 * Bounded device waits set bit 16 of *status (device int) on timeout. */
int moe_nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                   const uint8_t* b_scales, int M, int N, int K, float* D, int* status, void* stream);

/* Prefill activation quantiser (the A operand of the prefill GEMMs): each
 * token row of x [T, H] bf16 -> NVFP4 with a per-token FP32 scale
 * S_x = amax(x_t) / (6*448), E4M3 scales per 16 elements
 * s = E4M3(amax_block / (6 S_x)) and codes E2M1(v / (e4m3(s) S_x)), both
 * round-to-nearest-even and saturating (all codes 0 when e4m3(s) S_x == 0).
 * Outputs codes [T, H/2], scales [T, H/16], sx [T].  Limits: H % 256 == 0. */
int moe_nvfp4_quantize(const void* x_bf16, int T, int H, uint8_t* codes, uint8_t* scales, float* sx,
                       void* stream);

/* Prefill expert FFN (post.smzdm.com/p/aomxznrn "FreeToken干的事": prefill is
 * compute-bound and scheduled apart from decode).  Groups the (token, rank)
 * pairs by expert, quantises x to NVFP4 (as moe_nvfp4_quantize), runs the
 * gate/up GEMM on tcgen05 with a fused SiLU*up epilogue that re-quantises h to
 * NVFP4 (tensor scale 1), then the down GEMM, whose epilogue applies the
 * routing weight and stores one row per (token, rank):
 * y[t, j, :] = w[t, j] * S_down * (W_down h)_t for expert idx[t, j] read from
 * slot slot_of[t, j] (all chosen experts resident); y is y_part [T, k, H] fp32,
 * every row written by the call.
 * NVFP4 pools only; the expert block layout must divide into rows of H/2, H/16,
 * I/2 and I/16 bytes (MOE_EINVAL otherwise).  workspace: device memory of
 * moe_prefill_workspace_bytes(pool, T) bytes.  Device-side waits are bounded
 * and set bit 16 of *status (device int) on timeout.  moe_combine(y, T, k, H,
 * y_bf16) sums the k rows of each token in rank order in fp32 and rounds to
 * bf16, as in decode, so the result does not depend on timing. */
size_t moe_prefill_workspace_bytes(const moe_pool* pool, int T);
int moe_prefill_ffn(moe_pool* pool, int layer, const void* x_bf16, int T, const int32_t* idx,
                    const float* w, const int32_t* slot_of, float* y, void* workspace,
                    size_t workspace_bytes, int* status, void* stream);

/* Router-weighted combine (post.smzdm.com/p/a825qpgl section 二: results merged
 * by routing weight): y[t, :] = bf16(sum over j = 0..k-1 of y_part[t, j, :]),
 * summed in fp32 in rank order, rounded to nearest even. */
int moe_combine(const float* y_part, int T, int k, int H, void* y_bf16, void* stream);

/* One decode MoE layer in one call (the engine's per-layer sequence,
 * post.smzdm.com/p/aomxznrn "FreeToken干的事": resident experts compute on the
 * GPU while missing ones cross PCIe).  Runs moe_route, moe_slot_lookup_launch,
 * moe_expert_ffn with the combine fused in (y_bf16), moe_slot_lookup_result (the
 * one host wait, bounded) and moe_stream_misses on copy_stream, with the
 * arguments and rules of those calls; k, H and E come from the pool.  Caller-owned device
 * buffers: idx, w, slot_of [T, k]; y_part [T, k, H] fp32; y_bf16 [T, H];
 * status (device int); route_ws of moe_route_workspace_bytes(T, E) bytes.
 * res: host arrays that receive the lookup result (capacity >= min(T*k, E)),
 * or NULL.  copy_start / copy_end: CUDA events recorded on copy_stream before
 * and after the miss copies when the layer has misses, or NULL.  With overlap,
 * copy_stream must be a non-blocking stream other than `stream` (the FFN waits for
 * copies issued after it; MOE_EINVAL if it is the same stream or NULL).  overlap = 0
 * waits for the miss list and issues the copies before the FFN is enqueued
 * (for tools that serialise kernels).  Returns the first failing call's error;
 * a launched lookup is collected even when the FFN launch fails. */
int moe_decode_layer(moe_pool* pool, int layer, const void* x_bf16, int T, const void* wr_bf16,
                     const float* bias, int renormalize, int32_t* idx, float* w, int32_t* slot_of,
                     float* y_part, void* y_bf16, int* status, void* route_ws,
                     size_t route_ws_bytes, moe_lookup_result* res, void* copy_start,
                     void* copy_end, int overlap, void* stream, void* copy_stream);

/* All-resident decode of layers layer0 .. layer0+n_layers-1 (post.smzdm.com/p/
 * aomxznrn, "FreeToken干的事": decode runs on its own bandwidth-bound path): one
 * decode FFN launch per layer with the router (the same logits, choices and
 * weights as moe_route, bit for bit), the slot lookup and the combine fused in,
 * on `stream`, with no host wait anywhere, so the call may be captured into a
 * CUDA graph and replayed.  Every expert the
 * layers touch must already be resident (for instance a pool with
 * n_slots >= L * E after one pass of moe_decode_layer): each expert's slot comes
 * from the pool's key table and the hits' LRU clocks are refreshed exactly as
 * moe_slot_lookup refreshes them (ascending expert id); nothing is evicted,
 * streamed or written to the lookup's host record; slot_of receives the slots.
 * An expert that is not resident leaves the pool untouched apart from the hits'
 * clocks, sets MOE_STATUS_NOT_RESIDENT and MOE_STATUS_BAD_SLOT in *status, and
 * that layer's output is not valid.  x_bf16: [n_layers, T, H] (device); y_bf16:
 * [n_layers, T, H]; wr_bf16, bias: host arrays of n_layers device pointers
 * ([E, H] bf16 router weights; [E] fp32 bias or NULL; bias itself may be NULL);
 * idx, w, slot_of ([T, k], written: the last layer's choices, weights and
 * slots), y_part ([T, k, H] fp32) and status as for moe_decode_layer, reused by
 * every layer in stream order.  No lookup may be outstanding on the pool while
 * it runs, and calls on one pool must not run concurrently.  Errors:
 * MOE_EINVAL, MOE_EBOUNDS, and those of moe_expert_ffn. */
int moe_decode_resident(moe_pool* pool, int layer0, int n_layers, const void* x_bf16, int T,
                        const void* const* wr_bf16, const float* const* bias, int renormalize,
                        int32_t* idx, float* w, int32_t* slot_of, float* y_part, void* y_bf16,
                        int* status, void* stream);

/* q* split (post.smzdm.com/p/a825qpgl section 二: q* = m*B_p/B_h; "跑不快大模型，
 * 先别急着怪显卡" section 二: pull : compute = pcie_bw : (cpu_bw - pcie_bw)).
 * ratio = B_p/B_h; q_gpu = min(m, floor(m*ratio + 0.5)); q_cpu = m - q_gpu.
 * Host only.  Errors: MOE_EINVAL (m < 0 or a bandwidth <= 0). */
int qstar_split(int m, double b_pcie, double b_host, int* q_gpu, int* q_cpu, double* ratio);

/* Run-time bandwidth adaptation of q* (post.smzdm.com/p/a825qpgl section 二: the
 * split follows the machine's measured PCIe and host-memory bandwidths; "跑不快大
 * 模型，先别急着怪显卡" section 二: pull : compute = pcie_bw : (cpu_bw - pcie_bw)).
 * A moving estimate of each bandwidth, fed with observed transfers, from which
 * q* is recomputed whenever the caller asks (e.g. every step).  Host only. */
enum { MOE_BW_PCIE = 0, MOE_BW_HOST = 1 };
typedef struct {
    double alpha;               /* weight of a new observation, in (0, 1] */
    double b_pcie, b_host;      /* current estimates in GB/s; 0 = not yet known */
    long long n_pcie, n_host;   /* observations folded in */
} moe_bw_estimate;
/* Reset: alpha in (0, 1]; initial estimates >= 0 (0 = unknown).  MOE_EINVAL. */
int moe_bw_init(moe_bw_estimate* est, double alpha, double b_pcie0, double b_host0);
/* Fold one transfer of `bytes` in `seconds` (both > 0) over link `which`:
 * est = obs if the estimate is unknown, else (1 - alpha) * est + alpha * obs,
 * obs = bytes / seconds / 1e9.  MOE_EINVAL on bad arguments. */
int moe_bw_observe(moe_bw_estimate* est, int which, double bytes, double seconds);
/* qstar_split(m, b_pcie, b_host) of the current estimates; MOE_ESTATE while
 * either bandwidth is unknown. */
int moe_bw_qstar(const moe_bw_estimate* est, int m, int* q_gpu, int* q_cpu, double* ratio);

/* Dequantise tensor `which` (0 gate, 1 up, 2 down) of the expert in `slot`
 * to fp32 [rows, K] in canonical order: (e2m1(c) * scale) * S_tensor, two fp32
 * multiplies (the second only for NVFP4).  key = layer*E + expert selects the
 * tensor scale.  For checks of the slot contents. */
int moe_dequant_slot(moe_pool* pool, int slot, int key, int which, float* out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_FP4_H */
