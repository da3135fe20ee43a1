// Internal declarations shared by the library's translation units: the pool
// object, error reporting, and thin wrappers over sm_100a PTX (mbarrier,
// bulk asynchronous copies, bounded waits on the global timer).
#pragma once

#include <cuda.h>
#include <utility>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <stdint.h>
#include <string>

#include "../../include/moe_fp4.h"

namespace moe {

// ----------------------------------------------------------------- errors

void set_error(const std::string& msg);
int fail(int code, const std::string& msg);
int cuda_fail(cudaError_t e, const char* what);

#define MOE_CUDA_TRY(expr)                                   \
    do {                                                     \
        cudaError_t e_ = (expr);                             \
        if (e_ != cudaSuccess) return cuda_fail(e_, #expr);  \
    } while (0)

// ----------------------------------------------------------------- limits

constexpr int kMaxE = 1024;          // experts per layer
constexpr int kMaxK = 32;            // experts per token
constexpr int kMaxDecodeT = 16;      // tokens of one decode FFN call
constexpr int kMaxDecodePairs = 128; // (token, rank) pairs of one decode FFN call
constexpr int kMaxSlots = 1 << 20;
// A slot's ready word shows (ticket | kTicketPartA) once the gate and up tensors of
// its copy have landed, then the ticket itself once the whole block has.
constexpr uint32_t kTicketPartA = 0x80000000u;

// Per-call output of the lookup kernel, in mapped pinned host memory.
struct LookupOut {
    int n_uniq, n_miss, status, seq;
    int32_t uniq[kMaxE];
    int32_t is_hit[kMaxE];
    moe_miss miss[kMaxE];
};

// Byte layout of one expert block (4096-aligned tensors).
struct BlockLayout {
    size_t off[6];     // gate codes, gate scales, up codes, up scales, down codes, down scales
    size_t bytes;      // whole block, multiple of 4096
};

BlockLayout block_layout(const moe_config& c);

// Force-load the library's kernels (lazy module loading can wait for the device,
// which must not happen while a decode FFN waits for copies the host has yet to issue).
int preload_router_kernels();
int preload_lookup_kernels();
int preload_ffn_kernels();
int preload_gemm_kernels();
int preload_prefill_kernels();
int preload_pull_kernels();
cudaError_t launch_pull(const uint8_t* src_d, uint8_t* dst, size_t bytes, int num_sms, cudaStream_t s);
// The router fused into a resident decode FFN: router weights [E, H] bf16, bias
// [E] or null, and the caller's idx / w, which the FFN writes.
struct FfnRoute {
    const void* wr;
    const float* bias;
    int renormalize;
    int32_t* idx;
    float* w;
};
// The decode FFN; resident != 0 takes the slots from the pool's key table and
// applies the slot lookup's LRU touch itself (no lookup kernel before it); route
// (resident only) routes the tokens inside the kernel (no router kernel either).
int expert_ffn(moe_pool* p, int layer, const void* x_bf16, int T, const int32_t* idx, const float* w,
               const int32_t* slot_of, float* y_part, void* y_bf16, int* status, void* stream, int resident,
               const FfnRoute* route);

}  // namespace moe

struct moe_pool {
    moe_config cfg;
    int bs;                       // elements per block scale
    moe::BlockLayout lay;
    int host_layers;
    int n_active;                 // slots the LRU may use (<= cfg.n_slots)
    int device;
    int num_sms;
    int ffn_smem;                 // shared-memory bytes the decode FFN may take per CTA
    // storage
    uint8_t* slots;               // device [n_slots][block]
    uint8_t* host;                // pinned, mapped [host_layers][E][block]
    const uint8_t* host_d;        // its device alias (read by the pull kernel)
    uint8_t* host_loaded;         // host flags [host_layers * E]
    int copy_mode;                // MOE_COPY_SM or MOE_COPY_DMA
    // LRU metadata (device)
    int32_t* slot_key;            // [n_slots]
    unsigned long long* slot_clock;  // [n_slots]
    int32_t* key_slot;            // [L*E]
    unsigned long long* clock;    // [1]
    uint32_t* ticket;             // [1]
    uint32_t* need;               // [n_slots] ticket the slot must show before use
    uint32_t* ready;              // [n_slots] ticket published by the copy stream
    float* tscale;                // [L*E*3] NVFP4 tensor scales
    // lookup output
    moe::LookupOut* lk_h;         // mapped pinned
    moe::LookupOut* lk_d;         // its device alias
    cudaEvent_t lk_event;
    int lk_seq;                   // sequence number of the last launched lookup
    int lk_pending;               // a launched lookup whose record was not collected
    int lk_attr_set;
    // decode FFN counters: [0, H/16) groups done per 16-row tile of H (the fused
    // combine), then per group the h values published, per (token, rank) the
    // largest |h| (float bits), kMaxDecodePairs words each, then the abort flag,
    // the count of finished CTAs and the fused router's count of experts done
    unsigned int* ctr;
    float* hbuf;                  // decode FFN: [kMaxDecodePairs][I] h of each (token, rank)
    float* rlogits;               // decode FFN's fused router: [kMaxDecodeT][E] logits
    // copy engine ready-flag write
    void* write_value32;          // cuStreamWriteValue32 entry point
    int ffn_grid[2][2];           // decode FFN CTAs per launch (0: not yet set up), per (format, token tiles)
    moe_stats stats;
};

// ----------------------------------------------------------------- PTX wrappers
#ifdef __CUDACC__
namespace moe {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;"
        " selp.u32 %0, 1, 0, p; }"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase; false after `limit_ns` of global time.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) return false;
    }
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_acquire_sys_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(unsigned int* p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Programmatic dependent launch: let the next kernel of the stream launch now;
// wait until the previous kernel of the stream has completed and its memory is
// visible (both are no-ops for kernels launched without the attribute).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host: launch `kern` with programmatic stream serialisation, so that it may
// start while the previous kernel of the stream runs (the kernel must
// pdl_wait() before it touches anything that kernel writes or reads).
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
}

// Named barrier over `nthreads` threads (a multiple of 32) with id `id` (1..15).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace moe
#endif
