// K2 slot lookup: one CTA applies one call's LRU update to the global slot pool.
//
// Order of the update (the oracle's order): the unique experts of idx in
// ascending id; hits are touched first (clock = ++G, ascending id), then each
// miss (ascending id) takes the lowest-index free slot, else the occupied slot
// not used by this call with the oldest clock, gets clock = ++G and a fresh
// ticket.  Because every touch draws a distinct clock, the victims of one call
// are the (misses - free) smallest clocks among the unpinned occupied slots, in
// ascending clock order; the kernel finds them by repeated block-wide argmin.
// Results go to slot_of (device) and to a mapped pinned host record that the
// host waits for (bounded) to drive the copy engine.
#include <atomic>
#include <chrono>
#include <thread>

#include "common.cuh"

namespace moe {

constexpr int kLookupThreads = 1024;

struct LookupArgs {
    const int32_t* idx;
    int n;           // T*k
    int layer, E, S;
    int32_t* slot_key;
    unsigned long long* slot_clock;
    int32_t* key_slot;
    unsigned long long* clock;
    uint32_t* ticket;
    uint32_t* need;
    int32_t* slot_of;
    LookupOut* out;
    int seq;
};

__device__ __forceinline__ bool key_less(unsigned long long ca, int sa, unsigned long long cb, int sb) {
    return ca < cb || (ca == cb && sa < sb);
}

__global__ void __launch_bounds__(kLookupThreads) lookup_kernel(LookupArgs a) {
    __shared__ uint32_t used[kMaxE / 32];
    __shared__ int32_t uniq[kMaxE];
    __shared__ int32_t uslot[kMaxE];
    __shared__ int16_t umap[kMaxE];
    __shared__ int32_t miss_u[kMaxE];
    __shared__ int32_t miss_slot[kMaxE];
    __shared__ int s_nu, s_nh, s_nm, s_bad, s_nfree;
    __shared__ int s_wcount[32];
    __shared__ unsigned long long s_wclk[32];
    __shared__ int s_wslot[32];
    extern __shared__ uint32_t bits[];  // pinned [ceil(S/32)], then victim [ceil(S/32)]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();      // idx comes from the router
    pdl_trigger();   // the expert FFN may launch and stage its activations meanwhile
    const int nwords = (a.S + 31) / 32;
    uint32_t* pinned = bits;
    uint32_t* victim = bits + nwords;

    for (int i = tid; i < kMaxE / 32; i += blockDim.x) used[i] = 0;
    for (int i = tid; i < 2 * nwords; i += blockDim.x) bits[i] = 0;
    if (tid == 0) s_bad = 0;
    __syncthreads();
    for (int i = tid; i < a.n; i += blockDim.x) {
        const int e = a.idx[i];
        if (e < 0 || e >= a.E) s_bad = 1;
        else atomicOr(&used[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            a.out->n_uniq = 0;
            a.out->n_miss = 0;
            a.out->status = MOE_STATUS_BAD_EXPERT;
            __threadfence_system();
            a.out->seq = a.seq;
        }
        return;
    }
    // compact the used experts in ascending id (one warp, a word per lane)
    if (warp == 0) {
        int base = 0;
        for (int w0 = 0; w0 < (a.E + 31) / 32; w0 += 32) {
            const int wi = w0 + lane;
            const uint32_t word = wi < (a.E + 31) / 32 ? used[wi] : 0u;
            const int cnt = __popc(word);
            int incl = cnt;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += v;
            }
            int pos = base + incl - cnt;
            for (uint32_t m = word; m; m &= m - 1) {
                const int e = wi * 32 + __ffs(m) - 1;
                uniq[pos] = e;
                umap[e] = (int16_t)pos;
                pos++;
            }
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_nu = base;
    }
    __syncthreads();
    const int nu = s_nu;
    for (int u = tid; u < nu; u += blockDim.x) uslot[u] = a.key_slot[a.layer * a.E + uniq[u]];
    __syncthreads();
    const unsigned long long G0 = *a.clock;
    const uint32_t tk0 = *a.ticket;
    if (tid == 0) {
        int nh = 0, nm = 0;
        for (int u = 0; u < nu; u++) {
            if (uslot[u] >= 0) {
                const int s = uslot[u];
                a.slot_clock[s] = G0 + 1 + nh;
                atomicOr(&pinned[s >> 5], 1u << (s & 31));
                nh++;
            } else {
                miss_u[nm++] = u;
            }
        }
        s_nh = nh;
        s_nm = nm;
    }
    __syncthreads();
    const int nh = s_nh, nm = s_nm;

    // free slots, lowest index first: ranks by a block-wide scan over contiguous ranges
    const int per = (a.S + blockDim.x - 1) / blockDim.x;
    const int s_lo = min(a.S, tid * per), s_hi = min(a.S, s_lo + per);
    int myfree = 0;
    if (nm > 0)
        for (int s = s_lo; s < s_hi; s++) myfree += a.slot_key[s] < 0;
    int incl = myfree;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
    }
    if (lane == 31) s_wcount[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x / 32;
        int v = lane < nw ? s_wcount[lane] : 0;
        int inc = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane < nw) s_wcount[lane] = inc - v;  // exclusive prefix of warps
        if (lane == 31) s_nfree = inc;
    }
    __syncthreads();
    if (nm > 0) {
        int r = s_wcount[warp] + incl - myfree;
        for (int s = s_lo; s < s_hi && r < nm; s++)
            if (a.slot_key[s] < 0) miss_slot[r++] = s;
    }
    const int nf = min(nm, s_nfree);
    __syncthreads();

    // victims: the (nm - nf) oldest unpinned occupied slots, one block argmin per victim
    for (int r = nf; r < nm; r++) {
        unsigned long long bc = ~0ull;
        int bs = 0x7fffffff;
        for (int s = s_lo; s < s_hi; s++) {
            if (a.slot_key[s] < 0) continue;
            if ((pinned[s >> 5] | victim[s >> 5]) & (1u << (s & 31))) continue;
            const unsigned long long c = a.slot_clock[s];
            if (key_less(c, s, bc, bs)) { bc = c; bs = s; }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const unsigned long long oc = __shfl_xor_sync(0xffffffffu, bc, off);
            const int os = __shfl_xor_sync(0xffffffffu, bs, off);
            if (key_less(oc, os, bc, bs)) { bc = oc; bs = os; }
        }
        if (lane == 0) { s_wclk[warp] = bc; s_wslot[warp] = bs; }
        __syncthreads();
        if (warp == 0) {
            const int nw = blockDim.x / 32;
            bc = lane < nw ? s_wclk[lane] : ~0ull;
            bs = lane < nw ? s_wslot[lane] : 0x7fffffff;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const unsigned long long oc = __shfl_xor_sync(0xffffffffu, bc, off);
                const int os = __shfl_xor_sync(0xffffffffu, bs, off);
                if (key_less(oc, os, bc, bs)) { bc = oc; bs = os; }
            }
            if (lane == 0) {
                // the host checks capacity >= unique experts, so a candidate exists
                miss_slot[r] = bs < a.S ? bs : 0;
                if (bs < a.S) victim[bs >> 5] |= 1u << (bs & 31);
                else s_bad = 1;
            }
        }
        __syncthreads();
    }

    // apply the misses in ascending expert id
    if (tid == 0) {
        for (int r = 0; r < nm; r++) {
            const int u = miss_u[r], s = miss_slot[r];
            const int key = a.layer * a.E + uniq[u];
            const int old = a.slot_key[s];
            if (old >= 0) a.key_slot[old] = -1;
            a.slot_key[s] = key;
            a.key_slot[key] = s;
            a.slot_clock[s] = G0 + nh + 1 + r;
            const uint32_t tk = tk0 + 1 + r;
            a.need[s] = tk;
            uslot[u] = s;
            moe_miss m;
            m.expert = uniq[u];
            m.slot = s;
            m.ticket = tk;
            m.evicted_key = old;
            a.out->miss[r] = m;
        }
        *a.clock = G0 + nu;
        *a.ticket = tk0 + nm;
    }
    __syncthreads();
    for (int u = tid; u < nu; u += blockDim.x) {
        a.out->uniq[u] = uniq[u];
        a.out->is_hit[u] = 0;
    }
    __syncthreads();
    if (tid == 0) {
        // hits are the unique experts that are not in the miss list
        for (int u = 0; u < nu; u++) a.out->is_hit[u] = 1;
        for (int r = 0; r < nm; r++) a.out->is_hit[miss_u[r]] = 0;
    }
    for (int i = tid; i < a.n; i += blockDim.x) a.slot_of[i] = uslot[umap[a.idx[i]]];
    __syncthreads();
    if (tid == 0) {
        // the host polls seq in mapped memory: the record (and the miss list and
        // slot state above) must be visible system-wide before seq is
        a.out->n_uniq = nu;
        a.out->n_miss = nm;
        a.out->status = 0;
        __threadfence_system();
        a.out->seq = a.seq;
    }
}

int preload_lookup_kernels() {
    cudaFuncAttributes fa;
    MOE_CUDA_TRY(cudaFuncGetAttributes(&fa, lookup_kernel));
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" int moe_slot_lookup_launch(moe_pool* p, int layer, const int32_t* idx, int T, int k,
                                      int32_t* slot_of, void* stream) {
    if (!p || !idx || !slot_of) return fail(MOE_EINVAL, "null argument");
    const moe_config& c = p->cfg;
    if (layer < 0 || layer >= c.L) return fail(MOE_EBOUNDS, "layer outside the pool");
    if (T <= 0 || k <= 0 || k > c.E || (long long)T * k > (1LL << 24)) return fail(MOE_EINVAL, "bad T/k");
    // the pool must hold every expert one call can touch, or a miss finds no victim
    const int cap = T * k < c.E ? T * k : c.E;
    if (cap > p->n_active) return fail(MOE_EINVAL, "slot pool smaller than the unique experts one call can touch");
    if (p->lk_pending) return fail(MOE_ESTATE, "a launched lookup has not been collected");
    cudaStream_t s = (cudaStream_t)stream;
    LookupArgs a;
    a.idx = idx;
    a.n = T * k;
    a.layer = layer;
    a.E = c.E;
    a.S = p->n_active;
    a.slot_key = p->slot_key;
    a.slot_clock = p->slot_clock;
    a.key_slot = p->key_slot;
    a.clock = p->clock;
    a.ticket = p->ticket;
    a.need = p->need;
    a.slot_of = slot_of;
    a.out = p->lk_d;
    a.seq = ++p->lk_seq;
    const size_t smem = size_t(2) * ((p->n_active + 31) / 32) * sizeof(uint32_t);
    if (smem > 160 * 1024) return fail(MOE_EINVAL, "n_slots too large for the lookup kernel");
    if (!p->lk_attr_set) {
        MOE_CUDA_TRY(cudaFuncSetAttribute(lookup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024));
        p->lk_attr_set = 1;
    }
    {
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3(1);
        lc.blockDim = dim3(kLookupThreads);
        lc.dynamicSmemBytes = smem;
        lc.stream = s;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = at;
        lc.numAttrs = 1;
        MOE_CUDA_TRY(cudaLaunchKernelEx(&lc, lookup_kernel, a));
    }
    MOE_CUDA_TRY(cudaEventRecord(p->lk_event, s));
    p->lk_pending = 1;
    return MOE_OK;
}

extern "C" int moe_slot_lookup_result(moe_pool* p, moe_lookup_result* res) {
    if (!p || !res) return fail(MOE_EINVAL, "null argument");
    if (!res->uniq_h || !res->is_hit_h || !res->miss_h) return fail(MOE_EINVAL, "null result arrays");
    if (!p->lk_pending) return fail(MOE_ESTATE, "no launched lookup to collect");
    // bounded host wait: the copy engine can only be driven once the miss list is
    // known.  The record's seq (written last, behind a system fence) shows it as
    // soon as the kernel writes it; the completion event catches a failed launch.
    volatile LookupOut* o = p->lk_h;
    const auto t0 = std::chrono::steady_clock::now();
    for (unsigned it = 0;; it++) {
        if (o->seq == p->lk_seq) break;
        if ((it & 63) == 63) {
            cudaError_t q = cudaEventQuery(p->lk_event);
            if (q == cudaSuccess) {
                if (o->seq == p->lk_seq) break;
                p->lk_pending = 0;
                return fail(MOE_ECUDA, "lookup record not written");
            }
            if (q != cudaErrorNotReady) {
                p->lk_pending = 0;
                return cuda_fail(q, "lookup kernel");
            }
            if (std::chrono::steady_clock::now() - t0 > std::chrono::seconds(10))
                return fail(MOE_ETIMEOUT, "lookup kernel did not finish within 10 s");
        }
    }
    std::atomic_thread_fence(std::memory_order_acquire);
    p->lk_pending = 0;
    if (o->seq != p->lk_seq) return fail(MOE_ECUDA, "lookup record not written");
    if (o->status) return fail(MOE_EBOUNDS, "expert index outside [0, E)");
    res->n_uniq = o->n_uniq;
    res->n_miss = o->n_miss;
    for (int u = 0; u < o->n_uniq; u++) {
        res->uniq_h[u] = o->uniq[u];
        res->is_hit_h[u] = o->is_hit[u];
    }
    for (int r = 0; r < o->n_miss; r++) {
        moe_miss m;
        m.expert = o->miss[r].expert;
        m.slot = o->miss[r].slot;
        m.ticket = o->miss[r].ticket;
        m.evicted_key = o->miss[r].evicted_key;
        res->miss_h[r] = m;
    }
    p->stats.lookups += 1;
    p->stats.unique += o->n_uniq;
    p->stats.misses += o->n_miss;
    p->stats.hits += o->n_uniq - o->n_miss;
    for (int r = 0; r < o->n_miss; r++) p->stats.evictions += o->miss[r].evicted_key >= 0;
    return MOE_OK;
}

extern "C" int moe_slot_lookup(moe_pool* p, int layer, const int32_t* idx, int T, int k,
                               int32_t* slot_of, moe_lookup_result* res, void* stream) {
    if (!res) return fail(MOE_EINVAL, "null argument");
    if (!res->uniq_h || !res->is_hit_h || !res->miss_h) return fail(MOE_EINVAL, "null result arrays");
    int rc = moe_slot_lookup_launch(p, layer, idx, T, k, slot_of, stream);
    if (rc) return rc;
    return moe_slot_lookup_result(p, res);
}
