// Pool ownership (HBM slots, pinned host expert store, LRU metadata), the copy
// engine miss streaming, the q* split and error reporting.
#include <cstdio>
#include <cstring>
#include <cmath>
#include <string>

#include <vector>

#include "common.cuh"

namespace moe {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

int fail(int code, const std::string& msg) {
    set_error(msg);
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    set_error(std::string(what) + ": " + cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? MOE_ENOMEM : MOE_ECUDA;
}

static size_t align4k(size_t n) { return (n + 4095) & ~size_t(4095); }

BlockLayout block_layout(const moe_config& c) {
    // [gate codes][gate scales][up codes][up scales][down codes][down scales],
    // every tensor starting on a 4096-byte boundary
    const size_t bs = c.fmt == MOE_MXFP4 ? 32 : 16;
    const size_t sz[6] = {size_t(c.I) * c.H / 2, size_t(c.I) * c.H / bs,
                          size_t(c.I) * c.H / 2, size_t(c.I) * c.H / bs,
                          size_t(c.H) * c.I / 2, size_t(c.H) * c.I / bs};
    BlockLayout L{};
    size_t o = 0;
    for (int i = 0; i < 6; i++) {
        L.off[i] = o;
        o += align4k(sz[i]);
    }
    L.bytes = o;
    return L;
}

static int check_config(const moe_config* c) {
    if (!c) return fail(MOE_EINVAL, "null config");
    if (c->fmt != MOE_MXFP4 && c->fmt != MOE_NVFP4) return fail(MOE_EINVAL, "fmt must be MXFP4 or NVFP4");
    if (c->H <= 0 || c->H % 256 || c->I <= 0 || c->I % 256)
        return fail(MOE_EINVAL, "H and I must be positive multiples of 256");
    if (c->E <= 0 || c->E > kMaxE) return fail(MOE_EINVAL, "E must be in [1, 1024]");
    if (c->k <= 0 || c->k > kMaxK || c->k > c->E) return fail(MOE_EINVAL, "k must be in [1, min(E, 32)]");
    if (c->L <= 0) return fail(MOE_EINVAL, "L must be positive");
    if (c->n_slots <= 0 || c->n_slots > kMaxSlots) return fail(MOE_EINVAL, "n_slots out of range");
    if (c->max_tokens <= 0 || c->max_tokens > kMaxDecodeT || c->max_tokens * c->k > kMaxDecodePairs)
        return fail(MOE_EINVAL, "max_tokens must be in [1, 16] with max_tokens*k <= 128");
    if (c->host_layers < 0 || c->host_layers > c->L) return fail(MOE_EINVAL, "host_layers out of range");
    if ((long long)c->L * c->E > (1LL << 30)) return fail(MOE_EINVAL, "too many experts");
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" const char* moe_last_error(void) { return g_last_error.c_str(); }

extern "C" size_t moe_expert_block_bytes(const moe_config* cfg) {
    if (check_config(cfg) != MOE_OK) return 0;
    return block_layout(*cfg).bytes;
}

extern "C" int moe_pool_destroy(moe_pool* p) {
    if (!p) return MOE_OK;
    int prev = -1;
    cudaGetDevice(&prev);
    cudaSetDevice(p->device);
    cudaDeviceSynchronize();
    cudaFree(p->slots);
    cudaFree(p->slot_key);
    cudaFree(p->slot_clock);
    cudaFree(p->key_slot);
    cudaFree(p->clock);
    cudaFree(p->ticket);
    cudaFree(p->need);
    cudaFree(p->ready);
    cudaFree(p->tscale);
    cudaFree(p->ctr);
    cudaFree(p->hbuf);
    cudaFree(p->rlogits);
    if (p->host) cudaFreeHost(p->host);
    if (p->lk_h) cudaFreeHost(p->lk_h);
    if (p->lk_event) cudaEventDestroy(p->lk_event);
    delete[] p->host_loaded;
    if (prev >= 0) cudaSetDevice(prev);
    delete p;
    return MOE_OK;
}

extern "C" int moe_pool_create(const moe_config* cfg, moe_pool** out) {
    if (!out) return fail(MOE_EINVAL, "null out");
    *out = nullptr;
    int rc = check_config(cfg);
    if (rc) return rc;
    moe_pool* p = new moe_pool();
    memset(p, 0, sizeof(*p));
    p->cfg = *cfg;
    p->bs = cfg->fmt == MOE_MXFP4 ? 32 : 16;
    p->lay = block_layout(*cfg);
    p->host_layers = cfg->host_layers ? cfg->host_layers : cfg->L;
    p->n_active = cfg->n_slots;
    cudaGetDevice(&p->device);
    cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device);
    {
        // the decode FFN (one CTA per SM) leaves room for the shared-memory
        // reservation of one more CTA, so that the miss-copy kernel it waits for
        // can run beside it on every SM
        int per_sm = 0, reserved = 0, optin = 0;
        cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, p->device);
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, p->device);
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, p->device);
        p->ffn_smem = std::min(optin, per_sm - 2 * reserved - 1024);
    }
    const size_t S = cfg->n_slots, LE = size_t(cfg->L) * cfg->E;
    const size_t host_bytes = size_t(p->host_layers) * cfg->E * p->lay.bytes;
    cudaError_t e;
#define ALLOC(ptr, bytes)                                          \
    e = cudaMalloc((void**)&(ptr), (bytes));                       \
    if (e != cudaSuccess) { rc = cuda_fail(e, "cudaMalloc " #ptr); moe_pool_destroy(p); return rc; }
    ALLOC(p->slots, S * p->lay.bytes);
    ALLOC(p->slot_key, S * sizeof(int32_t));
    ALLOC(p->slot_clock, S * sizeof(unsigned long long));
    ALLOC(p->key_slot, LE * sizeof(int32_t));
    ALLOC(p->clock, sizeof(unsigned long long));
    ALLOC(p->ticket, sizeof(uint32_t));
    ALLOC(p->need, S * sizeof(uint32_t));
    ALLOC(p->ready, S * sizeof(uint32_t));
    ALLOC(p->tscale, LE * 3 * sizeof(float));
    ALLOC(p->ctr, ((size_t)cfg->H / 16 + 2 * kMaxDecodePairs + 8) * sizeof(unsigned int));
    ALLOC(p->hbuf, (size_t)kMaxDecodePairs * cfg->I * sizeof(float));
    ALLOC(p->rlogits, (size_t)kMaxDecodeT * cfg->E * sizeof(float));
#undef ALLOC
    cudaMemset(p->slot_key, 0xFF, S * sizeof(int32_t));
    cudaMemset(p->slot_clock, 0, S * sizeof(unsigned long long));
    cudaMemset(p->key_slot, 0xFF, LE * sizeof(int32_t));
    cudaMemset(p->clock, 0, sizeof(unsigned long long));
    cudaMemset(p->ticket, 0, sizeof(uint32_t));
    cudaMemset(p->need, 0, S * sizeof(uint32_t));
    cudaMemset(p->ready, 0, S * sizeof(uint32_t));
    cudaMemset(p->tscale, 0, LE * 3 * sizeof(float));
    cudaMemset(p->ctr, 0, ((size_t)cfg->H / 16 + 2 * kMaxDecodePairs + 8) * sizeof(unsigned int));
    e = cudaHostAlloc((void**)&p->host, host_bytes, cudaHostAllocMapped);
    if (e != cudaSuccess) {
        p->host = nullptr;
        rc = cuda_fail(e, "cudaHostAlloc (pinned expert store)");
        moe_pool_destroy(p);
        return rc;
    }
    {
        void* hd = nullptr;
        e = cudaHostGetDevicePointer(&hd, p->host, 0);
        if (e != cudaSuccess) { rc = cuda_fail(e, "cudaHostGetDevicePointer (expert store)"); moe_pool_destroy(p); return rc; }
        p->host_d = (const uint8_t*)hd;
    }
    p->copy_mode = MOE_COPY_DMA;
    e = cudaHostAlloc((void**)&p->lk_h, sizeof(LookupOut), cudaHostAllocMapped);
    if (e != cudaSuccess) {
        p->lk_h = nullptr;
        rc = cuda_fail(e, "cudaHostAlloc (lookup output)");
        moe_pool_destroy(p);
        return rc;
    }
    memset(p->lk_h, 0, sizeof(LookupOut));
    e = cudaHostGetDevicePointer((void**)&p->lk_d, p->lk_h, 0);
    if (e != cudaSuccess) { rc = cuda_fail(e, "cudaHostGetDevicePointer"); moe_pool_destroy(p); return rc; }
    e = cudaEventCreateWithFlags(&p->lk_event, cudaEventDisableTiming);
    if (e != cudaSuccess) { rc = cuda_fail(e, "cudaEventCreate"); moe_pool_destroy(p); return rc; }
    p->host_loaded = new uint8_t[size_t(p->host_layers) * cfg->E]();
    cudaDriverEntryPointQueryResult q;
    e = cudaGetDriverEntryPoint("cuStreamWriteValue32", &p->write_value32, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p->write_value32) {
        rc = fail(MOE_ECUDA, "cuStreamWriteValue32 entry point not available");
        moe_pool_destroy(p);
        return rc;
    }
    if ((rc = preload_router_kernels()) || (rc = preload_lookup_kernels()) || (rc = preload_ffn_kernels()) ||
        (rc = preload_gemm_kernels()) || (rc = preload_prefill_kernels()) || (rc = preload_pull_kernels())) {
        moe_pool_destroy(p);
        return rc;
    }
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) { rc = cuda_fail(e, "pool init"); moe_pool_destroy(p); return rc; }
    *out = p;
    return MOE_OK;
}

extern "C" int moe_pool_load_expert(moe_pool* p, int layer, int expert, const moe_expert_src* src) {
    if (!p || !src) return fail(MOE_EINVAL, "null argument");
    const moe_config& c = p->cfg;
    if (layer < 0 || layer >= p->host_layers || expert < 0 || expert >= c.E)
        return fail(MOE_EBOUNDS, "layer/expert outside the host store");
    const size_t bs = p->bs;
    const size_t sz[6] = {size_t(c.I) * c.H / 2, size_t(c.I) * c.H / bs,
                          size_t(c.I) * c.H / 2, size_t(c.I) * c.H / bs,
                          size_t(c.H) * c.I / 2, size_t(c.H) * c.I / bs};
    const uint8_t* srcs[6] = {src->codes_h[0], src->scales_h[0], src->codes_h[1],
                              src->scales_h[1], src->codes_h[2], src->scales_h[2]};
    uint8_t* blk = p->host + (size_t(layer) * c.E + expert) * p->lay.bytes;
    for (int i = 0; i < 6; i++) {
        if (!srcs[i]) return fail(MOE_EINVAL, "null tensor pointer");
        memcpy(blk + p->lay.off[i], srcs[i], sz[i]);
        size_t end = (i == 5 ? p->lay.bytes : p->lay.off[i + 1]);
        memset(blk + p->lay.off[i] + sz[i], 0, end - p->lay.off[i] - sz[i]);
    }
    // tensor scales of every layer position stored at this host layer
    float ts[3];
    for (int i = 0; i < 3; i++) ts[i] = c.fmt == MOE_NVFP4 ? src->tensor_scale[i] : 1.0f;
    for (int l = layer; l < c.L; l += p->host_layers) {
        cudaError_t e = cudaMemcpy(p->tscale + (size_t(l) * c.E + expert) * 3, ts, sizeof(ts),
                                   cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "tensor scale upload");
    }
    p->host_loaded[size_t(layer) * c.E + expert] = 1;
    return MOE_OK;
}

extern "C" int moe_pool_reset(moe_pool* p, int n_active_slots) {
    if (!p) return fail(MOE_EINVAL, "null pool");
    if (n_active_slots <= 0 || n_active_slots > p->cfg.n_slots)
        return fail(MOE_EINVAL, "reset: active slots must be in [1, n_slots]");
    if (p->lk_pending) return fail(MOE_ESTATE, "reset: a launched lookup has not been collected");
    const size_t S = p->cfg.n_slots, LE = size_t(p->cfg.L) * p->cfg.E;
    MOE_CUDA_TRY(cudaDeviceSynchronize());
    MOE_CUDA_TRY(cudaMemset(p->slot_key, 0xFF, S * sizeof(int32_t)));
    MOE_CUDA_TRY(cudaMemset(p->slot_clock, 0, S * sizeof(unsigned long long)));
    MOE_CUDA_TRY(cudaMemset(p->key_slot, 0xFF, LE * sizeof(int32_t)));
    MOE_CUDA_TRY(cudaMemset(p->clock, 0, sizeof(unsigned long long)));
    MOE_CUDA_TRY(cudaMemset(p->ticket, 0, sizeof(uint32_t)));
    MOE_CUDA_TRY(cudaMemset(p->need, 0, S * sizeof(uint32_t)));
    MOE_CUDA_TRY(cudaMemset(p->ready, 0, S * sizeof(uint32_t)));
    p->n_active = n_active_slots;
    memset(&p->stats, 0, sizeof(p->stats));
    return MOE_OK;
}

extern "C" int moe_lru_plan_resize(const int32_t* slot_key_h, const uint64_t* slot_clock_h, int n_old, int n_new,
                                   int32_t* evict_slot_h, int* n_evict, int32_t* move_from_h, int32_t* move_to_h,
                                   int* n_move) {
    if (!slot_key_h || !slot_clock_h || !evict_slot_h || !n_evict || !move_from_h || !move_to_h || !n_move)
        return fail(MOE_EINVAL, "null argument");
    if (n_old < 1 || n_new < 1) return fail(MOE_EINVAL, "resize plan: slot counts must be >= 1");
    *n_evict = 0;
    *n_move = 0;
    if (n_new >= n_old) return MOE_OK;                   // growing: new slots start empty
    // residents ordered by last touch, oldest first; the oldest go until n_new remain
    std::vector<std::pair<uint64_t, int>> res;
    for (int s = 0; s < n_old; s++)
        if (slot_key_h[s] >= 0) res.push_back({slot_clock_h[s], s});
    std::sort(res.begin(), res.end());
    const int drop = std::max(0, (int)res.size() - n_new);
    std::vector<char> gone(n_old, 0);
    for (int i = 0; i < drop; i++) {
        evict_slot_h[(*n_evict)++] = res[i].second;
        gone[res[i].second] = 1;
    }
    // survivors above the new end, in slot order, into the lowest free slots below it
    int dst = 0;
    for (int s = n_new; s < n_old; s++) {
        if (slot_key_h[s] < 0 || gone[s]) continue;
        while (dst < n_new && slot_key_h[dst] >= 0 && !gone[dst]) dst++;
        if (dst >= n_new) return fail(MOE_ESTATE, "resize plan: no free slot (inconsistent state)");
        move_from_h[*n_move] = s;
        move_to_h[*n_move] = dst;
        (*n_move)++;
        dst++;
    }
    return MOE_OK;
}

extern "C" int moe_pool_resize(moe_pool* p, int n_new) {
    if (!p) return fail(MOE_EINVAL, "null pool");
    if (n_new < 1 || n_new > p->cfg.n_slots) return fail(MOE_EINVAL, "resize: active slots must be in [1, n_slots]");
    if (p->lk_pending) return fail(MOE_ESTATE, "resize: a launched lookup has not been collected");
    const int S = p->cfg.n_slots, n_old = p->n_active;
    const size_t LE = size_t(p->cfg.L) * p->cfg.E;
    MOE_CUDA_TRY(cudaDeviceSynchronize());
    std::vector<int32_t> sk(S), ks(LE);
    std::vector<uint64_t> sc(S);
    std::vector<uint32_t> need(S), ready(S);
    MOE_CUDA_TRY(cudaMemcpy(sk.data(), p->slot_key, S * 4, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(sc.data(), p->slot_clock, S * 8, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(ks.data(), p->key_slot, LE * 4, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(need.data(), p->need, S * 4, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(ready.data(), p->ready, S * 4, cudaMemcpyDeviceToHost));
    // an entry whose copy never landed holds no expert: drop it first
    for (int s = 0; s < n_old; s++)
        if (sk[s] >= 0 && ready[s] != need[s]) {
            ks[sk[s]] = -1;
            sk[s] = -1;
            sc[s] = 0;
        }
    std::vector<int32_t> ev(S), mf(S), mt(S);
    int ne = 0, nm = 0;
    int rc = moe_lru_plan_resize(sk.data(), sc.data(), n_old, n_new, ev.data(), &ne, mf.data(), mt.data(), &nm);
    if (rc) return rc;
    for (int i = 0; i < ne; i++) {
        const int s = ev[i];
        ks[sk[s]] = -1;
        sk[s] = -1;
        sc[s] = 0;
    }
    for (int i = 0; i < nm; i++) {
        const int from = mf[i], to = mt[i];
        MOE_CUDA_TRY(cudaMemcpy(p->slots + size_t(to) * p->lay.bytes, p->slots + size_t(from) * p->lay.bytes,
                                p->lay.bytes, cudaMemcpyDeviceToDevice));
        sk[to] = sk[from];
        sc[to] = sc[from];
        ks[sk[to]] = to;
        need[to] = ready[to] = need[from];   // the block is present: its ticket is published
        sk[from] = -1;
        sc[from] = 0;
    }
    for (int s = std::min(n_old, n_new); s < S; s++) {   // slots outside the active range are empty
        sk[s] = -1;
        sc[s] = 0;
    }
    MOE_CUDA_TRY(cudaMemcpy(p->slot_key, sk.data(), S * 4, cudaMemcpyHostToDevice));
    MOE_CUDA_TRY(cudaMemcpy(p->slot_clock, sc.data(), S * 8, cudaMemcpyHostToDevice));
    MOE_CUDA_TRY(cudaMemcpy(p->key_slot, ks.data(), LE * 4, cudaMemcpyHostToDevice));
    MOE_CUDA_TRY(cudaMemcpy(p->need, need.data(), S * 4, cudaMemcpyHostToDevice));
    MOE_CUDA_TRY(cudaMemcpy(p->ready, ready.data(), S * 4, cudaMemcpyHostToDevice));
    p->n_active = n_new;
    p->stats.evictions += ne;
    return MOE_OK;
}

extern "C" int moe_pool_read_state(moe_pool* p, int32_t* slot_key_h, uint64_t* slot_clock_h,
                                   int32_t* key_slot_h, uint64_t* clock_h) {
    if (!p) return fail(MOE_EINVAL, "null pool");
    const size_t S = p->cfg.n_slots, LE = size_t(p->cfg.L) * p->cfg.E;
    if (slot_key_h) MOE_CUDA_TRY(cudaMemcpy(slot_key_h, p->slot_key, S * 4, cudaMemcpyDeviceToHost));
    if (slot_clock_h) MOE_CUDA_TRY(cudaMemcpy(slot_clock_h, p->slot_clock, S * 8, cudaMemcpyDeviceToHost));
    if (key_slot_h) MOE_CUDA_TRY(cudaMemcpy(key_slot_h, p->key_slot, LE * 4, cudaMemcpyDeviceToHost));
    if (clock_h) MOE_CUDA_TRY(cudaMemcpy(clock_h, p->clock, 8, cudaMemcpyDeviceToHost));
    return MOE_OK;
}

extern "C" int moe_pool_stats(const moe_pool* p, moe_stats* out) {
    if (!p || !out) return fail(MOE_EINVAL, "null argument");
    *out = p->stats;
    return MOE_OK;
}

extern "C" int moe_pool_slot_ptr(moe_pool* p, int slot, void** ptr, size_t* bytes) {
    if (!p || !ptr || !bytes) return fail(MOE_EINVAL, "null argument");
    if (slot < 0 || slot >= p->cfg.n_slots) return fail(MOE_EBOUNDS, "slot outside the pool");
    *ptr = p->slots + size_t(slot) * p->lay.bytes;
    *bytes = p->lay.bytes;
    return MOE_OK;
}

typedef CUresult (*write_value32_fn)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);

constexpr size_t kSplitBytes = size_t(8) << 20;   // blocks at least this large are copied in two parts

extern "C" int moe_stream_misses(moe_pool* p, int layer, const moe_miss* miss_h, int n_miss,
                                 void* copy_stream) {
    if (!p) return fail(MOE_EINVAL, "null pool");
    if (n_miss < 0 || (n_miss > 0 && !miss_h)) return fail(MOE_EINVAL, "bad miss list");
    const moe_config& c = p->cfg;
    if (layer < 0 || layer >= c.L) return fail(MOE_EBOUNDS, "layer outside the pool");
    cudaStream_t s = (cudaStream_t)copy_stream;
    const int hl = layer % p->host_layers;
    // validate the whole list before queueing anything
    for (int i = 0; i < n_miss; i++) {
        const moe_miss& m = miss_h[i];
        if (m.slot < 0 || m.slot >= c.n_slots || m.expert < 0 || m.expert >= c.E)
            return fail(MOE_EBOUNDS, "miss slot/expert outside the pool");
        if (!p->host_loaded[size_t(hl) * c.E + m.expert])
            return fail(MOE_ESTATE, "missed expert was never loaded into the host store");
    }
    auto wv = (write_value32_fn)p->write_value32;
    // large blocks go in two parts: gate and up (codes and scales, the block's
    // first bytes), published as ticket | kTicketPartA, then down, published as
    // the ticket; the FFN starts a missed expert's gate/up rows while its down
    // rows are still crossing.  A block under kSplitBytes goes in one copy: the
    // second copy's fixed cost outweighs the overlap there.
    const size_t part_a = p->lay.off[4];
    const int parts = p->lay.bytes >= kSplitBytes ? 2 : 1;
    for (int i = 0; i < n_miss; i++) {
        const moe_miss& m = miss_h[i];
        const uint8_t* src = p->host + (size_t(hl) * c.E + m.expert) * p->lay.bytes;
        uint8_t* dst = p->slots + size_t(m.slot) * p->lay.bytes;
        for (int part = 2 - parts; part < 2; part++) {
            const size_t o = part && parts == 2 ? part_a : 0;
            const size_t n = parts == 1 ? p->lay.bytes : part ? p->lay.bytes - part_a : part_a;
            if (p->copy_mode == MOE_COPY_DMA) {
                MOE_CUDA_TRY(cudaMemcpyAsync(dst + o, src + o, n, cudaMemcpyHostToDevice, s));
            } else {
                MOE_CUDA_TRY(launch_pull(p->host_d + (src - p->host) + o, dst + o, n, p->num_sms, s));
            }
            const uint32_t v = part ? m.ticket : (m.ticket | kTicketPartA);
            CUresult r = wv((CUstream)s, (CUdeviceptr)(p->ready + m.slot), v, 0);
            if (r != CUDA_SUCCESS) return fail(MOE_ECUDA, "cuStreamWriteValue32 failed");
        }
        p->stats.h2d_bytes += (long long)p->lay.bytes;
        p->stats.h2d_copies += 1;
    }
    return MOE_OK;
}

extern "C" int moe_pool_set_copy_mode(moe_pool* p, int mode) {
    if (!p) return fail(MOE_EINVAL, "null pool");
    if (mode != MOE_COPY_SM && mode != MOE_COPY_DMA) return fail(MOE_EINVAL, "copy mode: MOE_COPY_SM or MOE_COPY_DMA");
    p->copy_mode = mode;
    return MOE_OK;
}

extern "C" int moe_bw_init(moe_bw_estimate* est, double alpha, double b_pcie0, double b_host0) {
    if (!est) return fail(MOE_EINVAL, "null estimate");
    if (!(alpha > 0.0 && alpha <= 1.0) || !(b_pcie0 >= 0.0) || !(b_host0 >= 0.0) || !std::isfinite(b_pcie0) ||
        !std::isfinite(b_host0))
        return fail(MOE_EINVAL, "bandwidth estimate: alpha in (0, 1], initial bandwidths finite and >= 0");
    est->alpha = alpha;
    est->b_pcie = b_pcie0;
    est->b_host = b_host0;
    est->n_pcie = 0;
    est->n_host = 0;
    return MOE_OK;
}

extern "C" int moe_bw_observe(moe_bw_estimate* est, int which, double bytes, double seconds) {
    if (!est) return fail(MOE_EINVAL, "null estimate");
    if ((which != MOE_BW_PCIE && which != MOE_BW_HOST) || !(bytes > 0.0) || !(seconds > 0.0) ||
        !std::isfinite(bytes) || !std::isfinite(seconds))
        return fail(MOE_EINVAL, "bandwidth observation: link MOE_BW_PCIE/MOE_BW_HOST, bytes and seconds > 0");
    const double obs = bytes / seconds / 1e9;
    double& b = which == MOE_BW_PCIE ? est->b_pcie : est->b_host;
    long long& n = which == MOE_BW_PCIE ? est->n_pcie : est->n_host;
    b = b > 0.0 ? (1.0 - est->alpha) * b + est->alpha * obs : obs;
    n += 1;
    return MOE_OK;
}

extern "C" int moe_bw_qstar(const moe_bw_estimate* est, int m, int* q_gpu, int* q_cpu, double* ratio) {
    if (!est) return fail(MOE_EINVAL, "null estimate");
    if (!(est->b_pcie > 0.0) || !(est->b_host > 0.0)) return fail(MOE_ESTATE, "a bandwidth is not yet known");
    return qstar_split(m, est->b_pcie, est->b_host, q_gpu, q_cpu, ratio);
}

extern "C" int qstar_split(int m, double b_pcie, double b_host, int* q_gpu, int* q_cpu, double* ratio) {
    if (!q_gpu || !q_cpu || !ratio) return fail(MOE_EINVAL, "null output");
    if (m < 0 || !(b_pcie > 0.0) || !(b_host > 0.0) || !std::isfinite(b_pcie) || !std::isfinite(b_host))
        return fail(MOE_EINVAL, "q* needs m >= 0 and positive finite bandwidths");
    const double r = b_pcie / b_host;
    double q = std::floor(double(m) * r + 0.5);
    if (q > m) q = m;
    *q_gpu = int(q);
    *q_cpu = m - int(q);
    *ratio = r;
    return MOE_OK;
}
