// One decode MoE layer in one host call: the per-layer sequence of the engine
// (route, slot lookup, expert FFN, miss streaming, combine) issued natively, so
// the host's share of a layer is a handful of driver calls.
//
// Order (post.smzdm.com/p/aomxznrn, "FreeToken干的事": resident experts run
// on the GPU while missing ones cross PCIe): router and lookup are enqueued,
// then the FFN, whose CTAs on resident experts start at once; only then does
// the host wait (bounded) for the lookup's miss list and put the misses on the
// copy stream.  The combine is fused into the FFN kernel.
#include "common.cuh"

using namespace moe;

extern "C" int moe_decode_layer(moe_pool* p, int layer, const void* x_bf16, int T, const void* wr_bf16,
                                const float* bias, int renormalize, int32_t* idx, float* w,
                                int32_t* slot_of, float* y_part, void* y_bf16, int* status,
                                void* route_ws, size_t route_ws_bytes, moe_lookup_result* res,
                                void* copy_start, void* copy_end, int overlap, void* stream,
                                void* copy_stream) {
    if (!p) return fail(MOE_EINVAL, "null pool");
    // with overlap the FFN waits for copies issued after it: they need their own stream
    if (overlap && (copy_stream == stream || copy_stream == nullptr))
        return fail(MOE_EINVAL, "decode layer: copy_stream must be a stream other than the compute stream");
    const moe_config& c = p->cfg;
    // the caller's result arrays, else local ones of the largest size a call needs
    int32_t uniq_l[kMaxE], hit_l[kMaxE];
    moe_miss miss_l[kMaxE];
    moe_lookup_result local{0, 0, uniq_l, hit_l, miss_l};
    moe_lookup_result* r = res ? res : &local;
    cudaStream_t cs = (cudaStream_t)copy_stream;
    auto copies = [&]() -> int {
        if (r->n_miss == 0) return MOE_OK;
        if (copy_start) MOE_CUDA_TRY(cudaEventRecord((cudaEvent_t)copy_start, cs));
        const int rc = moe_stream_misses(p, layer, r->miss_h, r->n_miss, copy_stream);
        if (rc) return rc;
        if (copy_end) MOE_CUDA_TRY(cudaEventRecord((cudaEvent_t)copy_end, cs));
        return MOE_OK;
    };
    int rc = moe_route(x_bf16, wr_bf16, bias, T, c.H, c.E, c.k, renormalize, idx, w, route_ws,
                       route_ws_bytes, stream);
    if (rc) return rc;
    if (!overlap) {
        // misses streamed before the FFN is enqueued (for tools that serialise kernels)
        if ((rc = moe_slot_lookup(p, layer, idx, T, c.k, slot_of, r, stream))) return rc;
        if ((rc = copies())) return rc;
        return moe_expert_ffn(p, layer, x_bf16, T, idx, w, slot_of, y_part, y_bf16, status, stream);
    }
    if ((rc = moe_slot_lookup_launch(p, layer, idx, T, c.k, slot_of, stream))) return rc;
    rc = moe_expert_ffn(p, layer, x_bf16, T, idx, w, slot_of, y_part, y_bf16, status, stream);
    // the launched lookup is collected whatever the FFN launch returned
    const int rc2 = moe_slot_lookup_result(p, r);
    if (rc) return rc;
    if (rc2) return rc2;
    return copies();
}

// All-resident decode of consecutive layers (post.smzdm.com/p/aomxznrn,
// "FreeToken干的事": decode is scheduled on its own, bandwidth-bound path): one
// FFN launch per layer with the router, the slot lookup (its resident form: slots
// from the key table, the hits' LRU touch by CTA 0) and the combine fused in,
// chained by programmatic stream serialisation with no host wait in between, so
// a caller may capture the whole sequence in one CUDA graph.
extern "C" int moe_decode_resident(moe_pool* p, int layer0, int n_layers, const void* x_bf16, int T,
                                   const void* const* wr_bf16, const float* const* bias, int renormalize,
                                   int32_t* idx, float* w, int32_t* slot_of, float* y_part, void* y_bf16,
                                   int* status, void* stream) {
    if (!p || !x_bf16 || !wr_bf16 || !y_bf16 || !status) return fail(MOE_EINVAL, "null argument");
    const moe_config& c = p->cfg;
    if (n_layers <= 0 || layer0 < 0 || layer0 + n_layers > c.L) return fail(MOE_EBOUNDS, "layers outside the pool");
    if (T <= 0 || T > c.max_tokens) return fail(MOE_EINVAL, "T must be in [1, max_tokens]");
    if (!slot_of || !idx || !w || !y_part) return fail(MOE_EINVAL, "null argument");
    if (renormalize != 0 && renormalize != 1) return fail(MOE_EINVAL, "renormalize must be 0 or 1");
    const size_t xl = (size_t)T * c.H * 2;
    for (int i = 0; i < n_layers; i++) {
        if (!wr_bf16[i]) return fail(MOE_EINVAL, "null router weight");
        const uint8_t* x = (const uint8_t*)x_bf16 + i * xl;
        uint8_t* y = (uint8_t*)y_bf16 + i * xl;
        const FfnRoute route{wr_bf16[i], bias ? bias[i] : nullptr, renormalize, idx, w};
        const int rc = expert_ffn(p, layer0 + i, x, T, idx, w, slot_of, y_part, y, status, stream, 1, &route);
        if (rc) return rc;
    }
    return MOE_OK;
}
