// Top-k selection and routing weights of one token by one warp, shared by the
// router kernel and the decode FFN's fused router, so both give the same bits:
// the k largest logits in descending order (ties to the lower expert index),
// then softmax over the chosen (renorm != 0) or the full softmax read at the
// chosen experts (renorm == 0).  s_l: the token's E logits and s_taken: E bytes
// of scratch, both in shared memory.
#pragma once

#include <math.h>

namespace moe {

__device__ __forceinline__ void router_topk_warp(const float* s_l, unsigned char* s_taken, int E, int k,
                                                 int renorm, int lane, int32_t* idx_out, float* w_out) {
    for (int e = lane; e < E; e += 32) s_taken[e] = 0;
    __syncwarp();
    float my_l = 0.0f;
    int my_e = -1;
    for (int j = 0; j < k; j++) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const float v = s_l[e];
            if (!s_taken[e] && (v > bv || (v == bv && e < be) || be == 0x7fffffff)) {
                bv = v;
                be = e;
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oe = __shfl_xor_sync(0xffffffffu, be, off);
            if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
            }
        }
        if (lane == 0) s_taken[be] = 1;
        if (lane == j) {
            my_l = bv;
            my_e = be;
        }
        __syncwarp();
    }
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    float den = 0.0f;
    if (renorm) {
        den = lane < k ? expf(my_l - lmax) : 0.0f;
    } else {
        for (int e = lane; e < E; e += 32) den += expf(s_l[e] - lmax);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (lane < k) {
        idx_out[lane] = my_e;
        w_out[lane] = expf(my_l - lmax) / den;
    }
    __syncwarp();
}

}  // namespace moe
