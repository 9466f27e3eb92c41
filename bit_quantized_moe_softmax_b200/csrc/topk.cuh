// topk.cuh -- top-k selection and softmax of one token's router logits by one
// warp: order = logit descending, then expert index ascending; weights =
// softmax over the selected logits.
#pragma once

#include "ds4moe_internal.cuh"

namespace ds4 {

// Order-preserving map binary32 -> uint32 (larger logit, larger key).
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k and softmax of one token's logits by one warp.  Each lane keeps the
// best of its own candidates (experts lane, lane + 32, ...); a round picks the
// warp maximum with two warp reductions (largest key, then the lowest expert
// index among equal keys) and the winning lane advances to its next best.
// `buf` is E floats of shared memory.
static __device__ void topk_softmax_warp(const float* logits_g, float* buf, int E, int k, int32_t* ids, float* wts) {
    const int lane = threadIdx.x & 31;
    for (int e = lane; e < E; e += 32) buf[e] = __ldcg(logits_g + e);
    __syncwarp();
    uint32_t taken = 0;   // bit m: candidate lane + 32 m already chosen (E <= 1024)
    auto local_best = [&](uint32_t& key, int& idx) {
        key = 0;
        idx = 0x7fffffff;
        for (int m = 0; lane + 32 * m < E; ++m) {
            if (taken & (1u << m)) continue;
            const uint32_t kk = order_key(buf[lane + 32 * m]);
            if (kk > key) { key = kk; idx = lane + 32 * m; }   // ascending index: strict > keeps the lowest
        }
    };
    uint32_t key;
    int idx;
    local_best(key, idx);
    float my_l = 0.f;
    int my_id = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        const int win = (int)__reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)idx : 0xffffffffu);
        if (lane == j) { my_l = buf[win]; my_id = win; }
        if ((win & 31) == lane) {
            taken |= 1u << (win >> 5);
            local_best(key, idx);
        }
    }
    const float lmax = __shfl_sync(0xffffffffu, my_l, 0);
    const float ex = lane < k ? __expf(my_l - lmax) : 0.f;
    float den = ex;
    for (int off = 16; off >= 1; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    if (lane < k) {
        ids[lane] = my_id;
        wts[lane] = ex / den;
    }
}

}  // namespace ds4
