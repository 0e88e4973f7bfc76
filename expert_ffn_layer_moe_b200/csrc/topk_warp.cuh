// topk_warp.cuh -- top-k and routing weights of one token on one warp.
//
// MoE-latency article, section "dense 和 MoE 的差别": keep the k best-scoring experts
// and give k routing weights.  Picks in descending logit order, an equal value going to
// the lower expert index; w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0) (the softmax over
// all experts renormalised over the picks equals the softmax of the picked logits).
#pragma once

#include <cmath>

#include "common.cuh"

namespace moe {

constexpr int kTopkMaxE = 256;
constexpr int kTopkMaxK = 8;

// Top-k of one token's E logits (in `row`) on one warp; lane 0 writes the picks
// and their weights.
__device__ __forceinline__ void topk_warp(const float *row, int E, int k, int lane, int32_t *__restrict__ idx_out,
                                          float *__restrict__ w_out)
{
    constexpr int kPer = kTopkMaxE / 32;
    float v[kPer];
    bool taken[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
        const int e = lane + 32 * m;
        v[m] = e < E ? row[e] : 0.f;
        taken[m] = e >= E;
    }
    float pv[kTopkMaxK];
    int pi[kTopkMaxK];
#pragma unroll
    for (int j = 0; j < kTopkMaxK; ++j) {
        if (j >= k) break;
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int e = lane + 32 * m;
            if (!taken[m] && (v[m] > bv || (v[m] == bv && e < bi))) { bv = v[m]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (bi == 0x7fffffff) {  // only NaN left: take the lowest free index
            int lo = 0x7fffffff;
#pragma unroll
            for (int m = 0; m < kPer; ++m)
                if (!taken[m]) lo = min(lo, lane + 32 * m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            bi = lo;
            bv = row[bi];
        }
#pragma unroll
        for (int m = 0; m < kPer; ++m)
            if (lane + 32 * m == bi) taken[m] = true;
        pv[j] = bv;
        pi[j] = bi;
    }
    if (lane == 0) {
        const float l0 = pv[0];
        float ex[kTopkMaxK];
        float den = 0.f;
#pragma unroll
        for (int j = 0; j < kTopkMaxK; ++j)
            if (j < k) { ex[j] = expf(pv[j] - l0); den += ex[j]; }
#pragma unroll
        for (int j = 0; j < kTopkMaxK; ++j)
            if (j < k) { idx_out[j] = pi[j]; w_out[j] = ex[j] / den; }
    }
}


}  // namespace moe
