// router.cu -- router logits, top-k and routing weights (sm_100a).
//
// MoE-latency article, section "dense 和 MoE 的差别": the router reads each token's
// hidden state, scores every expert, keeps the top k and gives k routing weights.
//
//   logit[t,e] = sum_h x[t,h] * W_gate[h,e] (+ bias[e])        fp32 accumulation
//   picks      = k largest logits; equal values -> lower expert index first
//   w_j        = exp(l_j - l_0) / sum_i exp(l_i - l_0)          (softmax over all E
//                renormalised over the picks equals the softmax of the picked logits)
//
// One warp per token.  The logits are a skinny fp32 product (E <= 256 columns),
// too small and too precision-sensitive to be worth the tensor cores here; lanes
// split H, each lane accumulates kEC experts at a time, and a butterfly reduction
// gives every lane the sums.  The top-k then runs on the warp with one expert
// slice per lane and a shuffle arg-max per pick.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;     // tokens per block
constexpr int kEC = 8;        // experts accumulated per pass
constexpr int kMaxE = 256;

__global__ void __launch_bounds__(kWarps * 32)
    router_kernel(const uint16_t *__restrict__ x, const float *__restrict__ W_gate,
                  const float *__restrict__ bias, int64_t N, int H, int E, int k,
                  float *__restrict__ logits, int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    __shared__ float s_logit[kWarps][kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
    if (t >= N) return;  // whole warp leaves together; no block-wide barrier below
    const uint16_t *xr = x + t * H;

    // ---- logits: lanes stride H by 8 elements (one 16-byte load of x per step)
    for (int e0 = 0; e0 < E; e0 += kEC) {
        const int ne = min(kEC, E - e0);
        float acc[kEC];
#pragma unroll
        for (int j = 0; j < kEC; ++j) acc[j] = 0.f;
        for (int h0 = lane * 8; h0 < H; h0 += 32 * 8) {
            const uint4 xv = *reinterpret_cast<const uint4 *>(xr + h0);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const float2 xf = unpack_bf16x2(xw[p]);
                const float *w0 = W_gate + (int64_t)(h0 + 2 * p) * E + e0;
                const float *w1 = w0 + E;
#pragma unroll
                for (int j = 0; j < kEC; ++j) {
                    if (j < ne) {
                        acc[j] = fmaf(xf.x, __ldg(w0 + j), acc[j]);
                        acc[j] = fmaf(xf.y, __ldg(w1 + j), acc[j]);
                    }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kEC; ++j) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
        }
        if (lane < ne) {
            float v = acc[0];
#pragma unroll
            for (int j = 1; j < kEC; ++j)
                if (lane == j) v = acc[j];
            if (bias) v += bias[e0 + lane];
            s_logit[warp][e0 + lane] = v;
            if (logits) logits[t * E + e0 + lane] = v;
        }
    }
    __syncwarp();

    // ---- top-k: lane holds experts lane, lane+32, ...
    constexpr int kPer = kMaxE / 32;
    float v[kPer];
    bool taken[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
        const int e = lane + 32 * m;
        v[m] = e < E ? s_logit[warp][e] : 0.f;
        taken[m] = e >= E;
    }
    float picked[8];
    int picked_idx[8];
    for (int j = 0; j < k; ++j) {
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
        // a NaN-only remainder leaves bi unset: fall back to the lowest free index
        if (bi == 0x7fffffff) {
            int lo = 0x7fffffff;
#pragma unroll
            for (int m = 0; m < kPer; ++m)
                if (!taken[m]) lo = min(lo, lane + 32 * m);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            bi = lo;
            bv = s_logit[warp][bi];
        }
#pragma unroll
        for (int m = 0; m < kPer; ++m)
            if (lane + 32 * m == bi) taken[m] = true;
        picked[j] = bv;
        picked_idx[j] = bi;
    }
    if (lane == 0) {
        const float l0 = picked[0];
        float ex[8];
        float den = 0.f;
        for (int j = 0; j < k; ++j) { ex[j] = expf(picked[j] - l0); den += ex[j]; }
        for (int j = 0; j < k; ++j) {
            topk_idx[t * k + j] = picked_idx[j];
            topk_w[t * k + j] = ex[j] / den;
        }
    }
}

}  // namespace

cudaError_t launch_router(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H,
                          int E, int k, float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    const int64_t blocks = (N + kWarps - 1) / kWarps;
    router_kernel<<<(unsigned)blocks, kWarps * 32, 0, s>>>(x, W_gate, bias, N, H, E, k, logits, topk_idx,
                                                           topk_w);
    return cudaGetLastError();
}

}  // namespace moe
