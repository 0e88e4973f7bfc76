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
// One block per tile of TT tokens, 8 warps splitting H: warp w takes the 64-wide
// column chunks w, w+8, ... and each lane two adjacent columns, so a warp reads
// 128 contiguous bytes of x per token and 64 consecutive W_gate rows per step.  A
// lane accumulates TT tokens x 8 experts at a time; lanes then reduce with a
// butterfly and warps in a fixed order through shared memory (deterministic bits).
// TT shrinks for small batches so the grid still covers the SMs.  The top-k runs
// on one warp per token with an expert slice per lane and a shuffle arg-max per pick.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kEC = 8;      // experts accumulated per pass
constexpr int kChunk = 64;  // columns of H per warp step (2 per lane)
constexpr int kMaxE = 256;
constexpr int kMaxK = 8;

template <int TT>
__global__ void __launch_bounds__(kThreads)
    router_kernel(const uint16_t *__restrict__ x, const float *__restrict__ W_gate,
                  const float *__restrict__ bias, int64_t N, int H, int E, int k,
                  float *__restrict__ logits, int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    extern __shared__ float smem[];
    float *partial = smem;                        // [kWarps][TT][E]
    float *s_logit = smem + kWarps * TT * E;      // [TT][E]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * TT;
    const int nt = (N - t0) < TT ? (int)(N - t0) : TT;

    for (int e0 = 0; e0 < E; e0 += kEC) {
        const int ne = min(kEC, E - e0);
        float acc[TT][kEC];
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int j = 0; j < kEC; ++j) acc[t][j] = 0.f;
        // full 8-expert slices of rows whose start is 16-byte aligned load as float4
        const bool vec = ne == kEC && (E & 3) == 0;
#pragma unroll 4
        for (int c = warp * kChunk; c < H; c += kWarps * kChunk) {
            const int h = c + 2 * lane;
            float2 xv[TT];
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const uint32_t v = t < nt ? __ldg(reinterpret_cast<const uint32_t *>(x + (t0 + t) * H + h)) : 0u;
                xv[t] = unpack_bf16x2(v);
            }
            const float *w0 = W_gate + (int64_t)h * E + e0;
            const float *w1 = w0 + E;
            float a[kEC], b[kEC];
            if (vec) {
                const float4 a0 = __ldg(reinterpret_cast<const float4 *>(w0));
                const float4 a1 = __ldg(reinterpret_cast<const float4 *>(w0) + 1);
                const float4 b0 = __ldg(reinterpret_cast<const float4 *>(w1));
                const float4 b1 = __ldg(reinterpret_cast<const float4 *>(w1) + 1);
                a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w; a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
                b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w; b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
            } else {
#pragma unroll
                for (int j = 0; j < kEC; ++j) {
                    a[j] = j < ne ? __ldg(w0 + j) : 0.f;
                    b[j] = j < ne ? __ldg(w1 + j) : 0.f;
                }
            }
#pragma unroll
            for (int j = 0; j < kEC; ++j)
#pragma unroll
                for (int t = 0; t < TT; ++t) acc[t][j] = fmaf(xv[t].y, b[j], fmaf(xv[t].x, a[j], acc[t][j]));
        }
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int j = 0; j < kEC; ++j)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc[t][j] += __shfl_xor_sync(0xffffffffu, acc[t][j], o);
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < TT; ++t)
#pragma unroll
                for (int j = 0; j < kEC; ++j)
                    if (j < ne) partial[(warp * TT + t) * E + e0 + j] = acc[t][j];
        }
    }
    __syncthreads();

    // fixed-order sum over warps, bias, write logits
    for (int i = threadIdx.x; i < nt * E; i += kThreads) {
        const int t = i / E, e = i % E;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += partial[(w * TT + t) * E + e];
        if (bias) v += bias[e];
        s_logit[t * E + e] = v;
        if (logits) logits[(t0 + t) * E + e] = v;
    }
    __syncthreads();

    // top-k: warp t handles token t; lane holds experts lane, lane+32, ...
    for (int t = warp; t < nt; t += kWarps) {
        constexpr int kPer = kMaxE / 32;
        float v[kPer];
        bool taken[kPer];
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int e = lane + 32 * m;
            v[m] = e < E ? s_logit[t * E + e] : 0.f;
            taken[m] = e >= E;
        }
        float pv[kMaxK];
        int pi[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
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
                bv = s_logit[t * E + bi];
            }
#pragma unroll
            for (int m = 0; m < kPer; ++m)
                if (lane + 32 * m == bi) taken[m] = true;
            pv[j] = bv;
            pi[j] = bi;
        }
        if (lane == 0) {
            const float l0 = pv[0];
            float ex[kMaxK];
            float den = 0.f;
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                if (j < k) { ex[j] = expf(pv[j] - l0); den += ex[j]; }
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                if (j < k) {
                    topk_idx[(t0 + t) * k + j] = pi[j];
                    topk_w[(t0 + t) * k + j] = ex[j] / den;
                }
        }
    }
}

template <int TT>
cudaError_t launch_tt(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E, int k,
                      float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    const size_t smem = sizeof(float) * (size_t)(kWarps * TT * E + TT * E);
    auto kern = router_kernel<TT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const int64_t blocks = (N + TT - 1) / TT;
    kern<<<(unsigned)blocks, kThreads, smem, s>>>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E,
                          int k, float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    // tokens per block: keep at least ~2 blocks per SM before sharing W_gate reads
    const int64_t sms = device_sm_count();
    if (N >= 8 * 2 * sms) return launch_tt<8>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
    if (N >= 4 * 2 * sms) return launch_tt<4>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
    if (N >= 2 * 2 * sms) return launch_tt<2>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
    return launch_tt<1>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
}

}  // namespace moe
