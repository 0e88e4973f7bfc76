// decode_gemv.cu -- the expert FFN of a decode batch on CUDA cores (sm_100a).
//
// MoE-latency article, section "router 之后还有一串动作" (decode: launches, weight reads
// and token-row moves are what cost) and the section "核心公式" (the three matrices of
// one SwiGLU expert): with a few tokens, every expert GEMM is a GEMV that streams the
// picked experts' weights from HBM once.  The tensor-core grouped GEMM tiles such a layer
// by 64 weight rows per CTA -- 96 tiles of W1/W3 for 148 SMs at one token with top-8 of
// 128 experts -- and pays its pipeline's setup per launch, after a dispatch kernel.  Here
// the weight rows are dealt evenly over every SM, per pick, with no dispatch at all:
//
//   * w13: every block first ranks the batch itself from the router's partial logits
//     (the top-k of topk_warp), then for each pick a = t*k + j (expert e) and
//     intermediate feature i:  h[a][i] = bf16( silu(W1[e][i] . x[t]) * (W3[e][i] . x[t]) ).
//   * w2 + combine: for every output feature f and token t, in pick order j,
//       acc = fmaf(w[t,j], W2[e_j][f] . h[t*k + j], acc)
//     then acc += shared[t][f] and out[t][f] = bf16(acc) -- the combine's fma chain,
//     over y values that never leave registers, so the fp32 expert outputs make no
//     round trip through memory and the combine needs no launch of its own.
//
// Two tokens that pick the same expert read its rows twice (the second time mostly from
// L2); at the batch sizes this path takes that is rare.  Every dot product sums a lane's
// 8-element chunks in order, then the lanes by a fixed xor-shuffle tree: the bits do not
// depend on timing.  They differ from the tensor-core path's (another summation order),
// within the same fp32 accuracy.
#include "common.cuh"
#include "internal.h"
#include "topk_warp.cuh"

namespace moe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxE = 256;
constexpr int kBatch = 8;  // 16-byte chunks of each weight row a lane loads before it multiplies

__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8])
{
    const float2 a = unpack_bf16x2(v.x), b = unpack_bf16x2(v.y), c = unpack_bf16x2(v.z), d = unpack_bf16x2(v.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// A weight chunk read once: not kept in L1, where the token rows it meets stay.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// This block's share [lo, hi) of `units` equal units of work.
__device__ __forceinline__ void block_range(int64_t units, int64_t &lo, int64_t &hi)
{
    lo = units * blockIdx.x / gridDim.x;
    hi = units * (blockIdx.x + 1) / gridDim.x;
}

// The picks a block needs are in shared memory before its first weight load, so each
// unit of work waits for one load from HBM (its weight rows), not for a chain of
// dependent loads.
constexpr int kMaxR = MOE_DECODE_MAX_ROWS;
constexpr int kMaxK = 8;

// W1/W3 over units u = (pick a = u / I, feature i = u % I): the rows W1[e_a][i] and
// W3[e_a][i] against x[a / k], h[a][i] = bf16(silu(g) * u).  With P > 0 every block
// first ranks the batch itself from the router's P partial logits (summed in slice
// order, + bias) with topk_warp -- the picks and weights of the router's own top-k --
// and block 0 writes them (and the logits, when asked); with P == 0 the picks are read.
template <int P>
__global__ void __launch_bounds__(kThreads, 1)
    decode_w13_kernel(const uint16_t *__restrict__ x, const float *__restrict__ part, int64_t pstride,
                      const float *__restrict__ bias, float *__restrict__ logits, int32_t *__restrict__ topk_idx,
                      float *__restrict__ topk_w, int64_t N, int k, int E, int H, int I,
                      const uint16_t *__restrict__ W1, const uint16_t *__restrict__ W3, uint16_t *__restrict__ h,
                      int *err)
{
    __shared__ int32_t s_idx[kMaxR];
    __shared__ float s_w[kMaxR];
    __shared__ float s_row[P > 0 ? kWarps : 1][P > 0 ? kMaxE : 1];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t R = N * k;
    const bool lead = blockIdx.x == 0;
    const int nch = H / 8;  // 16-byte chunks of a row
    if (P > 0) {
        for (int64_t t = warp; t < N; t += kWarps) {
            for (int e = lane; e < E; e += 32) {
                const float *p = part + t * E + e;
                float v = p[0];
#pragma unroll
                for (int i = 1; i < P; ++i) v += p[i * pstride];
                if (bias) v += bias[e];
                if (logits && lead) logits[t * E + e] = v;
                s_row[warp][e] = v;
            }
            __syncwarp();
            topk_warp(s_row[warp], E, k, lane, s_idx + t * k, s_w + t * k);
            __syncwarp();
        }
        __syncthreads();
        if (lead)
            for (int64_t a = threadIdx.x; a < R; a += kThreads) {
                topk_idx[a] = s_idx[a];
                topk_w[a] = s_w[a];
            }
    } else {
        for (int64_t a = threadIdx.x; a < R; a += kThreads) s_idx[a] = topk_idx[a];
        __syncthreads();
    }
    int64_t lo, hi;
    block_range(R * I, lo, hi);
    for (int64_t u = lo + warp; u < hi; u += kWarps) {
        const int64_t a = u / I;
        const int i = (int)(u % I);
        const int e = s_idx[a];
        if (e < 0 || e >= E) {  // (reported by the W2 kernel, which skips the pick)
            if (lane == 0) h[a * I + i] = 0;
            continue;
        }
        const uint4 *w1 = reinterpret_cast<const uint4 *>(W1 + ((int64_t)e * I + i) * H);
        const uint4 *w3 = reinterpret_cast<const uint4 *>(W3 + ((int64_t)e * I + i) * H);
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + (a / k) * H);
        float ga = 0.f, ua = 0.f;
        // batches of kBatch chunks a lane: every load of a batch is issued before the
        // first multiply waits for one
        for (int c0 = lane; c0 < nch; c0 += 32 * kBatch) {
            uint4 wa[kBatch], wb[kBatch], xq[kBatch];
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                const int c = c0 + 32 * q;
                wa[q] = c < nch ? ld_stream(w1 + c) : make_uint4(0, 0, 0, 0);
                wb[q] = c < nch ? ld_stream(w3 + c) : make_uint4(0, 0, 0, 0);
                xq[q] = c < nch ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int q = 0; q < kBatch; ++q) {
                float fa[8], fb[8], xv[8];
                unpack8(wa[q], fa);
                unpack8(wb[q], fb);
                unpack8(xq[q], xv);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ga = fmaf(fa[j], xv[j], ga);
                    ua = fmaf(fb[j], xv[j], ua);
                }
            }
        }
        const float gs = warp_sum(ga), us = warp_sum(ua);
        if (lane == 0) h[a * I + i] = float_to_bf16_bits(silu(gs) * us);
    }
}

// W2 with the combine, units u = (feature f = u / N, token t = u % N): the token's k
// weight rows W2[e_j][f] (I each) against its k rows of h (rows t*k + j), added in pick
// order.
__global__ void __launch_bounds__(kThreads, 1)
    decode_w2_combine_kernel(const uint16_t *__restrict__ h, const int32_t *__restrict__ topk_idx,
                             const float *__restrict__ topk_w, const float *__restrict__ shared_out, int64_t N,
                             int E, int H, int I, int k, const uint16_t *__restrict__ W2, uint16_t *__restrict__ out,
                             int *err)
{
    __shared__ int s_e[kMaxR];  // expert of each pick, -1 when out of range
    __shared__ float s_w[kMaxR];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t R = N * k;
    for (int64_t a = threadIdx.x; a < R; a += kThreads) {
        const int e = topk_idx[a];
        const bool ok = e >= 0 && e < E;
        if (!ok) set_device_error(err, MOE_DEVERR_BAD_EXPERT_INDEX);
        s_e[a] = ok ? e : -1;
        s_w[a] = topk_w[a];
    }
    __syncthreads();
    int64_t lo, hi;
    block_range((int64_t)H * N, lo, hi);
    const int nch = I / 8;
    for (int64_t u = lo + warp; u < hi; u += kWarps) {
        const int f = (int)(u / N);
        const int64_t t = u % N;
        const uint4 *wr[kMaxK];
        const uint4 *hr[kMaxK];
        float wt[kMaxK];
        bool on[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            const int e = j < k ? s_e[t * k + j] : -1;
            on[j] = e >= 0;
            wt[j] = j < k ? s_w[t * k + j] : 0.f;
            wr[j] = reinterpret_cast<const uint4 *>(W2 + ((int64_t)(on[j] ? e : 0) * H + f) * I);
            hr[j] = reinterpret_cast<const uint4 *>(h + (t * k + (j < k ? j : 0)) * I);
        }
        float y[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) y[j] = 0.f;
        // one chunk of every pick's two rows a round: all sixteen loads in flight at once
        for (int c = lane; c < nch; c += 32) {
            uint4 wv[kMaxK], hv[kMaxK];
#pragma unroll
            for (int j = 0; j < kMaxK; ++j) {
                wv[j] = on[j] ? ld_stream(wr[j] + c) : make_uint4(0, 0, 0, 0);
                hv[j] = on[j] ? __ldg(hr[j] + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < kMaxK; ++j) {
                float fa[8], fb[8];
                unpack8(wv[j], fa);
                unpack8(hv[j], fb);
#pragma unroll
                for (int q = 0; q < 8; ++q) y[j] = fmaf(fa[q], fb[q], y[j]);
            }
        }
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            const float yj = warp_sum(y[j]);
            if (on[j]) acc = fmaf(wt[j], yj, acc);
        }
        if (lane == 0) {
            if (shared_out) acc += shared_out[t * H + f];
            out[t * H + f] = float_to_bf16_bits(acc);
        }
    }
}

}  // namespace

cudaError_t launch_decode_w13(const uint16_t *x, const RouterPartials &rp, int32_t *topk_idx, float *topk_w,
                              int64_t N, int k, int E, int H, int I, const uint16_t *W1, const uint16_t *W3,
                              uint16_t *h, int *err, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    if (E < 1 || E > kMaxE || k < 1 || k > kMaxK || H % 8 || I < 1 || N * (int64_t)k > kMaxR)
        return cudaErrorInvalidValue;
    const dim3 grid((unsigned)device_sm_count());
    switch (rp.P) {
        case 0: return launch_pdl(decode_w13_kernel<0>, grid, dim3(kThreads), 0, s, x, rp.part, rp.pstride, rp.bias,
                                  rp.logits, topk_idx, topk_w, N, k, E, H, I, W1, W3, h, err);
        case 1: return launch_pdl(decode_w13_kernel<1>, grid, dim3(kThreads), 0, s, x, rp.part, rp.pstride, rp.bias,
                                  rp.logits, topk_idx, topk_w, N, k, E, H, I, W1, W3, h, err);
        case 2: return launch_pdl(decode_w13_kernel<2>, grid, dim3(kThreads), 0, s, x, rp.part, rp.pstride, rp.bias,
                                  rp.logits, topk_idx, topk_w, N, k, E, H, I, W1, W3, h, err);
        case 4: return launch_pdl(decode_w13_kernel<4>, grid, dim3(kThreads), 0, s, x, rp.part, rp.pstride, rp.bias,
                                  rp.logits, topk_idx, topk_w, N, k, E, H, I, W1, W3, h, err);
        case 8: return launch_pdl(decode_w13_kernel<8>, grid, dim3(kThreads), 0, s, x, rp.part, rp.pstride, rp.bias,
                                  rp.logits, topk_idx, topk_w, N, k, E, H, I, W1, W3, h, err);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode_w2_combine(const uint16_t *h, const int32_t *topk_idx, const float *topk_w,
                                     const float *shared_out, int64_t N, int E, int H, int I, int k,
                                     const uint16_t *W2, uint16_t *out, int *err, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    if (k < 1 || k > kMaxK || I % 8 || H < 1 || N * (int64_t)k > kMaxR) return cudaErrorInvalidValue;
    return launch_pdl(decode_w2_combine_kernel, dim3((unsigned)device_sm_count()), dim3(kThreads), 0, s, h, topk_idx,
                      topk_w, shared_out, N, E, H, I, k, W2, out, err);
}

}  // namespace moe
