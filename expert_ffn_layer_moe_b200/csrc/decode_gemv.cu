// decode_gemv.cu -- the expert FFN of a decode batch on CUDA cores (sm_100a).
//
// MoE-latency article, section "router 之后还有一串动作" (decode: launches, weight reads
// and token-row moves are what cost) and the section "核心公式" (the three matrices of
// one SwiGLU expert): with a token or two per expert, every expert GEMM is a GEMV that
// streams the expert's weights from HBM once.  The tensor-core grouped GEMM tiles such a
// layer by 64 weight rows per CTA -- 96 tiles of W1/W3 for 148 SMs at one token with
// top-8 of 128 experts -- and pays its pipeline's setup per launch.  Here the weight rows
// are dealt evenly over every SM and read with plain 16-byte loads:
//
//   * w13: for every touched expert g and intermediate feature i, the rows W1[g][i] and
//     W3[g][i] against each of the group's token rows x[row_to_token[r]] (no permuted
//     copy of x):  h[r][i] = bf16( silu(W1[g][i] . x) * (W3[g][i] . x) ).
//   * w2 + combine: for every output feature f and token t, in pick order j,
//       acc = fmaf(w[t,j], W2[e_j][f] . h[token_to_row[t,j]], acc)
//     then acc += shared[t][f] and out[t][f] = bf16(acc) -- the combine's fma chain,
//     over y values that never leave registers, so the fp32 expert outputs make no
//     round trip through memory and the combine needs no launch of its own.
//
// Every dot product sums a lane's 8-element chunks in order, then the lanes by a fixed
// xor-shuffle tree: the bits do not depend on timing.  They differ from the tensor-core
// path's (another summation order), within the same fp32 accuracy.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = 32 * kWarps;
constexpr int kMaxE = 256;
constexpr int kTok = 4;    // token rows a warp multiplies against one weight row at a time
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

// The row maps and offsets a block needs are staged in shared memory first, so each
// unit of work waits for one load from HBM (its weight rows), not for a chain of
// dependent loads.
constexpr int kMaxR = MOE_DECODE_MAX_ROWS;

// Unit u = (touched group u / I, feature u % I): two weight rows of H against the
// group's token rows, kTok at a time.
__global__ void __launch_bounds__(kThreads, 1)
    decode_w13_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ offsets,
                      const int32_t *__restrict__ row_to_token, int64_t N, int64_t R, int E, int H, int I,
                      const uint16_t *__restrict__ W1, const uint16_t *__restrict__ W3, uint16_t *__restrict__ h,
                      int *err)
{
    __shared__ int s_off[kMaxE + 1];
    __shared__ int s_r2t[kMaxR];
    __shared__ int touched[kMaxE];
    __shared__ int ntouched;
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int g = threadIdx.x; g <= E; g += kThreads) {
        int o = offsets[g];
        if (o < 0 || o > R) {
            set_device_error(err, MOE_DEVERR_BAD_OFFSETS);
            o = o < 0 ? 0 : (int)R;
        }
        s_off[g] = o;
    }
    for (int r = threadIdx.x; r < R; r += kThreads) {
        int t = row_to_token[r];
        if (t < 0 || t >= N) {
            set_device_error(err, MOE_DEVERR_BAD_OFFSETS);
            t = 0;
        }
        s_r2t[r] = t;
    }
    __syncthreads();
    if (warp == 0) {
        // the non-empty groups in index order
        int count = 0;
        for (int base = 0; base < E; base += 32) {
            const int g = base + lane;
            const bool busy = g < E && s_off[g + 1] > s_off[g];
            const unsigned m = __ballot_sync(0xffffffffu, busy);
            if (busy) touched[count + __popc(m & ((1u << lane) - 1u))] = g;
            count += __popc(m);
        }
        if (lane == 0) ntouched = count;
    }
    __syncthreads();
    int64_t lo, hi;
    block_range((int64_t)ntouched * I, lo, hi);
    const int nch = H / 8;  // 16-byte chunks of a row
    for (int64_t u = lo + warp; u < hi; u += kWarps) {
        const int g = touched[u / I];
        const int i = (int)(u % I);
        const int r0 = s_off[g], r1 = s_off[g + 1];
        const uint4 *w1 = reinterpret_cast<const uint4 *>(W1 + ((int64_t)g * I + i) * H);
        const uint4 *w3 = reinterpret_cast<const uint4 *>(W3 + ((int64_t)g * I + i) * H);
        for (int r = r0; r < r1; r += kTok) {
            const int nt = min(kTok, r1 - r);
            const uint4 *xr[kTok];
#pragma unroll
            for (int q = 0; q < kTok; ++q) xr[q] = reinterpret_cast<const uint4 *>(x + (int64_t)s_r2t[q < nt ? r + q : r] * H);
            float ga[kTok], ua[kTok];
#pragma unroll
            for (int q = 0; q < kTok; ++q) ga[q] = ua[q] = 0.f;
            // batches of kBatch chunks a lane: every weight load of a batch is issued before
            // the first multiply waits for one
            for (int c0 = lane; c0 < nch; c0 += 32 * kBatch) {
                uint4 wa[kBatch], wb[kBatch];
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    const int c = c0 + 32 * q;
                    wa[q] = c < nch ? ld_stream(w1 + c) : make_uint4(0, 0, 0, 0);
                    wb[q] = c < nch ? ld_stream(w3 + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int tq = 0; tq < kTok; ++tq) {
                    if (tq < nt) {
                        uint4 xq[kBatch];
#pragma unroll
                        for (int q = 0; q < kBatch; ++q) {
                            const int c = c0 + 32 * q;
                            xq[q] = c < nch ? __ldg(xr[tq] + c) : make_uint4(0, 0, 0, 0);
                        }
#pragma unroll
                        for (int q = 0; q < kBatch; ++q) {
                            float a[8], b[8], xv[8];
                            unpack8(wa[q], a);
                            unpack8(wb[q], b);
                            unpack8(xq[q], xv);
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                ga[tq] = fmaf(a[e], xv[e], ga[tq]);
                                ua[tq] = fmaf(b[e], xv[e], ua[tq]);
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < kTok; ++q) {
                const float gs = warp_sum(ga[q]), us = warp_sum(ua[q]);
                if (lane == 0 && q < nt) h[(int64_t)(r + q) * I + i] = float_to_bf16_bits(silu(gs) * us);
            }
        }
    }
}

// Unit u = (feature u / N, token u % N): the token's k weight rows of W2 (I each)
// against its k rows of h, added in pick order.
constexpr int kMaxK = 8;
__global__ void __launch_bounds__(kThreads, 1)
    decode_w2_combine_kernel(const uint16_t *__restrict__ h, const int32_t *__restrict__ topk_idx,
                             const int32_t *__restrict__ token_to_row, const float *__restrict__ topk_w,
                             const float *__restrict__ shared_out, int64_t N, int64_t R, int E, int H, int I, int k,
                             const uint16_t *__restrict__ W2, uint16_t *__restrict__ out, int *err)
{
    __shared__ int s_e[kMaxR];    // expert of each pick, -1 when it or its row is out of range
    __shared__ int s_row[kMaxR];  // its row of h
    __shared__ float s_w[kMaxR];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int a = threadIdx.x; a < R; a += kThreads) {
        const int e = topk_idx[a], row = token_to_row[a];
        const bool ok = e >= 0 && e < E && row >= 0 && row < R;
        if (!ok) set_device_error(err, MOE_DEVERR_BAD_EXPERT_INDEX);
        s_e[a] = ok ? e : -1;
        s_row[a] = ok ? row : 0;
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
            hr[j] = reinterpret_cast<const uint4 *>(h + (int64_t)(j < k ? s_row[t * k + j] : 0) * I);
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
                float a[8], b[8];
                unpack8(wv[j], a);
                unpack8(hv[j], b);
#pragma unroll
                for (int e = 0; e < 8; ++e) y[j] = fmaf(a[e], b[e], y[j]);
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

cudaError_t launch_decode_w13(const uint16_t *x, const int32_t *offsets, const int32_t *row_to_token, int64_t N,
                              int k, int E, int H, int I, const uint16_t *W1, const uint16_t *W3, uint16_t *h,
                              int *err, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    if (E < 1 || E > kMaxE || H % 8 || I < 1 || N * (int64_t)k > kMaxR) return cudaErrorInvalidValue;
    return launch_pdl(decode_w13_kernel, dim3((unsigned)device_sm_count()), dim3(kThreads), 0, s, x, offsets,
                      row_to_token, N, N * (int64_t)k, E, H, I, W1, W3, h, err);
}

cudaError_t launch_decode_w2_combine(const uint16_t *h, const int32_t *topk_idx, const int32_t *token_to_row,
                                     const float *topk_w, const float *shared_out, int64_t N, int E, int H, int I,
                                     int k, const uint16_t *W2, uint16_t *out, int *err, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    if (k < 1 || k > kMaxK || I % 8 || H < 1 || N * (int64_t)k > kMaxR) return cudaErrorInvalidValue;
    return launch_pdl(decode_w2_combine_kernel, dim3((unsigned)device_sm_count()), dim3(kThreads), 0, s, h, topk_idx,
                      token_to_row, topk_w, shared_out, N, N * (int64_t)k, E, H, I, k, W2, out, err);
}

}  // namespace moe
