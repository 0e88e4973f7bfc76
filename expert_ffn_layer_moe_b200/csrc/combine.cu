// combine.cu -- combine / unpermutation (sm_100a).
//
// MoE-latency article, section "router 之后还有一串动作": the inverse mapping brings
// expert outputs back to token order, each is multiplied by its routing weight and
// the k results are added.  Deterministic gather-reduce (no atomics):
//
//   acc = 0;  for j in pick order: acc = fmaf(w[t,j], y_perm[token_to_row[t,j]], acc)
//   acc += shared_out[t]            (optional always-on shared experts, weight 1)
//   out[t] = bf16_rn(acc)
// The expert rows y_perm and the shared output arrive in fp32, so out is the only
// rounding after the expert GEMMs.  When the W2 GEMM split its K range, y_perm holds
// nsplit partial sums per row; they are added in slice order before the weighting.
//
// Grid = tokens x feature slices of kThreads*8 features: each thread owns 8
// consecutive features of one token (two 16-byte fp32 loads per picked row, one
// 16-byte bf16 store), so every load of a small decode batch is in flight at once.
// HBM-bound: k rows read, one row written per token.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxK = 8;

__global__ void __launch_bounds__(kThreads)
    combine_kernel(const float *__restrict__ y_perm, int nsplit, int64_t split_stride,
                   const int32_t *__restrict__ token_to_row, const float *__restrict__ topk_w,
                   const float *__restrict__ shared_out, int64_t N, int H, int k, uint16_t *__restrict__ out)
{
    pdl_entry();
    const int64_t t = blockIdx.y;
    int rows[kMaxK];
    float w[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        rows[j] = j < k ? token_to_row[t * k + j] : -1;
        w[j] = j < k ? topk_w[t * k + j] : 0.f;
    }
    const int nvec = H / 8;
    for (int v = blockIdx.x * kThreads + threadIdx.x; v < nvec; v += gridDim.x * kThreads) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (j < k && rows[j] >= 0) {
                const float4 *src = reinterpret_cast<const float4 *>(y_perm + (int64_t)rows[j] * H) + 2 * v;
                float4 lo = __ldg(src), hi = __ldg(src + 1);
                for (int p = 1; p < nsplit; ++p) {
                    const float4 *sp = reinterpret_cast<const float4 *>(y_perm + p * split_stride +
                                                                        (int64_t)rows[j] * H) + 2 * v;
                    const float4 l2 = __ldg(sp), h2 = __ldg(sp + 1);
                    lo.x += l2.x; lo.y += l2.y; lo.z += l2.z; lo.w += l2.w;
                    hi.x += h2.x; hi.y += h2.y; hi.z += h2.z; hi.w += h2.w;
                }
                const float yv[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(w[j], yv[i], acc[i]);
            }
        }
        if (shared_out) {
            const float4 *src = reinterpret_cast<const float4 *>(shared_out + t * H) + 2 * v;
            const float4 lo = __ldg(src), hi = __ldg(src + 1);
            const float sv[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += sv[i];
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        reinterpret_cast<uint4 *>(out + t * H)[v] = o;
    }
}

}  // namespace

cudaError_t launch_combine(const float *y_perm, int nsplit, int64_t split_stride, const int32_t *token_to_row,
                           const float *topk_w, const float *shared_out, int64_t N, int H, int k, uint16_t *out,
                           cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    if (N > 65535) {  // grid.y limit: process in slabs of 65535 tokens
        for (int64_t t0 = 0; t0 < N; t0 += 65535) {
            const int64_t n = N - t0 < 65535 ? N - t0 : 65535;
            cudaError_t e = launch_combine(y_perm, nsplit, split_stride, token_to_row + t0 * k, topk_w + t0 * k,
                                           shared_out ? shared_out + t0 * H : nullptr, n, H, k, out + t0 * H, s);
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    const dim3 grid((unsigned)((H / 8 + kThreads - 1) / kThreads), (unsigned)N);
    return launch_pdl(combine_kernel, grid, dim3(kThreads), 0, s, y_perm, nsplit, split_stride, token_to_row, topk_w,
                      shared_out, N, H, k, out);
}

}  // namespace moe
