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
// rounding after the expert GEMMs.
//
// One block per token row, each thread 8 consecutive features (two 16-byte fp32
// loads per row, one 16-byte bf16 store); HBM-bound: k rows read, one written.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxK = 8;

__global__ void __launch_bounds__(kThreads)
    combine_kernel(const float *__restrict__ y_perm, const int32_t *__restrict__ token_to_row,
                   const float *__restrict__ topk_w, const float *__restrict__ shared_out, int64_t N,
                   int H, int k, uint16_t *__restrict__ out)
{
    const int64_t t = blockIdx.x;
    int rows[kMaxK];
    float w[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
        rows[j] = j < k ? token_to_row[t * k + j] : -1;
        w[j] = j < k ? topk_w[t * k + j] : 0.f;
    }
    const int nvec = H / 8;
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (j < k && rows[j] >= 0) {
                const float4 *src = reinterpret_cast<const float4 *>(y_perm + (int64_t)rows[j] * H) + 2 * v;
                const float4 lo = __ldg(src), hi = __ldg(src + 1);
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

cudaError_t launch_combine(const float *y_perm, const int32_t *token_to_row, const float *topk_w,
                           const float *shared_out, int64_t N, int H, int k, uint16_t *out, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    combine_kernel<<<(unsigned)N, kThreads, 0, s>>>(y_perm, token_to_row, topk_w, shared_out, N, H, k, out);
    return cudaGetLastError();
}

}  // namespace moe
