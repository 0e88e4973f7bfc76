// router.cu -- router logits, top-k and routing weights (sm_100a).
//
// MoE-latency article, section "dense 和 MoE 的差别": the router reads each token's
// hidden state, scores every expert, keeps the top k and gives k routing weights.
//
//   logit[t,e] = sum_h x[t,h] * W_gate[h,e] (+ bias[e])        fp32-grade logits
//   picks      = k largest logits; equal values -> lower expert index first
//   w_j        = exp(l_j - l_0) / sum_i exp(l_i - l_0)          (softmax over all E
//                renormalised over the picks equals the softmax of the picked logits)
//
// Three paths, chosen by shape (router_path):
//  * kFused (E <= 16, or no buffer for logits): one kernel -- a block per tile of TT
//    tokens, 8 warps splitting H (warp w takes 64-column chunks w, w+8, ...; a lane two
//    adjacent columns), all experts in passes of 8, then the top-k in the same block;
//  * kSplitE (E > 16, small N): the logits kernel's grid also splits the experts into
//    slices of 8, so a batch of a few tokens still spreads W_gate over many SMs; a
//    second kernel does the top-k;
//  * kTensor (large N x E): the logits are a GEMM on the tcgen05 tensor cores.  W_gate
//    is split into three bf16 terms hi + mid + lo (each the bf16 rounding of what the
//    previous terms left; the remainder is below 2^-26 |w|), so x (bf16) times each
//    term is exact and accumulates in fp32 in TMEM; the grouped GEMM kernel runs once
//    over the stacked [3E, H] operand and the top-k kernel adds the three partial logits.
// All reductions run in a fixed order: the logits' bits do not depend on timing.
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

// Partial logits of TT tokens x one 8-expert slice [e0, e0+ne) over this warp's
// share of H, reduced over the warp's lanes (every lane ends with the sums).
template <int TT>
__device__ __forceinline__ void logits_slice(const uint16_t *__restrict__ x, const float *__restrict__ W_gate,
                                             int64_t t0, int nt, int H, int E, int e0, int ne, int warp, int lane,
                                             float (&acc)[TT][kEC])
{
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
}

// Top-k of one token's E logits (in `row`) on one warp; lane 0 writes the picks
// and their weights.
__device__ __forceinline__ void topk_warp(const float *row, int E, int k, int lane, int32_t *__restrict__ idx_out,
                                          float *__restrict__ w_out)
{
    constexpr int kPer = kMaxE / 32;
    float v[kPer];
    bool taken[kPer];
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
        const int e = lane + 32 * m;
        v[m] = e < E ? row[e] : 0.f;
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
        float ex[kMaxK];
        float den = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j < k) { ex[j] = expf(pv[j] - l0); den += ex[j]; }
#pragma unroll
        for (int j = 0; j < kMaxK; ++j)
            if (j < k) { idx_out[j] = pi[j]; w_out[j] = ex[j] / den; }
    }
}

// kFused: logits for all experts and the top-k in one block of TT tokens.
template <int TT>
__global__ void __launch_bounds__(kThreads)
    router_fused_kernel(const uint16_t *__restrict__ x, const float *__restrict__ W_gate,
                        const float *__restrict__ bias, int64_t N, int H, int E, int k,
                        float *__restrict__ logits, int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    extern __shared__ float smem[];
    float *partial = smem;                        // [kWarps][TT][E]
    float *s_logit = smem + kWarps * TT * E;      // [TT][E]
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * TT;
    const int nt = (N - t0) < TT ? (int)(N - t0) : TT;
    for (int e0 = 0; e0 < E; e0 += kEC) {
        const int ne = min(kEC, E - e0);
        float acc[TT][kEC];
        logits_slice<TT>(x, W_gate, t0, nt, H, E, e0, ne, warp, lane, acc);
        if (lane == 0) {
#pragma unroll
            for (int t = 0; t < TT; ++t)
#pragma unroll
                for (int j = 0; j < kEC; ++j)
                    if (j < ne) partial[(warp * TT + t) * E + e0 + j] = acc[t][j];
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nt * E; i += kThreads) {  // fixed-order sum over warps
        const int t = i / E, e = i % E;
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += partial[(w * TT + t) * E + e];
        if (bias) v += bias[e];
        s_logit[t * E + e] = v;
        if (logits) logits[(t0 + t) * E + e] = v;
    }
    __syncthreads();
    for (int t = warp; t < nt; t += kWarps)
        topk_warp(s_logit + t * E, E, k, lane, topk_idx + (t0 + t) * k, topk_w + (t0 + t) * k);
}

// kSplitE: logits of TT tokens x one 8-expert slice (blockIdx.y) per block.
template <int TT>
__global__ void __launch_bounds__(kThreads)
    router_logits_kernel(const uint16_t *__restrict__ x, const float *__restrict__ W_gate,
                         const float *__restrict__ bias, int64_t N, int H, int E, float *__restrict__ logits)
{
    __shared__ float partial[kWarps][TT][kEC];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * TT;
    const int nt = (N - t0) < TT ? (int)(N - t0) : TT;
    const int e0 = blockIdx.y * kEC;
    const int ne = min(kEC, E - e0);
    float acc[TT][kEC];
    logits_slice<TT>(x, W_gate, t0, nt, H, E, e0, ne, warp, lane, acc);
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < TT; ++t)
#pragma unroll
            for (int j = 0; j < kEC; ++j) partial[warp][t][j] = acc[t][j];
    }
    __syncthreads();
    if (threadIdx.x < nt * kEC) {
        const int t = threadIdx.x / kEC, j = threadIdx.x % kEC;
        if (j < ne) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += partial[w][t][j];
            if (bias) v += bias[e0 + j];
            logits[(t0 + t) * E + e0 + j] = v;
        }
    }
}

// Top-k, one warp per token.  parts == 1: `lin` holds the logits [N,E].  parts == 3:
// `lin` holds the three partial logits [N,3E] of the tensor path (hi, mid, lo terms
// of W_gate); they are summed (+ bias), written to `logits`, then ranked.
__global__ void __launch_bounds__(kThreads)
    router_topk_kernel(const float *__restrict__ lin, int parts, const float *__restrict__ bias, int64_t N, int E,
                       int k, float *__restrict__ logits, int32_t *__restrict__ topk_idx,
                       float *__restrict__ topk_w)
{
    __shared__ float row[kWarps][kMaxE];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
    if (t >= N) return;  // the whole warp leaves; no block-wide barrier below
    for (int e = lane; e < E; e += 32) {
        float v;
        if (parts == 3) {
            const float *p = lin + t * 3 * E;
            v = (p[e] + p[E + e]) + p[2 * E + e];
            if (bias) v += bias[e];
            if (logits) logits[t * E + e] = v;
        } else {
            v = lin[t * E + e];
        }
        row[warp][e] = v;
    }
    __syncwarp();
    topk_warp(row[warp], E, k, lane, topk_idx + t * k, topk_w + t * k);
}

// kTensor: W_gate [H,E] fp32 -> three bf16 terms, stacked K-major as [3E, H]:
// rows e, E+e, 2E+e hold hi, mid, lo of column e.  32x32 tiles through shared
// memory keep both the read and the transposed write coalesced.
__global__ void __launch_bounds__(kThreads)
    router_split_kernel(const float *__restrict__ W_gate, int H, int E, uint16_t *__restrict__ wsplit)
{
    __shared__ float tile[32][33];
    pdl_entry();
    const int h0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int i = ty; i < 32; i += kWarps) {
        const int h = h0 + i, e = e0 + tx;
        tile[i][tx] = (h < H && e < E) ? W_gate[(int64_t)h * E + e] : 0.f;
    }
    __syncthreads();
    for (int i = ty; i < 32; i += kWarps) {
        const int e = e0 + i, h = h0 + tx;
        if (e < E && h < H) {
            const float w = tile[tx][i];
            const uint16_t hi = float_to_bf16_bits(w);
            const float r1 = w - bf16_bits_to_float(hi);  // exact
            const uint16_t mid = float_to_bf16_bits(r1);
            const float r2 = r1 - bf16_bits_to_float(mid);  // exact
            const uint16_t lo = float_to_bf16_bits(r2);
            wsplit[(int64_t)e * H + h] = hi;
            wsplit[(int64_t)(E + e) * H + h] = mid;
            wsplit[(int64_t)(2 * E + e) * H + h] = lo;
        }
    }
}

template <int TT>
cudaError_t launch_fused(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E, int k,
                         float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    const size_t smem = sizeof(float) * (size_t)(kWarps * TT * E + TT * E);
    auto kern = router_fused_kernel<TT>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3((unsigned)((N + TT - 1) / TT)), dim3(kThreads), smem, s, x, W_gate, bias, N, H, E, k,
                      logits, topk_idx, topk_w);
}

template <int TT>
cudaError_t launch_split_e(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E,
                           int k, float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    const dim3 grid((unsigned)((N + TT - 1) / TT), (unsigned)((E + kEC - 1) / kEC));
    cudaError_t e = launch_pdl(router_logits_kernel<TT>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H, E, logits);
    if (e != cudaSuccess) return e;
    return launch_pdl(router_topk_kernel, dim3((unsigned)((N + kWarps - 1) / kWarps)), dim3(kThreads), 0, s,
                      (const float *)logits, 1, (const float *)nullptr, N, E, k, (float *)nullptr, topk_idx, topk_w);
}

// Tokens per block for the CUDA-core paths: keep about two blocks per SM (times the
// expert slices) before sharing W_gate reads between tokens.
int tokens_per_block(int64_t N, int64_t slices)
{
    const int64_t want = 2 * (int64_t)device_sm_count();
    if (N * slices >= 8 * want) return 8;
    if (N * slices >= 4 * want) return 4;
    if (N * slices >= 2 * want) return 2;
    return 1;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

}  // namespace

RouterPath router_path(int64_t N, int E, bool have_logits_buffer, bool have_ws)
{
    if (have_ws && N >= 256 && N * (int64_t)E >= 32768) return RouterPath::kTensor;
    if (E > 16 && (have_logits_buffer || have_ws)) return RouterPath::kSplitE;
    return RouterPath::kFused;
}

size_t router_ws_bytes(int64_t N, int H, int E)
{
    return align256((size_t)3 * E * H * 2) + align256((size_t)N * 3 * E * 4) + align256((size_t)N * E * 4);
}

cudaError_t launch_router(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E,
                          int k, float *logits, int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                          int *dev_err, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    const bool have_ws = ws != nullptr && ws_bytes >= router_ws_bytes(N, H, E);
    const RouterPath path = router_path(N, E, logits != nullptr, have_ws);
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    const size_t split_bytes = align256((size_t)3 * E * H * 2);
    const size_t parts_bytes = align256((size_t)N * 3 * E * 4);
    float *lbuf = logits ? logits : (have_ws ? reinterpret_cast<float *>(w8 + split_bytes + parts_bytes) : nullptr);

    if (path == RouterPath::kTensor) {
        uint16_t *wsplit = reinterpret_cast<uint16_t *>(w8);
        float *parts = reinterpret_cast<float *>(w8 + split_bytes);
        const dim3 sgrid((unsigned)((H + 31) / 32), (unsigned)((E + 31) / 32));
        cudaError_t e = launch_pdl(router_split_kernel, sgrid, dim3(kThreads), 0, s, W_gate, H, E, wsplit);
        if (e != cudaSuccess) return e;
        GroupedGemmArgs g{};
        g.act = x; g.w_a = wsplit; g.w_b = nullptr; g.offsets = nullptr; g.groups = 1; g.R = N;
        g.rows_single = (int)N; g.K = H; g.Nout = 3 * E; g.out = parts; g.dev_err = dev_err; g.token_tile = 128;
        e = launch_gemm2(g, s);
        if (e != cudaSuccess) return e;
        return launch_pdl(router_topk_kernel, dim3((unsigned)((N + kWarps - 1) / kWarps)), dim3(kThreads), 0, s,
                          (const float *)parts, 3, bias, N, E, k, lbuf, topk_idx, topk_w);
    }
    if (path == RouterPath::kSplitE) {
        switch (tokens_per_block(N, (E + kEC - 1) / kEC)) {
            case 8: return launch_split_e<8>(x, W_gate, bias, N, H, E, k, lbuf, topk_idx, topk_w, s);
            case 4: return launch_split_e<4>(x, W_gate, bias, N, H, E, k, lbuf, topk_idx, topk_w, s);
            case 2: return launch_split_e<2>(x, W_gate, bias, N, H, E, k, lbuf, topk_idx, topk_w, s);
            default: return launch_split_e<1>(x, W_gate, bias, N, H, E, k, lbuf, topk_idx, topk_w, s);
        }
    }
    switch (tokens_per_block(N, 1)) {
        case 8: return launch_fused<8>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
        case 4: return launch_fused<4>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
        case 2: return launch_fused<2>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
        default: return launch_fused<1>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
    }
}

}  // namespace moe
