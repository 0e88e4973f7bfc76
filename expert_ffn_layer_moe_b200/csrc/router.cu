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
//  * kFused (no buffer for logits at all): one kernel -- a block per tile of TT
//    tokens, 8 warps splitting H (warp w takes 64-column chunks w, w+8, ...; a lane two
//    adjacent columns), all experts in passes of 8, then the top-k in the same block;
//  * kSplit (small N): the logits kernel's grid splits the tokens into tiles of up to
//    8, the experts into slices of 8 and H into Z slices, so that a batch of a few
//    tokens still spreads the W_gate read over every SM; the top-k kernel adds the Z
//    partial sums in slice order.  Where one slice of H is all it would use and the
//    experts fit two slices of 8, the fused kernel runs instead (same blocks, one
//    launch);
//  * kTensor (large N x E): the logits are a GEMM on the tcgen05 tensor cores.  W_gate
//    is split into three bf16 terms hi + mid + lo (each the bf16 rounding of what the
//    previous terms left; the remainder is below 2^-26 |w|), so x (bf16) times each
//    term is exact and accumulates in fp32 in TMEM.  The grouped GEMM kernel runs once
//    over the stacked [3E, H] operand -- on single-CTA tiles of 128 rows where those
//    pad 3E less than CTA pairs' 256 (E = 128: 384 rows instead of 512), with K split
//    into S slices so that mid-size batches cover the SMs -- and the top-k kernel adds
//    the 3 S partial logits (slices interleaved in each output row, so they sit one
//    stride apart) in a fixed order.
// All reductions run in a fixed order: the logits' bits do not depend on timing.
#include "common.cuh"
#include "dispatch_block.cuh"
#include "internal.h"
#include "topk_warp.cuh"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kEC = 8;      // experts accumulated per pass
constexpr int kChunk = 64;  // columns of H per warp step (2 per lane)
constexpr int kMaxE = 256;
constexpr int kMaxK = 8;

// Partial logits of TT tokens x one 8-expert slice [e0, e0+ne) over this warp's
// share of the columns [h_begin, h_end) of H, per lane (warp_sum_store adds the lanes).
template <int TT>
__device__ __forceinline__ void logits_slice(const uint16_t *__restrict__ x, const float *__restrict__ W_gate,
                                             int64_t t0, int nt, int H, int h_begin, int h_end, int E, int e0,
                                             int ne, int warp, int lane, float (&acc)[TT][kEC])
{
#pragma unroll
    for (int t = 0; t < TT; ++t)
#pragma unroll
        for (int j = 0; j < kEC; ++j) acc[t][j] = 0.f;
    // full 8-expert slices of rows whose start is 16-byte aligned load as float4
    const bool vec = ne == kEC && (E & 3) == 0;
#pragma unroll 4
    for (int c = h_begin + warp * kChunk; c < h_end; c += kWarps * kChunk) {
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
}

// Sum each of the V = TT*8 per-lane values acc[t][j] over the warp's 32 lanes and
// store the sums to out[t * tstride + j] (j < ne).  A reduce-scatter: at each step a
// lane keeps one half of its values, sends the other half to the lane `o` apart and
// adds what it receives, so the sums end up spread over the lanes after V - V/32
// shuffles (instead of 5 V for a butterfly on every value); once a lane holds one
// value the remaining steps are a butterfly.  The additions run in a fixed order.
template <int TT>
__device__ __forceinline__ void warp_sum_store(const float (&acc)[TT][kEC], int lane, float *out, int tstride,
                                               int ne)
{
    constexpr int V = TT * kEC;
    float v[V];
#pragma unroll
    for (int f = 0; f < V; ++f) v[f] = acc[f / kEC][f % kEC];
    int base = 0;  // index of v[0] among the V values after the halving steps
#pragma unroll
    for (int st = 0; st < 5; ++st) {
        const int o = 16 >> st;
        const int S = V >> st;  // values per lane before this step (a constant once unrolled)
        if (S > 1) {
            const int h = S >> 1;
            const bool up = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < h; ++i) {
                const float send = up ? v[i] : v[i + h];
                const float keep = up ? v[i + h] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
            if (up) base += h;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
        }
    }
    constexpr int kLeft = V >= 32 ? V / 32 : 1;           // sums held per lane
    constexpr int kSame = V >= 32 ? 0 : (32 / V) - 1;    // lanes holding copies of a sum
    if ((lane & kSame) == 0) {
#pragma unroll
        for (int r = 0; r < kLeft; ++r) {
            const int f = base + r;
            const int t = f / kEC, j = f % kEC;
            if (j < ne) out[t * tstride + j] = v[r];
        }
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
        logits_slice<TT>(x, W_gate, t0, nt, H, 0, H, E, e0, ne, warp, lane, acc);
        warp_sum_store<TT>(acc, lane, partial + warp * TT * E + e0, E, ne);
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

// kSplit: partial logits of TT tokens x one 8-expert slice (blockIdx.y) over one
// slice of H (blockIdx.z, columns [z*hz, z*hz + hz)) per block, summed over the
// block's warps in warp order, stored as part[z][t][e].  With one H slice the bias is
// added here and `part` holds the logits.
template <int TT>
__global__ void __launch_bounds__(kThreads)
    router_partial_kernel(const uint16_t *__restrict__ x, const float *__restrict__ W_gate,
                          const float *__restrict__ bias, int64_t N, int H, int E, int hz, float *__restrict__ part)
{
    __shared__ float partial[kWarps][TT][kEC];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = (int64_t)blockIdx.x * TT;
    const int nt = (N - t0) < TT ? (int)(N - t0) : TT;
    const int e0 = blockIdx.y * kEC;
    const int ne = min(kEC, E - e0);
    const int h0 = (int)blockIdx.z * hz;
    float acc[TT][kEC];
    logits_slice<TT>(x, W_gate, t0, nt, H, h0, min(H, h0 + hz), E, e0, ne, warp, lane, acc);
    warp_sum_store<TT>(acc, lane, &partial[warp][0][0], kEC, kEC);
    __syncthreads();
    if (threadIdx.x < nt * kEC) {
        const int t = threadIdx.x / kEC, j = threadIdx.x % kEC;
        if (j < ne) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += partial[w][t][j];
            if (bias && gridDim.z == 1) v += bias[e0 + j];
            part[((int64_t)blockIdx.z * N + t0 + t) * E + e0 + j] = v;
        }
    }
}

// Top-k, one warp per token.  `lin` holds P partial logits of each token: part p of
// token t, expert e at lin[p * pstride + t * tstride + e] -- the P slices of H of the
// split path ([P][N][E]) or the 3 S terms and K slices of the tensor path ([N][S][3][E]).  They
// are added in part order (+ bias), written to `logits` when it is given, then ranked.
// With P == 1 and no bias `lin` already holds the logits.  P is a template argument so
// that the loads of one expert's parts, and of consecutive experts, issue together.
template <int P>
__global__ void __launch_bounds__(kThreads)
    router_topk_kernel(const float *__restrict__ lin, int64_t pstride, int64_t tstride,
                       const float *__restrict__ bias, int64_t N, int E, int k, float *__restrict__ logits,
                       int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    __shared__ float row[kWarps][kMaxE];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * kWarps + warp;
    if (t >= N) return;  // the whole warp leaves; no block-wide barrier below
    for (int e = lane; e < E; e += 32) {
        const float *p = lin + t * tstride + e;
        float part[P];
#pragma unroll
        for (int i = 0; i < P; ++i) part[i] = p[i * pstride];
        float v = part[0];
#pragma unroll
        for (int i = 1; i < P; ++i) v += part[i];
        if (bias) v += bias[e];
        if (logits) logits[t * E + e] = v;
        row[warp][e] = v;
    }
    __syncwarp();
    topk_warp(row[warp], E, k, lane, topk_idx + t * k, topk_w + t * k);
}

// Top-k from the tensor-core router's expert-major partial logits ([P][E][N]: part p of
// expert e of token t at lin[(p * E + e) * N + t]).  A block takes 32 tokens, one per
// lane, and each of its kColSplit warps an equal share of the experts: consecutive lanes read
// consecutive words.  The parts of each expert are added in part order (+ bias) as
// router_topk_kernel adds them.  Each candidate becomes one 64-bit key whose unsigned
// order is the picks' order: the high word maps the value's bits to an increasing
// integer (-0 counted as +0, NaN below every number), the low word is ~e (a lower index
// ranks higher on equal values).  The experts go in chunks of eight: a sorting network
// orders a chunk, and a bitonic merge keeps the best eight of the chunk and of the list
// so far -- no branches, so the lanes never diverge; the warps' lists then merge in a
// binary tree.  The weights use the same operations, in pick order, as topk_warp: the picks,
// weights and logits are the ones the warp kernel gives.
constexpr int kColSplit = 4;  // warps per block of 32 tokens, each ranking a quarter of the experts
static_assert((kColSplit & (kColSplit - 1)) == 0, "the lists merge in a binary tree");

__device__ __forceinline__ uint64_t pick_key(float v, int e)
{
    const uint32_t u = __float_as_uint(v + 0.0f);  // -0 + 0 = +0
    const uint32_t hi = isnan(v) ? 0u : ((u & 0x80000000u) ? ~u : (u | 0x80000000u));
    return ((uint64_t)hi << 32) | (uint32_t)~(uint32_t)e;
}
__device__ __forceinline__ float key_value(uint64_t key)
{
    const uint32_t hi = (uint32_t)(key >> 32);
    if (hi == 0u) return __uint_as_float(0x7fc00000u);
    return __uint_as_float((hi & 0x80000000u) ? (hi & 0x7fffffffu) : ~hi);
}
__device__ __forceinline__ int key_index(uint64_t key) { return (int)~(uint32_t)key; }
// compare-exchange: the larger key to a, the smaller to b
__device__ __forceinline__ void cx(uint64_t &a, uint64_t &b)
{
    const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
    a = hi;
    b = lo;
}
// Batcher's odd-even merge sort of eight, descending (19 compare-exchanges)
__device__ __forceinline__ void sort8_desc(uint64_t (&c)[8])
{
    cx(c[0], c[1]); cx(c[2], c[3]); cx(c[4], c[5]); cx(c[6], c[7]);
    cx(c[0], c[2]); cx(c[1], c[3]); cx(c[4], c[6]); cx(c[5], c[7]);
    cx(c[1], c[2]); cx(c[5], c[6]);
    cx(c[0], c[4]); cx(c[1], c[5]); cx(c[2], c[6]); cx(c[3], c[7]);
    cx(c[2], c[4]); cx(c[3], c[5]);
    cx(c[1], c[2]); cx(c[3], c[4]); cx(c[5], c[6]);
}
// top := the best eight of two descending lists of eight (top and c).  Pairing one list
// with the other reversed gives a bitonic sequence holding them, which three
// half-cleaner rounds sort.
__device__ __forceinline__ void merge8_desc(uint64_t (&top)[8], const uint64_t (&c)[8])
{
#pragma unroll
    for (int j = 0; j < 8; ++j) top[j] = top[j] > c[7 - j] ? top[j] : c[7 - j];
    cx(top[0], top[4]); cx(top[1], top[5]); cx(top[2], top[6]); cx(top[3], top[7]);
    cx(top[0], top[2]); cx(top[1], top[3]); cx(top[4], top[6]); cx(top[5], top[7]);
    cx(top[0], top[1]); cx(top[2], top[3]); cx(top[4], top[5]); cx(top[6], top[7]);
}

template <int P>
__global__ void __launch_bounds__(32 * kColSplit)
    router_topk_cols_kernel(const float *__restrict__ lin, const float *__restrict__ bias, int64_t N, int E, int k,
                            float *__restrict__ logits, int32_t *__restrict__ topk_idx, float *__restrict__ topk_w)
{
    __shared__ uint64_t lists[kColSplit][8][32];  // each warp's best eight, lane-major
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 32 + lane;
    const bool live = t < N;
    // warp w ranks experts [e_lo, e_hi): its share, in whole chunks of eight
    const int span = ((E + kColSplit - 1) / kColSplit + 7) / 8 * 8;
    const int e_lo = warp * span, e_hi = min(E, e_lo + span);
    uint64_t top[8];  // the best eight so far, in descending key order; 0 is below every candidate
#pragma unroll
    for (int j = 0; j < 8; ++j) top[j] = 0;
    const int64_t pstride = (int64_t)E * N;
    for (int e0 = e_lo; e0 < e_hi; e0 += 8) {
        float part[8][P];
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int i = 0; i < P; ++i)
                part[u][i] = live && e0 + u < e_hi ? __ldg(lin + i * pstride + (int64_t)(e0 + u) * N + t) : 0.f;
        uint64_t c[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e0 + u;
            float v = part[u][0];
#pragma unroll
            for (int i = 1; i < P; ++i) v += part[u][i];
            if (e < e_hi && bias) v += bias[e];
            if (live && e < e_hi && logits) logits[t * E + e] = v;
            c[u] = e < e_hi ? pick_key(v, e) : 0;
        }
        sort8_desc(c);
        merge8_desc(top, c);
    }
    // merge the warps' lists in a tree: at distance d, warp w (a multiple of 2d) takes
    // warp w + d's list
#pragma unroll
    for (int j = 0; j < 8; ++j) lists[warp][j][lane] = top[j];
#pragma unroll
    for (int d = 1; d < kColSplit; d <<= 1) {
        __syncthreads();
        if (warp % (2 * d) == 0) {
            uint64_t c[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) c[j] = lists[warp + d][j][lane];
            merge8_desc(top, c);
#pragma unroll
            for (int j = 0; j < 8; ++j) lists[warp][j][lane] = top[j];
        }
    }
    if (warp > 0 || !live) return;
    const float l0 = key_value(top[0]);
    float ex[kMaxK];
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
        if (j < k) { ex[j] = expf(key_value(top[j]) - l0); den += ex[j]; }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
        if (j < k) { topk_idx[t * k + j] = key_index(top[j]); topk_w[t * k + j] = ex[j] / den; }
}

template <int P>
cudaError_t launch_topk(const float *lin, int64_t pstride, int64_t tstride, const float *bias, int64_t N, int E,
                        int k, float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    return launch_pdl(router_topk_kernel<P>, dim3((unsigned)((N + kWarps - 1) / kWarps)), dim3(kThreads), 0, s, lin,
                      pstride, tstride, bias, N, E, k, logits, topk_idx, topk_w);
}

// Small batches: the top-k of every token (from P partial logits, summed as the top-k
// kernel sums them -- or, with P == 0, the picks the router already made), the stable
// dispatch and the row scatter in one kernel.  Every block ranks and dispatches the
// whole batch in its own shared memory (a few hundred assignments: repeating that costs
// less than a launch) and then copies the rows of its share of the tokens; block 0 also
// writes the routing and dispatch outputs.  No block waits on another.
constexpr int kFuseMaxR = 512;      // assignments of a batch this kernel takes
// Tokens every block ranks for itself (P > 0).  Past 8 the separate top-k, dispatch and
// scatter kernels win: measured on the Qwen3-30B shape (whole layer, L2 flushed), 10 / 12
// / 16 / 24 / 32 / 48 / 64 tokens took 158 / 164 / 186 / 219 / 248 / 256 / 314 us with
// every block ranking the batch and 153 / 161 / 181 / 216 / 231 / 243 / 257 us without.
constexpr int kFuseMaxTopkN = 8;
template <int P>
__global__ void __launch_bounds__(kDispThreads)
    route_dispatch_small_kernel(const float *__restrict__ lin, int64_t pstride, int64_t tstride,
                                const float *__restrict__ bias, int64_t N, int E, int k, float *__restrict__ logits,
                                int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                                const uint16_t *__restrict__ x, int H, int32_t *__restrict__ counts,
                                int32_t *__restrict__ offsets, int32_t *__restrict__ row_to_token,
                                int32_t *__restrict__ token_to_row, uint16_t *__restrict__ x_perm, int *err)
{
    static_assert(kDispThreads == kThreads, "one block size for the ranking and the dispatch");
    __shared__ DispatchSmem sm;
    __shared__ int32_t s_idx[kFuseMaxR];
    __shared__ float s_w[kFuseMaxR];
    __shared__ int32_t s_t2r[kFuseMaxR];
    __shared__ float row[P > 0 ? kWarps : 1][kMaxE];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t R = N * k;
    const bool lead = blockIdx.x == 0;
    if (P > 0) {
        for (int64_t t = warp; t < N; t += kWarps) {
            for (int e = lane; e < E; e += 32) {
                const float *p = lin + t * tstride + e;
                float part[P > 0 ? P : 1];
#pragma unroll
                for (int i = 0; i < P; ++i) part[i] = p[i * pstride];
                float v = part[0];
#pragma unroll
                for (int i = 1; i < P; ++i) v += part[i];
                if (bias) v += bias[e];
                if (logits && lead) logits[t * E + e] = v;
                row[warp][e] = v;
            }
            __syncwarp();
            topk_warp(row[warp], E, k, lane, s_idx + t * k, s_w + t * k);
            __syncwarp();
        }
        __syncthreads();
        if (lead)
            for (int64_t a = threadIdx.x; a < R; a += kDispThreads) {
                topk_idx[a] = s_idx[a];
                topk_w[a] = s_w[a];
            }
    } else {
        for (int64_t a = threadIdx.x; a < R; a += kDispThreads) s_idx[a] = topk_idx[a];
        __syncthreads();
    }
    dispatch_block(s_idx, R, k, E, lead ? counts : nullptr, lead ? offsets : nullptr,
                   lead ? row_to_token : nullptr, s_t2r, lead ? err : nullptr, sm);
    if (lead)
        for (int64_t a = threadIdx.x; a < R; a += kDispThreads) token_to_row[a] = s_t2r[a];
    // x_perm[token_to_row[t,j]] = x[t] for this block's tokens t (16-byte vectors);
    // no x_perm: dispatch only (the expert kernels read x through the row maps)
    if (!x_perm) return;
    const int nvec = H / 8;
    for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * H);
        for (int v = threadIdx.x; v < nvec; v += kDispThreads) {
            const uint4 val = __ldg(src + v);
            for (int j = 0; j < k; ++j) {
                const int r = s_t2r[t * k + j];
                if (r >= 0) reinterpret_cast<uint4 *>(x_perm + (int64_t)r * H)[v] = val;
            }
        }
    }
}

template <int P>
cudaError_t launch_route_dispatch(const float *lin, int64_t pstride, int64_t tstride, const float *bias, int64_t N,
                                  int E, int k, float *logits, int32_t *topk_idx, float *topk_w, const uint16_t *x,
                                  int H, int32_t *counts, int32_t *offsets, int32_t *r2t, int32_t *t2r,
                                  uint16_t *x_perm, int *err, cudaStream_t s)
{
    const int64_t cap = 2 * (int64_t)device_sm_count();
    const unsigned grid = x_perm ? (unsigned)(N < cap ? N : cap) : 1u;  // without rows to copy, block 0 alone
    return launch_pdl(route_dispatch_small_kernel<P>, dim3(grid), dim3(kDispThreads), 0, s, lin, pstride, tstride,
                      bias, N, E, k, logits, topk_idx, topk_w, x, H, counts, offsets, r2t, t2r, x_perm, err);
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
cudaError_t launch_split(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E, int k,
                         int Z, float *part, float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    const int hz = (H / Z / kChunk) * kChunk;  // Z divides H / 64 (split_shape)
    const dim3 grid((unsigned)((N + TT - 1) / TT), (unsigned)((E + kEC - 1) / kEC), (unsigned)Z);
    cudaError_t e = launch_pdl(router_partial_kernel<TT>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H, E, hz,
                               part);
    if (e != cudaSuccess) return e;
    const int64_t ps = N * E;
    switch (Z) {  // Z == 1: `part` holds the logits, bias included
        case 1: return launch_topk<1>(part, ps, E, nullptr, N, E, k, nullptr, topk_idx, topk_w, s);
        case 2: return launch_topk<2>(part, ps, E, bias, N, E, k, logits, topk_idx, topk_w, s);
        case 4: return launch_topk<4>(part, ps, E, bias, N, E, k, logits, topk_idx, topk_w, s);
        case 8: return launch_topk<8>(part, ps, E, bias, N, E, k, logits, topk_idx, topk_w, s);
        default: return cudaErrorInvalidValue;
    }
}

// Tokens per block for the fused path: keep about two blocks per SM before sharing
// W_gate reads between tokens.
int tokens_per_block(int64_t N)
{
    const int64_t want = 2 * (int64_t)device_sm_count();
    if (N >= 8 * want) return 8;
    if (N >= 4 * want) return 4;
    if (N >= 2 * want) return 2;
    return 1;
}

// Shape of the split path: the most tokens per block (up to 4, each W_gate load then
// serves them all; 8 would take more than 128 registers a thread and halve the blocks
// an SM holds) for which the blocks, times at most `zmax` slices of H, still come to
// about two per SM; then the fewest H slices that get there.  The slice count is a
// power of two up to 8 that divides H / 64 and leaves every warp at least one 64-column
// chunk.
void split_shape(int64_t N, int H, int E, int64_t zcap, int *tt, int *z)
{
    const int64_t want = 2 * (int64_t)device_sm_count();
    const int64_t slices = (E + kEC - 1) / kEC;
    const int nch = H / kChunk;
    int zmax = 1;
    for (int c = 2; c <= 8; c *= 2)
        if (nch % c == 0 && nch / c >= kWarps && c <= zcap) zmax = c;
    *tt = 1;
    for (int c = 4; c > 1; c >>= 1)
        if (N >= c && ((N + c - 1) / c) * slices * zmax >= want) { *tt = c; break; }
    const int64_t blocks = ((N + *tt - 1) / *tt) * slices;
    int zz = 1;
    while (zz < zmax && blocks * zz < want) zz *= 2;
    *z = zz;
}

cudaError_t launch_fused_for(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E,
                             int k, float *logits, int32_t *topk_idx, float *topk_w, cudaStream_t s)
{
    switch (tokens_per_block(N)) {
        case 8: return launch_fused<8>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
        case 4: return launch_fused<4>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
        case 2: return launch_fused<2>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
        default: return launch_fused<1>(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
    }
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

constexpr int kTensorMaxSlices = 4;
// Batches from this size on run the tensor-core router transposed (at 8192 tokens the
// 128 x 128 tiles below measured faster: 64 transposed tiles leave 10 of the 74 SM
// pairs idle).
constexpr int64_t kTensorTransposedMinN = 16384;

// Tensor-core path shape: single-CTA tiles (128 operand rows) where they pad the 3E rows
// less than pairs (256), the token tile, and the K slices S: double S while the tiles
// cover fewer than the SMs (or pairs) and each slice keeps at least 8 K blocks.
void tensor_shape(int64_t N, int H, int E, int *bn, int *S, bool *single)
{
    const int64_t sms = device_sm_count();
    const int rows = 3 * E;
    *single = (rows + 127) / 128 * 128 < (rows + 255) / 256 * 256;
    *bn = N >= 2048 ? 128 : 64;
    const int per_tile = *single ? 128 : 256;
    const int64_t tiles = ((N + *bn - 1) / *bn) * ((rows + per_tile - 1) / per_tile);
    const int64_t units = *single ? sms : sms / 2;
    const int kblocks = H / 64;
    int sl = 1;
    while (sl < kTensorMaxSlices && tiles * sl < units && kblocks / (2 * sl) >= 8) sl *= 2;
    *S = sl;
}

}  // namespace

RouterPath router_path(int64_t N, int E, bool have_logits_buffer, bool have_ws)
{
    if (have_ws && N >= 256 && N * (int64_t)E >= 32768) return RouterPath::kTensor;
    if (have_logits_buffer || have_ws) return RouterPath::kSplit;
    return RouterPath::kFused;
}

cudaError_t launch_route_dispatch_small(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H,
                                        int E, int k, float *logits, int32_t *topk_idx, float *topk_w, void *ws,
                                        size_t ws_bytes, int32_t *counts, int32_t *offsets, int32_t *row_to_token,
                                        int32_t *token_to_row, uint16_t *x_perm, int *dev_err, cudaStream_t s)
{
    if (N <= 0 || N * (int64_t)k > kFuseMaxR) return cudaErrorNotSupported;
    const bool have_ws = ws != nullptr && ws_bytes >= router_ws_bytes(N, H, E);
    const RouterPath path = router_path(N, E, logits != nullptr, have_ws);
    if (path == RouterPath::kTensor) return cudaErrorNotSupported;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    const size_t split_bytes = align256((size_t)3 * E * H * 2);
    const size_t parts_bytes = align256((size_t)kTensorMaxSlices * N * 3 * E * 4);
    float *lbuf = logits ? logits : (have_ws ? reinterpret_cast<float *>(w8 + split_bytes + parts_bytes) : nullptr);
    if (path == RouterPath::kSplit) {
        float *part = have_ws ? reinterpret_cast<float *>(w8) : lbuf;
        const int64_t zcap = have_ws ? (int64_t)((split_bytes + parts_bytes) / ((size_t)N * E * 4)) : 1;
        int tt, z;
        split_shape(N, H, E, zcap, &tt, &z);
        if (!(z == 1 && E <= 2 * kEC)) {
            if (N > kFuseMaxTopkN) return cudaErrorNotSupported;
            if (z == 1) part = lbuf;
            const int hz = (H / z / kChunk) * kChunk;
            const dim3 grid((unsigned)((N + tt - 1) / tt), (unsigned)((E + kEC - 1) / kEC), (unsigned)z);
            cudaError_t e;
            switch (tt) {
                case 4: e = launch_pdl(router_partial_kernel<4>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H, E,
                                       hz, part); break;
                case 2: e = launch_pdl(router_partial_kernel<2>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H, E,
                                       hz, part); break;
                default: e = launch_pdl(router_partial_kernel<1>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H,
                                        E, hz, part); break;
            }
            if (e != cudaSuccess) return e;
            const int64_t ps = N * E;
            switch (z) {  // z == 1: `part` holds the logits, bias included
                case 1: return launch_route_dispatch<1>(part, ps, E, nullptr, N, E, k, nullptr, topk_idx, topk_w, x, H,
                                                        counts, offsets, row_to_token, token_to_row, x_perm, dev_err, s);
                case 2: return launch_route_dispatch<2>(part, ps, E, bias, N, E, k, lbuf, topk_idx, topk_w, x, H, counts,
                                                        offsets, row_to_token, token_to_row, x_perm, dev_err, s);
                case 4: return launch_route_dispatch<4>(part, ps, E, bias, N, E, k, lbuf, topk_idx, topk_w, x, H, counts,
                                                        offsets, row_to_token, token_to_row, x_perm, dev_err, s);
                case 8: return launch_route_dispatch<8>(part, ps, E, bias, N, E, k, lbuf, topk_idx, topk_w, x, H, counts,
                                                        offsets, row_to_token, token_to_row, x_perm, dev_err, s);
                default: return cudaErrorInvalidValue;
            }
        }
    }
    // the one-kernel router makes the picks; then the dispatch and the rows
    cudaError_t e = launch_fused_for(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
    if (e != cudaSuccess) return e;
    return launch_route_dispatch<0>(nullptr, 0, 0, nullptr, N, E, k, nullptr, topk_idx, topk_w, x, H, counts, offsets,
                                    row_to_token, token_to_row, x_perm, dev_err, s);
}

// Decode batches: the router's partial logits only; the top-k runs in the first decode
// GEMV kernel (every block ranks the few tokens itself).  With the one-kernel router
// (one slice of H and E <= 16) the picks are made here instead (rp->P = 0).
cudaError_t launch_router_partials(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E,
                                   int k, float *logits, int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                                   RouterPartials *rp, cudaStream_t s)
{
    if (N <= 0 || N > MOE_DECODE_MAX_TOKENS) return cudaErrorNotSupported;
    const bool have_ws = ws != nullptr && ws_bytes >= router_ws_bytes(N, H, E);
    const RouterPath path = router_path(N, E, logits != nullptr, have_ws);
    if (path == RouterPath::kTensor) return cudaErrorNotSupported;
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    const size_t split_bytes = align256((size_t)3 * E * H * 2);
    const size_t parts_bytes = align256((size_t)kTensorMaxSlices * N * 3 * E * 4);
    float *lbuf = logits ? logits : (have_ws ? reinterpret_cast<float *>(w8 + split_bytes + parts_bytes) : nullptr);
    if (path == RouterPath::kSplit) {
        float *part = have_ws ? reinterpret_cast<float *>(w8) : lbuf;
        const int64_t zcap = have_ws ? (int64_t)((split_bytes + parts_bytes) / ((size_t)N * E * 4)) : 1;
        int tt, z;
        split_shape(N, H, E, zcap, &tt, &z);
        if (!(z == 1 && E <= 2 * kEC)) {
            if (z == 1) part = lbuf;
            const int hz = (H / z / kChunk) * kChunk;
            const dim3 grid((unsigned)((N + tt - 1) / tt), (unsigned)((E + kEC - 1) / kEC), (unsigned)z);
            cudaError_t e;
            switch (tt) {
                case 4: e = launch_pdl(router_partial_kernel<4>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H, E,
                                       hz, part); break;
                case 2: e = launch_pdl(router_partial_kernel<2>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H, E,
                                       hz, part); break;
                default: e = launch_pdl(router_partial_kernel<1>, grid, dim3(kThreads), 0, s, x, W_gate, bias, N, H,
                                        E, hz, part); break;
            }
            if (e != cudaSuccess) return e;
            // z == 1: `part` holds the logits, bias included
            rp->part = part;
            rp->P = z;
            rp->pstride = N * E;
            rp->bias = z == 1 ? nullptr : bias;
            rp->logits = z == 1 ? nullptr : lbuf;
            return cudaSuccess;
        }
    }
    rp->part = nullptr;
    rp->P = 0;
    rp->pstride = 0;
    rp->bias = nullptr;
    rp->logits = nullptr;
    return launch_fused_for(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
}

size_t router_ws_bytes(int64_t N, int H, int E)
{
    return align256((size_t)3 * E * H * 2) + align256((size_t)kTensorMaxSlices * N * 3 * E * 4) +
           align256((size_t)N * E * 4);
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
    const size_t parts_bytes = align256((size_t)kTensorMaxSlices * N * 3 * E * 4);
    float *lbuf = logits ? logits : (have_ws ? reinterpret_cast<float *>(w8 + split_bytes + parts_bytes) : nullptr);

    if (path == RouterPath::kTensor) {
        uint16_t *wsplit = reinterpret_cast<uint16_t *>(w8);
        float *parts = reinterpret_cast<float *>(w8 + split_bytes);
        const dim3 sgrid((unsigned)((H + 31) / 32), (unsigned)((E + 31) / 32));
        cudaError_t e = launch_pdl(router_split_kernel, sgrid, dim3(kThreads), 0, s, W_gate, H, E, wsplit);
        if (e != cudaSuccess) return e;
        if (N >= kTensorTransposedMinN) {
            // tokens on the MMA's M side (256 per CTA pair), the 3E terms on its N side in
            // at most 256-row tiles: each operand byte serves more FLOPs than the 128 x 128
            // tiles below, and the output [3E][N] is expert-major
            float *parts = reinterpret_cast<float *>(w8 + split_bytes);
            const int rows = 3 * E;
            const int ntiles = (rows + 255) / 256;
            const int bn = ((rows + ntiles - 1) / ntiles + 31) / 32 * 32;
            GroupedGemmArgs g{};
            g.w_a = x; g.act = wsplit; g.w_b = nullptr; g.offsets = nullptr; g.groups = 1; g.R = rows;
            g.rows_single = rows; g.K = H; g.Nout = (int)N; g.out = parts; g.dev_err = dev_err;
            g.token_tile = bn; g.ldo = N;
            e = launch_gemm2(g, s);
            if (e != cudaSuccess) return e;
            return launch_pdl(router_topk_cols_kernel<3>, dim3((unsigned)((N + 31) / 32)), dim3(32 * kColSplit), 0,
                              s, parts, bias, N, E, k, lbuf, topk_idx, topk_w);
        }
        int bn, S;
        bool single;
        tensor_shape(N, H, E, &bn, &S, &single);
        // K slice s of token t's three terms lands at parts + t*3ES + s*3E (row stride 3ES,
        // slices 3E apart): part p = 3s + term of expert e sits at t*3ES + p*E + e
        GroupedGemmArgs g{};
        g.act = x; g.w_a = wsplit; g.w_b = nullptr; g.offsets = nullptr; g.groups = 1; g.R = N;
        g.rows_single = (int)N; g.K = H; g.Nout = 3 * E; g.out = parts; g.dev_err = dev_err;
        g.token_tile = bn; g.single_cta = single; g.ksplit = S;
        g.ldo = (int64_t)3 * E * S; g.split_stride = (int64_t)3 * E;
        e = launch_gemm2(g, s);
        if (e != cudaSuccess) return e;
        const int64_t ts = (int64_t)3 * E * S;
        switch (S) {
            case 1: return launch_topk<3>(parts, E, ts, bias, N, E, k, lbuf, topk_idx, topk_w, s);
            case 2: return launch_topk<6>(parts, E, ts, bias, N, E, k, lbuf, topk_idx, topk_w, s);
            case 4: return launch_topk<12>(parts, E, ts, bias, N, E, k, lbuf, topk_idx, topk_w, s);
            default: return cudaErrorInvalidValue;
        }
    }
    if (path == RouterPath::kSplit) {
        // the H-slice partials go to the scratch (its first two regions), else the
        // caller's logits buffer holds the one slice
        float *part = have_ws ? reinterpret_cast<float *>(w8) : lbuf;
        const int64_t zcap = have_ws ? (int64_t)((split_bytes + parts_bytes) / ((size_t)N * E * 4)) : 1;
        int tt, z;
        split_shape(N, H, E, zcap, &tt, &z);
        if (z == 1 && E <= 2 * kEC) {
            // nothing to gain from slicing: the one-kernel path runs the same blocks
            return launch_fused_for(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
        }
        if (z == 1) part = lbuf;
        switch (tt) {
            case 4: return launch_split<4>(x, W_gate, bias, N, H, E, k, z, part, lbuf, topk_idx, topk_w, s);
            case 2: return launch_split<2>(x, W_gate, bias, N, H, E, k, z, part, lbuf, topk_idx, topk_w, s);
            default: return launch_split<1>(x, W_gate, bias, N, H, E, k, z, part, lbuf, topk_idx, topk_w, s);
        }
    }
    return launch_fused_for(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, s);
}

}  // namespace moe
