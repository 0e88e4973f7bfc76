// permute.cu -- dispatch and permutation of token rows into expert-contiguous order.
//
// MoE-latency article, section "router 之后还有一串动作": N tokens at top-k give N*k
// assignments; grouping them by expert is dispatch, sorting the token rows by expert
// is the permutation.  The result is deterministic and stable: assignment
// a = t*k + j of expert e lands at row offsets[e] + #{a' < a : e(a') = e}.
//
// No atomics decide the row order.  Large batches take four launches:
//   1. count  : per block of permute_chunk(R) assignments, a per-expert histogram;
//   2. scan   : one block -- counts[e], offsets = exclusive scan, and every block's
//               starting row per expert (in place over the histograms);
//   3. rank   : per block again, the stable rank of each assignment inside its
//               block (warp match + per-warp counts, warps in order) -> row maps;
//   4. copy   : x_perm[token_to_row[t,j]] = x[t] for j < k -- a warp reads 2 KB of a
//               token's row once (16-byte vectors) and writes its k copies, so x is read
//               from HBM once however many experts share a token.
// Batches of at most kSmallR (1024) assignments do 1-3 in one single-block launch,
// then the gather: two launches instead of four.  Mid-sized batches (fewer than
// kPermuteFineMaxR assignments) take blocks of 256 and fold 2 into 3: each rank block
// sums the (at most 128) histograms itself, which saves the scan's launch.
#include "common.cuh"
#include "dispatch_block.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = kDispThreads;
constexpr int kWarps = kDispWarps;
constexpr int kMaxE = kDispMaxE;
// One-block dispatch up to this many assignments.  Measured on the Qwen3-30B shape (whole
// layer): 1024 assignments 263 us in one block against 265 us in the count/scan/rank
// kernels; 1600 and 2048 assignments 274 / 272 us in one block against 271 / 267 us.
constexpr int64_t kSmallR = 1024;
static_assert(kPermuteChunk % kThreads == 0, "chunk is whole rounds of the block");

__global__ void __launch_bounds__(kThreads)
    count_kernel(const int32_t *__restrict__ idx, int64_t R, int E, int chunk, int32_t *__restrict__ blk_cnt,
                 int *err)
{
    __shared__ int hist[kMaxE];
    pdl_entry();
    for (int e = threadIdx.x; e < E; e += kThreads) hist[e] = 0;
    __syncthreads();
    const int64_t a0 = (int64_t)blockIdx.x * chunk;
    for (int i = threadIdx.x; i < chunk; i += kThreads) {
        const int64_t a = a0 + i;
        if (a >= R) break;
        const int e = idx[a];
        if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
        else set_device_error(err, MOE_DEVERR_BAD_EXPERT_INDEX);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kThreads) blk_cnt[(int64_t)blockIdx.x * E + e] = hist[e];
}

// One block: totals per expert, exclusive scan, and per-block starting rows.
__global__ void __launch_bounds__(kThreads)
    scan_kernel(int32_t *__restrict__ blk_cnt, int64_t nblk, int E, int32_t *__restrict__ counts,
                int32_t *__restrict__ offsets)
{
    __shared__ int s[kMaxE];
    pdl_entry();
    const int e = threadIdx.x;
    int total = 0;
    if (e < E)
        for (int64_t b = 0; b < nblk; ++b) total += blk_cnt[b * E + e];
    s[e] = e < E ? total : 0;
    __syncthreads();
    // inclusive Hillis-Steele scan over kThreads (>= E) entries
    for (int o = 1; o < kThreads; o <<= 1) {
        const int v = e >= o ? s[e - o] : 0;
        __syncthreads();
        s[e] += v;
        __syncthreads();
    }
    if (e < E) {
        const int start = s[e] - total;
        counts[e] = total;
        offsets[e] = start;
        if (e == E - 1) offsets[E] = s[e];
        int run = start;
        for (int64_t b = 0; b < nblk; ++b) {
            const int c = blk_cnt[b * E + e];
            blk_cnt[b * E + e] = run;
            run += c;
        }
    }
}

// Small batches: histogram, exclusive scan and stable ranks in one block.
__global__ void __launch_bounds__(kThreads)
    dispatch_small_kernel(const int32_t *__restrict__ idx, int64_t R, int k, int E, int32_t *__restrict__ counts,
                          int32_t *__restrict__ offsets, int32_t *__restrict__ row_to_token,
                          int32_t *__restrict__ token_to_row, int *err)
{
    __shared__ DispatchSmem sm;
    pdl_entry();
    dispatch_block(idx, R, k, E, counts, offsets, row_to_token, token_to_row, err, sm);
}

__global__ void __launch_bounds__(kThreads)
    rank_kernel(const int32_t *__restrict__ idx, int64_t R, int k, int E,
                const int32_t *__restrict__ blk_base, int32_t *__restrict__ row_to_token,
                int32_t *__restrict__ token_to_row)
{
    __shared__ int base[kMaxE];
    __shared__ int wcnt[kWarps][kMaxE];
    pdl_entry();
    for (int e = threadIdx.x; e < E; e += kThreads) base[e] = blk_base[(int64_t)blockIdx.x * E + e];
    const int64_t a0 = (int64_t)blockIdx.x * kPermuteChunk;
    for (int round = 0; round < kPermuteChunk / kThreads; ++round) {
        const int64_t ar = a0 + (int64_t)round * kThreads;
        if (ar >= R) break;  // uniform across the block
        rank_round(idx, R, k, E, ar, base, wcnt, row_to_token, token_to_row);
    }
}

// Mid-sized batches: the scan and the rank of one block of kPermuteFineChunk (one round of
// the block) assignments.  Thread e sums expert e's histogram entries over all nblk
// blocks (the total) and over the blocks before this one; an exclusive scan of the
// totals gives offsets, and this block's rows of expert e start at offsets[e] plus the
// earlier blocks' count.  Block 0 writes counts and offsets.  The histograms stay as they
// are (every block reads all of them).
__global__ void __launch_bounds__(kThreads)
    rank_scan_kernel(const int32_t *__restrict__ idx, int64_t R, int k, int E,
                     const int32_t *__restrict__ blk_cnt, int64_t nblk, int32_t *__restrict__ counts,
                     int32_t *__restrict__ offsets, int32_t *__restrict__ row_to_token,
                     int32_t *__restrict__ token_to_row)
{
    static_assert(kPermuteFineChunk == kThreads, "one round per block");
    __shared__ int base[kMaxE];
    __shared__ int s[kThreads];
    __shared__ int wcnt[kWarps][kMaxE];
    pdl_entry();
    const int e = threadIdx.x;
    int total = 0, before = 0;
    if (e < E) {
#pragma unroll 8
        for (int64_t b = 0; b < nblk; ++b) {
            const int c = blk_cnt[b * E + e];
            total += c;
            before += b < (int64_t)blockIdx.x ? c : 0;
        }
    }
    s[e] = total;
    __syncthreads();
    for (int o = 1; o < kThreads; o <<= 1) {  // inclusive Hillis-Steele scan
        const int v = e >= o ? s[e - o] : 0;
        __syncthreads();
        s[e] += v;
        __syncthreads();
    }
    if (e < E) {
        const int start = s[e] - total;
        base[e] = start + before;
        if (blockIdx.x == 0) {
            counts[e] = total;
            offsets[e] = start;
            if (e == E - 1) offsets[E] = s[e];
        }
    }
    __syncthreads();
    rank_round(idx, R, k, E, (int64_t)blockIdx.x * kPermuteFineChunk, base, wcnt, row_to_token, token_to_row);
}

// x_perm[token_to_row[t,j]] = x[t] for every assignment with a valid row.  A warp's
// unit of work is 2 KB of one token's row (128 16-byte vectors, four per lane, all in
// flight at once), read once and written to the token's k rows; units run grid-stride.
// Rows are H 16-bit words (bf16 values, or pairs of e4m3 bytes); with scale_in the
// per-row scales move the same way (scale_out[token_to_row[t,j]] = scale_in[t]).  Target
// rows outside [0, out_rows) are skipped.
constexpr int kScatterVec = 128;
__global__ void __launch_bounds__(kThreads)
    scatter_rows_kernel(const uint16_t *__restrict__ x, const int32_t *__restrict__ token_to_row, int64_t N, int k,
                        int H, uint16_t *__restrict__ x_perm, int64_t out_rows, const float *__restrict__ scale_in,
                        float *__restrict__ scale_out)
{
    pdl_entry();
    const int nvec = H / 8;
    const int chunks = (nvec + kScatterVec - 1) / kScatterVec;
    const int64_t warp_global = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const int lane = threadIdx.x & 31;
    for (int64_t unit = warp_global; unit < N * chunks; unit += nwarps) {
        const int64_t t = unit / chunks;
        const int v0 = (int)(unit % chunks) * kScatterVec + lane;
        int rows[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = j < k ? token_to_row[t * k + j] : -1;
            rows[j] = r < out_rows ? r : -1;  // outside the target: skipped
        }
        if (scale_in && v0 == lane && lane < k) {  // first chunk of the row: lane j moves pick j's scale
            const int r = token_to_row[t * k + lane];
            if (r >= 0 && r < out_rows) scale_out[r] = scale_in[t];
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * H);
        {
            uint4 buf[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (v0 + 32 * u < nvec) buf[u] = __ldg(src + v0 + 32 * u);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (rows[j] < 0) continue;
                uint4 *dst = reinterpret_cast<uint4 *>(x_perm + (int64_t)rows[j] * H);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (v0 + 32 * u < nvec) dst[v0 + 32 * u] = buf[u];
            }
        }
    }
}

}  // namespace

cudaError_t launch_scatter_rows(const uint16_t *x, const float *scale_in, const int32_t *token_to_row, int64_t N,
                                int k, int H, uint16_t *x_perm, int64_t out_rows, float *scale_out, cudaStream_t s)
{
    if (N <= 0) return cudaSuccess;
    const int64_t units = N * ((H / 8 + kScatterVec - 1) / kScatterVec);
    const int64_t want = (units + kWarps - 1) / kWarps;
    const int gblocks = (int)(want < 148 * 8 ? want : 148 * 8);
    return launch_pdl(scatter_rows_kernel, dim3(gblocks), dim3(kThreads), 0, s, x, token_to_row, N, k, H, x_perm,
                      out_rows, scale_in, scale_out);
}

cudaError_t launch_permute(const uint16_t *x, const int32_t *topk_idx, int64_t N, int H, int E, int k,
                           int32_t *counts, int32_t *offsets, int32_t *row_to_token, int32_t *token_to_row,
                           uint16_t *x_perm, int32_t *scratch, int *dev_err, cudaStream_t s)
{
    const int64_t R = N * k;
    if (R <= 0) return cudaSuccess;
    if (R <= kSmallR) {
        cudaError_t e = launch_pdl(dispatch_small_kernel, dim3(1), dim3(kThreads), 0, s, topk_idx, R, k, E, counts,
                                   offsets, row_to_token, token_to_row, dev_err);
        if (e != cudaSuccess) return e;
    } else {
        const int64_t chunk = permute_chunk(R), nblk = permute_blocks(R);
        cudaError_t e = launch_pdl(count_kernel, dim3((unsigned)nblk), dim3(kThreads), 0, s, topk_idx, R, E,
                                   (int)chunk, scratch, dev_err);
        if (e == cudaSuccess && chunk == kPermuteFineChunk) {
            e = launch_pdl(rank_scan_kernel, dim3((unsigned)nblk), dim3(kThreads), 0, s, (const int32_t *)topk_idx, R,
                           k, E, (const int32_t *)scratch, nblk, counts, offsets, row_to_token, token_to_row);
        } else {
            if (e == cudaSuccess)
                e = launch_pdl(scan_kernel, dim3(1), dim3(kThreads), 0, s, scratch, nblk, E, counts, offsets);
            if (e == cudaSuccess)
                e = launch_pdl(rank_kernel, dim3((unsigned)nblk), dim3(kThreads), 0, s, (const int32_t *)topk_idx, R,
                               k, E, (const int32_t *)scratch, row_to_token, token_to_row);
        }
        if (e != cudaSuccess) return e;
    }
    if (!x_perm) return cudaSuccess;  // dispatch only: the caller moves the rows itself
    return launch_scatter_rows(x, nullptr, token_to_row, N, k, H, x_perm, R, nullptr, s);
}

}  // namespace moe
