// dispatch_block.cuh -- the stable dispatch of a batch of assignments by one block of
// 256 threads: per-expert histogram, exclusive scan, stable ranks.
//
// MoE-latency article, section "router 之后还有一串动作": the N*k assignments are
// grouped by expert (dispatch) and the rows sorted by expert (permutation).  Stable:
// assignment a = t*k + j of expert e goes to row offsets[e] + #{a' < a : e(a') = e}.
// No atomics decide the row order (warp match + per-warp counts, warps in order).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kDispThreads = 256;
constexpr int kDispWarps = kDispThreads / 32;
constexpr int kDispMaxE = 256;

// Shared memory of one block's dispatch.
struct DispatchSmem {
    int base[kDispMaxE];
    int scan[kDispThreads];
    int wcnt[kDispWarps][kDispMaxE];
};

// One round of the stable rank: kDispThreads consecutive assignments starting at a0,
// placed after base[e] rows of their expert; advances base.  Block-wide.
// row_to_token may be null (only token_to_row is then written).
__device__ __forceinline__ void rank_round(const int32_t *idx, int64_t R, int k, int E, int64_t a0, int *base,
                                           int (*wcnt)[kDispMaxE], int32_t *row_to_token, int32_t *token_to_row)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int i = threadIdx.x; i < kDispWarps * E; i += kDispThreads) wcnt[i / E][i % E] = 0;
    __syncthreads();
    const int64_t a = a0 + threadIdx.x;
    int e = -1;
    if (a < R) e = idx[a];
    const bool valid = a < R && e >= 0 && e < E;
    // lanes with equal keys form one group; invalid lanes get a key of their own
    const int key = valid ? e : (kDispMaxE + lane);
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int rank_in_warp = __popc(peers & lt_mask);
    if (valid && rank_in_warp == 0) wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (a < R) {
        if (valid) {
            int before = 0;
            for (int w = 0; w < warp; ++w) before += wcnt[w][e];
            const int row = base[e] + before + rank_in_warp;
            if (row_to_token) row_to_token[row] = (int32_t)(a / k);
            token_to_row[a] = row;
        } else {
            token_to_row[a] = -1;
        }
    }
    __syncthreads();
    for (int ee = threadIdx.x; ee < E; ee += kDispThreads) {
        int add = 0;
        for (int w = 0; w < kDispWarps; ++w) add += wcnt[w][ee];
        base[ee] += add;
    }
    __syncthreads();
}

// Histogram, exclusive scan and stable ranks of all R assignments in one block.
// counts, offsets and row_to_token may be null (not written); token_to_row is always
// written (global or shared memory).  An index outside [0,E) is skipped and reported.
__device__ __forceinline__ void dispatch_block(const int32_t *idx, int64_t R, int k, int E, int32_t *counts,
                                               int32_t *offsets, int32_t *row_to_token, int32_t *token_to_row,
                                               int *err, DispatchSmem &sm)
{
    const int tid = threadIdx.x;
    if (tid < E) sm.base[tid] = 0;
    __syncthreads();
    for (int64_t a = tid; a < R; a += kDispThreads) {
        const int e = idx[a];
        if (e >= 0 && e < E) atomicAdd(&sm.base[e], 1);
        else set_device_error(err, MOE_DEVERR_BAD_EXPERT_INDEX);
    }
    __syncthreads();
    const int c = tid < E ? sm.base[tid] : 0;
    sm.scan[tid] = c;
    __syncthreads();
    for (int o = 1; o < kDispThreads; o <<= 1) {  // inclusive scan
        const int v = tid >= o ? sm.scan[tid - o] : 0;
        __syncthreads();
        sm.scan[tid] += v;
        __syncthreads();
    }
    if (tid < E) {
        if (counts) counts[tid] = c;
        if (offsets) {
            offsets[tid] = sm.scan[tid] - c;
            if (tid == E - 1) offsets[E] = sm.scan[tid];
        }
        sm.base[tid] = sm.scan[tid] - c;
    }
    __syncthreads();
    for (int64_t a0 = 0; a0 < R; a0 += kDispThreads)
        rank_round(idx, R, k, E, a0, sm.base, sm.wcnt, row_to_token, token_to_row);
}

}  // namespace moe
