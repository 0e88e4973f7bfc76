// internal.h -- host-side launch interfaces between the kernel files and the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

// Host-side count of kernels this library launched (every launch goes through
// launch_pdl or the grouped GEMM's launcher, which call this on success).
void count_launch();
uint64_t launches_so_far();

// The calling thread's current CUDA context (a driver handle), or nullptr when none
// is bound.  Caches of per-device addresses are keyed on it: after cudaDeviceReset, or
// under another context on the same device, a cached address would be stale.
void *current_context();

// Micro-batches of large layers (moe_set_microbatches): 1 or 2.
int layer_microbatches();
// Whether the shared experts run on a second stream beside the dispatch (moe_set_shared_stream).
bool layer_shared_side();

// Whether the bf16 layer gathers its W1/W3 token rows from x (moe_set_gather_mode).
bool layer_gathers(int64_t N, int k, int H);

// Launch with programmatic stream serialization (the kernel calls pdl_entry/pdl_wait
// before its first global memory access).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
    if (e == cudaSuccess) count_launch();
    return e;
}

// Router: logits (fp32), top-k indices and renormalised weights.  `ws` (nullable)
// of at least router_ws_bytes(N, H, E) bytes enables the tensor-core path and
// the split path's slices of H; a logits buffer alone enables the split path.
enum class RouterPath { kFused, kSplit, kTensor };
RouterPath router_path(int64_t N, int E, bool have_logits_buffer, bool have_ws);
size_t router_ws_bytes(int64_t N, int H, int E);
cudaError_t launch_router(const uint16_t *x, const float *W_gate, const float *bias, int64_t N,
                          int H, int E, int k, float *logits, int32_t *topk_idx, float *topk_w,
                          void *ws, size_t ws_bytes, int *dev_err, cudaStream_t s);

// Router, dispatch and row scatter of a small batch (N*k <= 512) in two kernels: the
// router's logits (or its one-kernel form with the picks), then top-k, the stable
// dispatch and the rows in one.  Same outputs as launch_router followed by
// launch_permute.  cudaErrorNotSupported (nothing launched) for other shapes.
cudaError_t launch_route_dispatch_small(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H,
                                        int E, int k, float *logits, int32_t *topk_idx, float *topk_w, void *ws,
                                        size_t ws_bytes, int32_t *counts, int32_t *offsets, int32_t *row_to_token,
                                        int32_t *token_to_row, uint16_t *x_perm, int *dev_err, cudaStream_t s);

// Dispatch / permutation.  `scratch` holds permute_scratch_ints(R, E) ints.  The count and
// rank passes take blocks of permute_chunk(R) assignments: kPermuteFineChunk below
// kPermuteFineMaxR assignments (more blocks for mid-sized batches; their rank blocks fold
// the scan in), kPermuteChunk from there on (the scan kernel then leaves every block's
// starting row per expert in the scratch).
constexpr int kPermuteChunk = 1024;
constexpr int kPermuteFineChunk = 256;
constexpr int64_t kPermuteFineMaxR = 32768;
inline int64_t permute_chunk(int64_t R) { return R < kPermuteFineMaxR ? kPermuteFineChunk : kPermuteChunk; }
inline int64_t permute_blocks(int64_t R) { return (R + permute_chunk(R) - 1) / permute_chunk(R); }
inline int64_t permute_scratch_ints(int64_t R, int E) { return permute_blocks(R) * E; }
// x_perm == nullptr: dispatch only (counts, offsets, the two row maps), no row copy.
cudaError_t launch_permute(const uint16_t *x, const int32_t *topk_idx, int64_t N, int H, int E,
                           int k, int32_t *counts, int32_t *offsets, int32_t *row_to_token,
                           int32_t *token_to_row, uint16_t *x_perm, int32_t *scratch,
                           int *dev_err, cudaStream_t s);
// x_perm[token_to_row[t,j]] = x[t]: rows of H 16-bit words (H a multiple of 8; e4m3
// rows of 2H bytes pass as H words); with scale_in, scale_out[token_to_row[t,j]] = scale_in[t].
// Target rows outside [0, out_rows) are skipped.
cudaError_t launch_scatter_rows(const uint16_t *x, const float *scale_in, const int32_t *token_to_row, int64_t N,
                                int k, int H, uint16_t *x_perm, int64_t out_rows, float *scale_out, cudaStream_t s);

// Grouped GEMMs on tcgen05.  Weights are [groups, Nout, K]; activations [R, K];
// rows of group g are offsets[g] .. offsets[g+1]-1 (offsets == nullptr: one group
// of `rows_single` rows starting at row 0).
struct GroupedGemmArgs {
    const void *act;         // [R, K] bf16, or e4m3 bytes when a8
    const void *w_a;         // [groups, Nout, K] bf16, or e4m3 bytes when w8 (W1, or W2)
    const void *w_b;         // [groups, Nout, K] likewise (W3) -- SwiGLU only
    bool w8;                 // weights are e4m3 with one fp32 scale per row (scale_a, scale_b)
    const float *scale_a;    // [groups, Nout] row scales of w_a (w8 only)
    const float *scale_b;    // [groups, Nout] row scales of w_b (w8, SwiGLU only)
    bool a8;                 // activations are e4m3 too (needs w8): native fp8 MMA
    const float *scale_act;  // [R] row scales of act (a8 only)
    const int32_t *offsets;  // [groups + 1] device, or nullptr
    const int32_t *ends;     // [groups] device, or nullptr: group g is rows [offsets[g], ends[g])
                             // instead of [offsets[g], offsets[g + 1])
    int groups;
    int64_t R;               // rows of `act` (and of `out`)
    int rows_single;         // rows when offsets == nullptr
    int K;
    int Nout;
    void *out;               // [R, Nout] (row stride ldo): bf16 (SwiGLU GEMM) or fp32 (W2 GEMM)
    int *dev_err;
    int token_tile;          // 0 = choose from the shape
    int ksplit;              // plain GEMM: K slices (0/1 = none); partial sums at out + s*split_stride
    int64_t split_stride;    // elements between the partial-sum buffers
    int64_t ldo;             // plain GEMM: elements between output rows (0 = Nout)
    bool single_cta;         // plain bf16 GEMM: single-CTA tiles (token_tile 32, 64 or 128)
    const int32_t *gather_rows;  // bf16 SwiGLU GEMM: nullptr, or act is x [gather_src_rows, K] and row r
                                 // of the groups reads x row gather_rows[r] (no permuted copy)
    int64_t gather_src_rows;
};
cudaError_t launch_gemm13_swiglu(const GroupedGemmArgs &a, cudaStream_t s);
cudaError_t launch_gemm2(const GroupedGemmArgs &a, cudaStream_t s);
int gemm_choose_token_tile(int64_t R, int groups, bool swiglu);
int gemm2_ksplit(int64_t R, int groups, int K, int Nout);
int device_sm_count();

// e4m3 weights with one fp32 scale per row: q [rows, K] bytes, scale [rows].
cudaError_t launch_quantize_fp8(const uint16_t *W, int64_t rows, int K, uint8_t *q, float *scale, cudaStream_t s);

// The router's partial logits of a decode batch, for the first decode kernel to rank:
// part [P][N][E] (pstride = N*E), summed in slice order (+ bias when bias is given;
// written to logits when given).  P = 0: the picks are already in topk_idx/topk_w.
struct RouterPartials {
    const float *part;
    int P;
    int64_t pstride;
    const float *bias;
    float *logits;
};
cudaError_t launch_router_partials(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E,
                                   int k, float *logits, int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                                   RouterPartials *rp, cudaStream_t s);

// The expert FFN of a decode batch on CUDA cores (a few tokens): W1/W3 with the SwiGLU
// over (pick, feature) units -- its blocks finish the router's top-k from the partial
// logits first, and block 0 writes the picks and weights -- h [N*k, I] in pick order
// (row t*k + j); then W2 with the combine folded in (out written, no fp32 expert outputs).
cudaError_t launch_decode_w13(const uint16_t *x, const RouterPartials &rp, int32_t *topk_idx, float *topk_w,
                              int64_t N, int k, int E, int H, int I, const uint16_t *W1, const uint16_t *W3,
                              uint16_t *h, int *err, cudaStream_t s);
cudaError_t launch_decode_w2_combine(const uint16_t *h, const int32_t *topk_idx, const float *topk_w,
                                     const float *shared_out, int64_t N, int E, int H, int I, int k,
                                     const uint16_t *W2, uint16_t *out, int *err, cudaStream_t s);
// Whether the layer runs its expert FFN with the kernels above (moe_set_decode_gemv).
bool layer_decode_gemv(int64_t N, int k, int E, int H, int I);

// Combine / unpermutation.
// y_perm holds `nsplit` partial-sum buffers `split_stride` elements apart (1 = one).
cudaError_t launch_combine(const float *y_perm, int nsplit, int64_t split_stride,
                           const int32_t *token_to_row, const float *topk_w, const float *shared_out,
                           int64_t N, int H, int k, uint16_t *out, cudaStream_t s);

}  // namespace moe
