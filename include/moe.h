/*
 * moe.h -- C ABI of the B200 (sm_100a) MoE expert layer library, libmoe_b200.so.
 *
 * One MoE layer: router top-k, dispatch/permutation of token rows into
 * expert-contiguous groups, a SwiGLU FFN per expert as two grouped GEMMs
 * (W1/W3 with a fused SwiGLU epilogue, then W2) on the tcgen05 tensor cores,
 * optional always-on shared experts, and a deterministic weighted combine.
 *
 * Sources (web pages on the subject; cited by title and section):
 *  [MoE-latency] "MoE 少算 FLOPs,延迟反而涨了:慢在搬 token 的路上",
 *     sections "dense 和 MoE 的差别" (router, top-k, routing weights) and
 *     "router 之后还有一串动作" (assignments, dispatch, permutation, grouped
 *     GEMM, inverse mapping, weighting and summing = combine/unpermutation).
 *  [FinDEP] "FinDEP: Efficient MoE Inference with Fine-Grained Scheduling of
 *     Disaggregated Expert Parallelism", section "核心公式" (three GEMMs per
 *     expert) and section "问题定义" (shared experts).
 *
 * Conventions for every call:
 *  - bf16 tensors are passed as uint16_t storage (IEEE binary32's top half).
 *  - Row-major layouts.  Weights are [out, in] (nn.Linear layout), so both
 *    operands of every GEMM are K-contiguous.
 *  - Pointers are DEVICE pointers owned by the caller unless a call says
 *    otherwise; the library never frees them.  Every pointer a kernel reads
 *    with TMA (x, x_perm, weights, outputs of the GEMMs) must be 16-byte
 *    aligned; otherwise the call returns MOE_ERR_UNSUPPORTED.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls are asynchronous on it and launch nothing when argument
 *    checks fail.
 *  - Sizes: 1 <= E <= 256; 1 <= k <= min(E, 8); H and I multiples of 64
 *    (H, I <= 65536); N*k < 2^31.  N == 0 returns MOE_OK with no launch.
 *  - Device-side faults (an expert index outside [0,E) handed to
 *    moe_permute, a pipeline wait that timed out) never trap: the kernel
 *    skips the offending work and records a code in a per-device error word
 *    that moe_get_device_error() reads and clears.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* a size or pointer is out of the documented range */
    MOE_ERR_UNSUPPORTED = 2, /* a valid request this library does not handle (alignment, device) */
    MOE_ERR_WORKSPACE = 3,   /* workspace pointer NULL or smaller than moe_workspace_bytes() */
    MOE_ERR_CUDA = 4,        /* a CUDA runtime call failed; see moe_last_cuda_error() */
    MOE_ERR_DEVICE = 5       /* a kernel reported a device-side fault (moe_get_device_error) */
} moe_status_t;

/* Device error codes (moe_get_device_error). */
#define MOE_DEVERR_NONE 0
#define MOE_DEVERR_BAD_EXPERT_INDEX 1 /* moe_permute saw topk_idx outside [0,E) */
#define MOE_DEVERR_PIPELINE_TIMEOUT 2 /* a grouped-GEMM pipeline wait exceeded its limit */
#define MOE_DEVERR_BAD_OFFSETS 3      /* offsets not monotone or beyond R */

/* Text of a status code (static storage). */
MOE_API const char *moe_status_string(moe_status_t status);

/* Text of the last CUDA error seen by this thread's calls (static storage). */
MOE_API const char *moe_last_cuda_error(void);

/*
 * Bytes of device workspace moe_layer_forward_ex needs for this shape
 * (Is = total width of the shared experts, 0 for none).  Returns 0 on
 * invalid sizes.  The same number covers moe_permute and moe_expert_ffn.
 */
MOE_API size_t moe_workspace_bytes(int64_t N, int H, int I, int E, int k, int Is);

/*
 * Router ([MoE-latency] "dense 和 MoE 的差别"): score every expert, pick the
 * top k, give k routing weights.
 *   x         [N,H] bf16           token hidden states
 *   W_gate    [H,E] fp32           router weights
 *   bias      [E] fp32 or NULL     added to every logit (e.g. a load bias)
 *   logits    [N,E] fp32 or NULL   output: logit[t,e] = sum_h x[t,h] W_gate[h,e] (+ bias[e]),
 *                                  fp32 accumulation
 *   topk_idx  [N,k] int32          output: experts in pick order -- larger logit
 *                                  first, equal logits by lower expert index
 *   topk_w    [N,k] fp32           output: w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)
 *                                  over the k picks (softmax renormalised over the picks)
 *   ws, ws_bytes                   device scratch or NULL/0.  With at least
 *                                  moe_workspace_bytes(N,H,64,E,k,0) bytes, large batches
 *                                  compute the logits on the tensor cores (W_gate split
 *                                  into three bf16 terms, exact products, fp32
 *                                  accumulation) and small batches split H, the
 *                                  experts and the tokens over every SM (partial sums
 *                                  added in a fixed order); with NULL ws and a logits
 *                                  buffer the split runs without slices of H; with
 *                                  neither, a single fp32 CUDA-core kernel runs.
 * The logits are fp32-grade on every path; which path ran can change their last bits,
 * and the expert choice is taken on the logits this call produced.
 * NaN logits are unsupported input (the pick among them is unspecified).
 */
MOE_API moe_status_t moe_route(const uint16_t *x, const float *W_gate, const float *bias, int64_t N,
                       int H, int E, int k, float *logits, int32_t *topk_idx, float *topk_w,
                       void *ws, size_t ws_bytes, void *stream);

/*
 * Dispatch and permutation ([MoE-latency] "router 之后还有一串动作"): group
 * the N*k assignments by expert and copy token rows into expert-contiguous
 * order.  Deterministic and stable: within expert e, rows follow the
 * assignment id a = t*k + j.
 *   topk_idx      [N,k] int32      input
 *   counts        [E] int32        output: rows per expert
 *   offsets       [E+1] int32      output: exclusive scan of counts, offsets[E] = rows placed
 *   row_to_token  [N*k] int32      output: token of each permuted row
 *   token_to_row  [N,k] int32      output: permuted row of each assignment (-1 if the
 *                                  assignment's expert index was invalid)
 *   x_perm        [N*k,H] bf16     output: x_perm[r] = x[row_to_token[r]]
 *   ws, ws_bytes                   device scratch, >= moe_workspace_bytes(N,H,64,E,k,0)
 * An index outside [0,E) is skipped and sets MOE_DEVERR_BAD_EXPERT_INDEX.
 */
MOE_API moe_status_t moe_permute(const uint16_t *x, const int32_t *topk_idx, int64_t N, int H, int E,
                         int k, int32_t *counts, int32_t *offsets, int32_t *row_to_token,
                         int32_t *token_to_row, uint16_t *x_perm, void *ws, size_t ws_bytes,
                         void *stream);

/*
 * moe_permute for callers that cannot allocate device memory.  The pages
 * describe no such call; it exists for library users, not for the method.
 *
 * Some callers cannot call cudaMalloc at all or cannot hand out a workspace:
 * a serving process whose own pool has already claimed the device memory, a
 * plugin whose host framework owns every allocation, or code with a strict
 * latency budget (cudaMalloc may synchronise the device and has no time
 * bound).  This call takes the same inputs and outputs as moe_permute but no
 * workspace: its scratch (the per-block expert histograms of the dispatch)
 * lives in a fixed 1 MiB array inside the library, which every GPU that loads
 * the library holds until the process exits.  Nothing is allocated by the call.
 *
 * Limit: ceil(N*k / 1024) * E <= MOE_PERMUTE_NOALLOC_MAX_SCRATCH_INTS, i.e.
 * up to 1,048,576 assignments at E = 256 (more at smaller E).  Larger requests
 * return MOE_ERR_UNSUPPORTED before any launch.  (Below 32,768 assignments the
 * dispatch takes blocks of 256, at most 128 of them: always within the limit.)
 *
 * The first call on each device looks up the array's device address on that
 * device (the device must be current); make that first call before any stream
 * capture.  The address is looked up again whenever the calling thread's
 * current context differs from the one it was taken in (after a device reset,
 * or under a non-primary context); such a first call under a new context
 * should likewise come before any capture.  All calls share the one array: two calls whose kernels overlap on
 * the GPU (different streams, or host threads) race on it and must be ordered
 * by the caller.  The array keeps the previous call's contents; the dispatch
 * writes every entry it later reads, so no clearing is needed.
 */
#define MOE_PERMUTE_NOALLOC_MAX_SCRATCH_INTS 262144
MOE_API moe_status_t moe_permute_noalloc(const uint16_t *x, const int32_t *topk_idx, int64_t N, int H,
                                 int E, int k, int32_t *counts, int32_t *offsets,
                                 int32_t *row_to_token, int32_t *token_to_row, uint16_t *x_perm,
                                 void *stream);

/*
 * Expert FFN as two grouped GEMMs ([MoE-latency] "router 之后还有一串动作":
 * each expert runs its own matrix, merged into one launch; [FinDEP] "核心公式":
 * three GEMMs per expert).  For rows r in [offsets[e], offsets[e+1]):
 *   h[r]      = bf16( silu(x_perm[r] W1[e]^T) * (x_perm[r] W3[e]^T) )   fp32 accumulation,
 *               silu(z) = z / (1 + exp(-z))
 *   y_perm[r] = h[r] W2[e]^T                                           fp32 accumulation, fp32 out
 *   x_perm  [R,H] bf16; offsets [E+1] int32 (device; monotone, offsets[E] <= R)
 *   W1, W3  [E,I,H] bf16; W2 [E,H,I] bf16; y_perm [R,H] fp32 (rows beyond offsets[E] untouched)
 * h is the only rounding inside the FFN (bf16, the second GEMM's operand); y stays
 * fp32 so the combine rounds once.
 *   ws, ws_bytes: device scratch for h, >= moe_workspace_bytes(R,H,I,E,1,0)
 */
MOE_API moe_status_t moe_expert_ffn(const uint16_t *x_perm, const int32_t *offsets, const uint16_t *W1,
                            const uint16_t *W3, const uint16_t *W2, int64_t R, int H, int I,
                            int E, float *y_perm, void *ws, size_t ws_bytes, void *stream);

/*
 * Row scatter, the local reorder steps of expert parallelism ([MoE-latency] "跨 GPU
 * 时,激活要出门": rows received from other ranks are regrouped by local expert, and
 * the expert outputs are put back in the order they travel home in):
 *   dst[dst_row[i]] = src[i] for i in [0, rows) with 0 <= dst_row[i] < dst_rows (other
 *   target rows are skipped on the device)
 *   src [rows], dst [dst_rows]: rows of `width` 16-bit words (bf16 values, or fp32 values
 *   as word pairs: width = 2 * columns); width a multiple of 8; src, dst 16-byte aligned
 *   device pointers; dst_row [rows] int32 device, each target row written once (distinct
 *   rows; a repeated row is a race).  Asynchronous on `stream`.
 */
MOE_API moe_status_t moe_scatter_rows(const uint16_t *src, const int32_t *dst_row, int64_t rows, int width,
                                      uint16_t *dst, int64_t dst_rows, void *stream);

/*
 * Combine / unpermutation ([MoE-latency] "router 之后还有一串动作": inverse
 * mapping to token order, multiply by routing weight, add):
 *   out[t] = bf16( fma-chain over j = 0..k-1 of topk_w[t,j] * y_perm[token_to_row[t,j]]
 *                  (+ shared_out[t]) )   fp32, picks in order; rows < 0 are skipped
 *   y_perm [R,H] fp32; token_to_row [N,k] int32; topk_w [N,k] fp32;
 *   shared_out [N,H] fp32 or NULL; out [N,H] bf16 (the only rounding of the sum).
 */
MOE_API moe_status_t moe_combine(const float *y_perm, const int32_t *token_to_row,
                         const float *topk_w, const float *shared_out, int64_t N, int H, int k,
                         uint16_t *out, void *stream);

/*
 * The whole layer, short form: route -> permute -> expert FFN -> combine,
 * no bias, no shared experts, on the legacy default stream, with a
 * library-owned workspace that grows on demand (not thread-safe).
 *   x [N,H] bf16 and out [N,H] bf16 may be HOST or DEVICE pointers: host
 *   buffers are copied in and out by the call (which then returns only after
 *   out is written).  W_gate [H,E] fp32, W1, W3 [E,I,H] and W2 [E,H,I] bf16
 *   must be device pointers (weights stay resident).
 */
MOE_API moe_status_t moe_layer_forward(const uint16_t *x, const float *W_gate, const uint16_t *W1,
                               const uint16_t *W3, const uint16_t *W2, int64_t N, int H, int I,
                               int E, int k, uint16_t *out);

/*
 * The whole layer, explicit form: everything on `stream`, caller's workspace,
 * no allocation.  All pointers are device pointers.
 *   bias [E] fp32 or NULL; Ws1, Ws3 [Is,H], Ws2 [H,Is] bf16 = shared experts
 *   ([FinDEP] "问题定义"), their widths concatenated into Is (0 = none, then the
 *   three pointers are ignored); their output is added with weight 1 after
 *   the routed sum.  logits [N,E] fp32 is an optional output (NULL = keep it
 *   in the workspace).
 *   phase_events: NULL, or an array of MOE_NUM_PHASES + 1 cudaEvent_t (as
 *   void*) recorded on `stream` before the first and after each phase, for
 *   per-kernel timing.
 */
#define MOE_PHASE_ROUTE 0
#define MOE_PHASE_PERMUTE 1
#define MOE_PHASE_GEMM13 2
#define MOE_PHASE_GEMM2 3
#define MOE_PHASE_SHARED 4
#define MOE_PHASE_COMBINE 5
#define MOE_NUM_PHASES 6
MOE_API moe_status_t moe_layer_forward_ex(const uint16_t *x, const float *W_gate, const float *bias,
                                  const uint16_t *W1, const uint16_t *W3, const uint16_t *W2,
                                  const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2,
                                  int64_t N, int H, int I, int E, int k, int Is, uint16_t *out,
                                  float *logits, void *ws, size_t ws_bytes, void *stream,
                                  void *const *phase_events);

/*
 * FP8 expert weights ([MoE-latency] "优化从测量开始": quantizing the weights cuts
 * memory bytes; its numerical error is measured as an experiment of its own).
 * The pages fix no format; this library uses OCP e4m3 bytes (largest finite 448)
 * with one fp32 scale per output channel (weight row), and the weight a GEMM uses
 * is e4m3(q) * scale.  Activations, routing, combine and shared experts stay as in
 * the bf16 calls.
 *
 * moe_quantize_fp8: W [rows,K] bf16 -> q [rows,K] e4m3 bytes and scale [rows] fp32:
 *   scale[r] = max_c |W[r,c]| / 448 (fp32, correctly rounded; 1 for an all-zero row),
 *   q[r,c] = e4m3(W[r,c] / scale[r]) (fp32 quotient; nearest, ties to even; saturating).
 *   Run once per weight set (W1 and W3 as [E*I, H], W2 as [E*H, I]).  K a multiple
 *   of 64; W, q, scale 16-byte aligned device pointers.  Asynchronous on `stream`.
 */
MOE_API moe_status_t moe_quantize_fp8(const uint16_t *W, int64_t rows, int K, uint8_t *q, float *scale,
                                      void *stream);

/*
 * moe_expert_ffn with e4m3 weights: W1q, W3q [E,I,H] and W2q [E,H,I] bytes, scales
 * s1, s3 [E,I] and s2 [E,H] fp32 (from moe_quantize_fp8).  The grouped GEMMs stream
 * the bytes and widen them to bf16 on chip; the products accumulate in fp32 and each
 * output channel is multiplied by its scale before SwiGLU (W1/W3) or before the store
 * (W2).  Other arguments, layouts and errors as moe_expert_ffn.
 */
MOE_API moe_status_t moe_expert_ffn_fp8(const uint16_t *x_perm, const int32_t *offsets, const uint8_t *W1q,
                                        const float *s1, const uint8_t *W3q, const float *s3,
                                        const uint8_t *W2q, const float *s2, int64_t R, int H, int I, int E,
                                        float *y_perm, void *ws, size_t ws_bytes, void *stream);

/*
 * moe_layer_forward_ex with e4m3 routed-expert weights and their scales (as in
 * moe_expert_ffn_fp8); the shared experts, when Is > 0, stay bf16.  Same workspace
 * (moe_workspace_bytes), stream, phase events and errors as moe_layer_forward_ex.
 */
MOE_API moe_status_t moe_layer_forward_fp8_ex(const uint16_t *x, const float *W_gate, const float *bias,
                                              const uint8_t *W1q, const float *s1, const uint8_t *W3q,
                                              const float *s3, const uint8_t *W2q, const float *s2,
                                              const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2,
                                              int64_t N, int H, int I, int E, int k, int Is, uint16_t *out,
                                              float *logits, void *ws, size_t ws_bytes, void *stream,
                                              void *const *phase_events);

/*
 * FP8 weights and FP8 activations (the same section names activations beside the
 * weights).  On top of the e4m3 weights above, every activation row the two routed
 * GEMMs read is quantized per row exactly as moe_quantize_fp8 does: the permuted
 * token rows x_perm [R,H] before W1/W3, and the SwiGLU output h [R,I] after its
 * bf16 rounding, before W2.  Both GEMMs then multiply e4m3 by e4m3 on the tensor
 * cores (tcgen05 kind::f8f6f4, fp32 accumulation of exact products) and each
 * output is multiplied by its weight row's scale and its token row's scale.
 * Routing, combine and the shared experts stay as in the bf16 calls.
 *
 * moe_expert_ffn_w8a8: arguments, layouts and errors as moe_expert_ffn_fp8, plus
 *   h        nullable device bf16 [R,I]: receives h (before its quantization);
 *   ws       >= moe_expert_ffn_w8a8_ws_bytes(R,H,I) bytes (quantized rows, scales
 *            and, when h is NULL, h itself).
 */
MOE_API size_t moe_expert_ffn_w8a8_ws_bytes(int64_t R, int H, int I);
MOE_API moe_status_t moe_expert_ffn_w8a8(const uint16_t *x_perm, const int32_t *offsets, const uint8_t *W1q,
                                         const float *s1, const uint8_t *W3q, const float *s3,
                                         const uint8_t *W2q, const float *s2, int64_t R, int H, int I, int E,
                                         float *y_perm, uint16_t *h, void *ws, size_t ws_bytes, void *stream);

/*
 * moe_layer_forward_fp8_ex with the activations quantized as well.  Workspace:
 * moe_workspace_bytes_w8a8(N,H,I,E,k,Is) bytes (moe_workspace_bytes plus the
 * quantized rows and their scales).  The x quantization is timed in the permute
 * phase, the h quantization in the W1/W3 phase.  Other arguments and errors as
 * moe_layer_forward_fp8_ex.
 */
MOE_API size_t moe_workspace_bytes_w8a8(int64_t N, int H, int I, int E, int k, int Is);
MOE_API moe_status_t moe_layer_forward_w8a8_ex(const uint16_t *x, const float *W_gate, const float *bias,
                                               const uint8_t *W1q, const float *s1, const uint8_t *W3q,
                                               const float *s3, const uint8_t *W2q, const float *s2,
                                               const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2,
                                               int64_t N, int H, int I, int E, int k, int Is, uint16_t *out,
                                               float *logits, void *ws, size_t ws_bytes, void *stream,
                                               void *const *phase_events);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device.  *code receives a MOE_DEVERR_* value.  Returns MOE_OK, or
 * MOE_ERR_CUDA if the synchronisation itself failed.
 */
MOE_API moe_status_t moe_get_device_error(void *stream, int32_t *code);

/* Number of streaming multiprocessors the grouped GEMM sizes its persistent grid to. */
MOE_API int moe_device_sm_count(void);

/*
 * Buffers shared between processes, and device-to-device copies, for the
 * expert-parallel layer's own row exchange ([MoE-latency] "跨 GPU 时,激活要出门":
 * a token whose expert lives on another GPU sends its activation row there and
 * gets the expert's output back).  A rank exports its receive buffers once; the
 * other ranks import them and copy rows straight into them, one copy per
 * contiguous range.  Nothing here waits on another process: the caller orders the
 * ranks (each rank's copies complete, then a host-side barrier).
 *
 * moe_ipc_export: ptr, a device pointer inside an allocation made by cudaMalloc
 *   (the caching allocator of PyTorch makes such allocations) -> handle, the
 *   allocation's IPC handle (MOE_IPC_HANDLE_BYTES bytes, caller-owned), and offset,
 *   the byte offset of ptr inside it.  MOE_ERR_UNSUPPORTED for memory the IPC API
 *   cannot share (e.g. virtual-memory mappings).
 * moe_ipc_import: (handle, offset) from another process on the same node -> *ptr,
 *   this process's pointer to the same bytes (valid until moe_ipc_close).  A handle
 *   cannot be imported by the process that exported it.  MOE_ERR_CUDA on failure.
 * moe_ipc_close: releases an imported mapping (ptr and offset as imported).
 * moe_copy_async: bytes from src to dst, both device pointers (either may be an
 *   imported peer pointer), asynchronous on stream.
 */
#define MOE_IPC_HANDLE_BYTES 64
MOE_API moe_status_t moe_ipc_export(const void *ptr, void *handle, size_t *offset);
MOE_API moe_status_t moe_ipc_import(const void *handle, size_t offset, void **ptr);
MOE_API moe_status_t moe_ipc_close(void *ptr, size_t offset);
MOE_API moe_status_t moe_copy_async(void *dst, const void *src, size_t bytes, void *stream);

/*
 * How the bf16 layer calls (moe_layer_forward, moe_layer_forward_ex) feed the
 * W1/W3 GEMM its token rows.  The pages' dispatch copies every assignment's row
 * into expert order ([MoE-latency] "router 之后还有一串动作": the permutation, and
 * the cost of moving token rows it names); with gathering on, the dispatch only
 * builds the row maps and the GEMM loads each row straight from x through
 * row_to_token (tile::gather4 TMA), so the permuted copy x_perm is never written.
 * The results are identical either way.
 *   mode  MOE_GATHER_AUTO (the default: the library chooses; measured on B200,
 *         gathering was slower on every workload shape, so it picks the copy),
 *         MOE_GATHER_OFF (always the permuted copy), MOE_GATHER_ON (always gather).
 * Process-wide; takes effect for calls enqueued after it returns.  Returns the
 * previous mode, or -1 for a mode outside these three.
 */
#define MOE_GATHER_AUTO 0
#define MOE_GATHER_OFF 1
#define MOE_GATHER_ON 2
MOE_API int moe_set_gather_mode(int mode);

/*
 * Micro-batches of the layer calls (moe_layer_forward_ex and its fp8 forms) on
 * batches of at least 32768 assignments (N*k).  With m = 2 the batch runs as two
 * halves: rows [0, N0) on the caller's stream, rows [N0, N) on a second stream of
 * the library's that starts once the first half has dispatched, joined back
 * before the call's work ends on the caller's stream.  The first half's grouped
 * GEMMs then run beside the second half's router, dispatch and row copies, and
 * the second half's GEMMs beside the first half's combine (MegaScale-Infer
 * summary page, "核心设计": splitting a batch into micro-batches so that one
 * micro-batch's work hides another's; here the hidden work is the token-row
 * movement the MoE-latency article's section "router 之后还有一串动作" names).
 * Results are identical to m = 1 (every token's arithmetic is unchanged).  The
 * first such call on a device creates the stream and two events (kept for the
 * process); it should come before any stream capture.  A call with phase events
 * runs in one piece.  m = 1 (the default) or 2; returns the previous value, or -1.
 * Process-wide, like moe_set_gather_mode.
 */
MOE_API int moe_set_microbatches(int m);

/*
 * Where the layer calls run the always-on shared experts ([FinDEP] "问题定义").
 * on = 1 (the default): on a second stream of the library's, forked at the start of
 * the call and joined before the combine, so the router, the dispatch and the row
 * copies of the routed experts run beside the shared experts' GEMMs (measured 5%
 * faster at the DeepSeek-V2 shape); on = 0: on the caller's stream after the routed
 * experts.  Same
 * results either way.  The first call with shared experts on a device creates the
 * stream (and two events) for the process; make it before any stream capture.  A
 * call with phase events runs on the caller's stream.  Process-wide; returns the
 * previous value, or -1.
 */
MOE_API int moe_set_shared_stream(int on);

/*
 * How the bf16 layer calls (moe_layer_forward_ex, moe_layer_forward) run the routed
 * experts' FFN for decode batches (MoE-latency article, section "router 之后还有一串
 * 动作": at decode, launches, weight reads and row moves are the cost).  With a few
 * tokens every expert GEMM is a GEMV: after the router's partial logits, two CUDA-core
 * kernels deal the picked experts' weight rows evenly over all SMs -- W1/W3 with the
 * SwiGLU, per pick (each block first finishes the top-k itself; no dispatch, no row
 * copies), then W2 with the combine folded in (each token's k products added in pick
 * order in registers, no fp32 expert outputs in memory) -- instead of the top-k and
 * dispatch kernel, the tensor-core grouped GEMMs and the combine kernel: three
 * launches in all.  The picks, weights and logits are the other paths' bits.
 * Deterministic; the bits differ from the tensor-core path's (another summation order
 * inside each dot product), within the same fp32 accuracy.
 * It takes batches of at most MOE_DECODE_MAX_TOKENS tokens and MOE_DECODE_MAX_ROWS
 * assignments.
 *   mode  MOE_DECODE_AUTO (the default: for 2*N*k <= E, at most half an assignment
 *         per expert on average, H <= 2048 and I <= 1024 -- where it measured
 *         faster: the Qwen3-30B shape at 1, 2, 4 and 8 tokens, 28 / 41 / 67 / 111 us
 *         against 43 / 62 / 86 / 118 us through the grouped GEMMs; not with
 *         DeepSeek-V2's longer rows),
 *         MOE_DECODE_OFF (always the grouped GEMMs), MOE_DECODE_ON (whenever the
 *         batch is within those limits).
 * fp8 layers always use the grouped GEMMs.  Process-wide; returns the previous mode,
 * or -1 for a mode outside these three.
 */
#define MOE_DECODE_AUTO 0
#define MOE_DECODE_OFF 1
#define MOE_DECODE_ON 2
#define MOE_DECODE_MAX_ROWS 512  /* N*k */
#define MOE_DECODE_MAX_TOKENS 64 /* N: every block of the first kernel ranks the batch */
MOE_API int moe_set_decode_gemv(int mode);

/*
 * Kernels this library has launched in this process so far, counted on the host
 * at each successful launch (all threads, all devices; never reset).  The
 * difference across a region is the number of the library's kernels it ran.
 */
MOE_API uint64_t moe_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
