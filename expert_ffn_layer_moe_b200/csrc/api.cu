// api.cu -- the C ABI (include/moe.h): argument checks, workspace layout, launch order.
//
// Every entry point validates its arguments on the host and launches nothing when a
// check fails.  Kernels report device-side faults through one error word per device
// (read and cleared by moe_get_device_error), never by trapping.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {
namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_gather_mode{MOE_GATHER_AUTO};
std::atomic<int> g_microbatches{1};
std::atomic<int> g_shared_side{1};
std::atomic<int> g_decode_gemv{MOE_DECODE_AUTO};
}  // namespace
int layer_microbatches() { return g_microbatches.load(std::memory_order_relaxed); }
bool layer_shared_side() { return g_shared_side.load(std::memory_order_relaxed) != 0; }
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
uint64_t launches_so_far() { return g_launches.load(std::memory_order_relaxed); }

// Whether the bf16 layer gathers its W1/W3 token rows from x (no permuted copy).  By
// default it does not: each tile::gather4 request (four 128-byte rows) costs the TMA unit
// about 85 cycles on B200, so a prefill-sized token tile (128 rows per CTA per K step)
// takes about 2,700 cycles to gather against about 500 for the MMAs it feeds -- W1/W3
// ran 3x slower gathered than from the permuted copy on every workload shape measured,
// more than the copy it saves.
bool layer_gathers(int64_t N, int k, int H)
{
    const int mode = g_gather_mode.load(std::memory_order_relaxed);
    if (mode == MOE_GATHER_ON) return true;
    (void)N; (void)k; (void)H;
    return false;
}

// Whether the bf16 layer runs its expert FFN as the decode GEMV kernels.  By default for
// batches of at most half an assignment per expert on average (2 N*k <= E), with
// H <= 2048 and I <= 1024, where the grouped GEMM's tiles leave SMs idle and pay their
// pipeline's setup for a token or two.  Measured (graph replay) at the Qwen3-30B shape
// (H = 2048, I = 768, E = 128, top-8): N = 1, 2, 4, 8 took 28 / 41 / 67 / 111 us against
// 43 / 62 / 86 / 118 us through the grouped GEMMs.  At the DeepSeek-V2 shape (H = 5120,
// I = 1536) an earlier form lost at N = 4 (283 against 237 us): a GEMV lane holds its
// loads in flight in registers, and longer rows need more rounds of them, where the
// grouped GEMM keeps 200 KB in flight in shared memory.
bool layer_decode_gemv(int64_t N, int k, int E, int H, int I)
{
    const int mode = g_decode_gemv.load(std::memory_order_relaxed);
    const int64_t R = N * k;
    if (mode == MOE_DECODE_OFF || R > MOE_DECODE_MAX_ROWS || N > MOE_DECODE_MAX_TOKENS) return false;
    if (mode == MOE_DECODE_ON) return true;
    return 2 * R <= (int64_t)E && H <= 2048 && I <= 1024;
}

void *current_context()
{
    using GetCurrent = int (*)(void **);
    static GetCurrent fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<GetCurrent>(p);
    }();
    void *ctx = nullptr;
    if (!fn || fn(&ctx) != 0) return nullptr;
    return ctx;
}
}  // namespace moe

namespace {

__device__ int g_moe_device_error;  // per device: first MOE_DEVERR_* code since the last read

thread_local char g_last_cuda_error[256] = "no error";

moe_status_t cuda_fail(cudaError_t e)
{
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

#define MOE_CUDA(call)                                   \
    do {                                                 \
        cudaError_t e_ = (call);                         \
        if (e_ != cudaSuccess) return cuda_fail(e_);     \
    } while (0)

// Device address of the error word on the current device (host code must not use
// the symbol itself as a pointer).  Cached per device and looked up again when the
// thread's current context is not the one the address was taken in.
int *device_error_word()
{
    static std::mutex mu;
    static int *addr[64] = {nullptr};
    static void *ctx_of[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    void *ctx = moe::current_context();
    if (!addr[dev] || !ctx || ctx != ctx_of[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_moe_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<int *>(p);
        ctx_of[dev] = moe::current_context();  // bound now, if the lookup initialised it
    }
    return addr[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_hidden(int v) { return v >= 64 && v <= 65536 && v % 64 == 0; }

bool valid_ek(int E, int k) { return E >= 1 && E <= 256 && k >= 1 && k <= 8 && k <= E; }

// N * k < 2^31, checked without forming a product that could overflow
bool valid_rows(int64_t N, int k) { return k >= 1 && N >= 0 && N < ((int64_t(1) << 31) + k - 1) / k; }

size_t round_up(size_t v) { return (v + 255) & ~size_t(255); }

struct WsLayout {
    size_t logits, idx, w, counts, offsets, r2t, t2r, perm, x_perm, h, hs, y_perm, s, router, router_bytes;
    size_t xqt, xst, xq, xsc, hq, hsc;  // fp8 activations only: quantized rows and their scales
    size_t total;
};

// Carve the layer's workspace; every buffer starts on a 256-byte boundary.  a8 adds
// the quantized activation rows.
void ws_layout(int64_t N, int H, int I, int E, int k, int Is, bool a8, WsLayout *L)
{
    const int64_t R = N * k;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off += round_up(bytes ? bytes : 1); return at; };
    L->logits = take((size_t)N * E * 4);
    L->idx = take((size_t)R * 4);
    L->w = take((size_t)R * 4);
    L->counts = take((size_t)E * 4);
    L->offsets = take((size_t)(E + 1) * 4);
    L->r2t = take((size_t)R * 4);
    L->t2r = take((size_t)R * 4);
    L->perm = take((size_t)moe::permute_scratch_ints(R, E) * 4);
    L->x_perm = take((size_t)R * H * 2);
    L->h = take((size_t)R * I * 2);
    L->hs = take((size_t)N * (Is > 0 ? Is : 0) * 2);
    L->y_perm = take((size_t)moe::gemm2_ksplit(R, E, I, H) * R * H * 4);  // one buffer per K slice
    L->s = take((size_t)N * (Is > 0 ? H : 0) * 4);
    L->router_bytes = moe::router_ws_bytes(N, H, E);
    L->router = take(L->router_bytes);
    L->xqt = take(a8 ? (size_t)N * H : 0);  // token order
    L->xst = take(a8 ? (size_t)N * 4 : 0);
    L->xq = take(a8 ? (size_t)R * H : 0);
    L->xsc = take(a8 ? (size_t)R * 4 : 0);
    L->hq = take(a8 ? (size_t)R * I : 0);
    L->hsc = take(a8 ? (size_t)R * 4 : 0);
    L->total = off;
}

// Tokens of the first half when the layer runs its expert GEMMs as two micro-batches (0:
// in one piece): batches of at least kMicroMinRows assignments, when moe_set_microbatches
// asked for 2.  The first half ends on a block of the dispatch (N0 * k a multiple of
// kPermuteChunk), whose per-block table then holds where the second half's rows of every
// expert start.
constexpr int64_t kMicroMinRows = 32768;
static_assert(kMicroMinRows >= moe::kPermuteFineMaxR, "the dispatch of such batches runs blocks of kPermuteChunk");
int64_t micro_split(int64_t N, int k)
{
    if (moe::layer_microbatches() < 2 || N * k < kMicroMinRows) return 0;
    int64_t g = moe::kPermuteChunk, kk = k;  // step = kPermuteChunk / gcd(k, kPermuteChunk) tokens
    while (kk) { const int64_t r = g % kk; g = kk; kk = r; }
    const int64_t step = moe::kPermuteChunk / g;
    const int64_t N0 = (N / 2) / step * step;
    return (N0 > 0 && N0 < N) ? N0 : 0;
}

size_t layer_ws_bytes(int64_t N, int H, int I, int E, int k, int Is, bool a8)
{
    WsLayout L;
    ws_layout(N, H, I, E, k, Is, a8, &L);
    return L.total;
}

// The routed experts' weights: bf16, or e4m3 bytes with one fp32 scale per row
// (optionally with e4m3 activations as well).
struct Experts {
    const void *W1, *W3, *W2;
    const float *s1, *s3, *s2;  // fp8 only
    bool fp8;
    bool a8;                    // activations quantized too (fp8 weights only)
};

// Buffers of the quantized activation rows (a8 only): x_perm and h, with their scales
// (the layer also quantizes x in token order first: xqt, xst).
struct ActQ {
    uint8_t *xq; float *xsc; uint8_t *hq; float *hsc; uint8_t *xqt; float *xst;
};

void set_weights13(moe::GroupedGemmArgs *a, const Experts &X)
{
    a->w_a = X.W1; a->w_b = X.W3; a->w8 = X.fp8; a->scale_a = X.s1; a->scale_b = X.s3;
}

void set_weights2(moe::GroupedGemmArgs *b, const Experts &X)
{
    b->w_a = X.W2; b->w_b = nullptr; b->w8 = X.fp8; b->scale_a = X.s2; b->scale_b = nullptr;
}

// The activation operand of a GEMM: the bf16 rows, or (a8) their quantized form,
// produced here from the bf16 rows.
moe_status_t set_act(moe::GroupedGemmArgs *g, const uint16_t *rows, int64_t R, int K, uint8_t *q, float *sc,
                     bool a8, cudaStream_t s)
{
    if (!a8) { g->act = rows; return MOE_OK; }
    MOE_CUDA(moe::launch_quantize_fp8(rows, R, K, q, sc, s));
    g->act = q; g->a8 = true; g->scale_act = sc;
    return MOE_OK;
}

moe_status_t expert_ffn_impl(const uint16_t *x_perm, const int32_t *offsets, const Experts &X, int64_t R, int H,
                             int I, int E, uint16_t *h, float *y_perm, const ActQ &Q, int *err, cudaStream_t s)
{
    if (R == 0) return MOE_OK;
    moe::GroupedGemmArgs a{};
    a.offsets = offsets; a.groups = E; a.R = R;
    a.K = H; a.Nout = I; a.out = h; a.dev_err = err;
    set_weights13(&a, X);
    if (moe_status_t st = set_act(&a, x_perm, R, H, Q.xq, Q.xsc, X.a8, s)) return st;
    MOE_CUDA(moe::launch_gemm13_swiglu(a, s));
    moe::GroupedGemmArgs b{};
    b.offsets = offsets; b.groups = E; b.R = R;
    b.K = I; b.Nout = H; b.out = y_perm; b.dev_err = err;
    set_weights2(&b, X);
    if (moe_status_t st = set_act(&b, h, R, I, Q.hq, Q.hsc, X.a8, s)) return st;
    MOE_CUDA(moe::launch_gemm2(b, s));
    return MOE_OK;
}

// Shared experts: one dense SwiGLU FFN over all N rows = the grouped kernels with a
// single group whose rows are x itself.
moe_status_t shared_ffn_impl(const uint16_t *x, const uint16_t *Ws1, const uint16_t *Ws3,
                             const uint16_t *Ws2, int64_t N, int H, int Is, uint16_t *hs, float *s_out,
                             int *err, cudaStream_t s)
{
    if (N == 0) return MOE_OK;
    moe::GroupedGemmArgs a{};
    a.act = x; a.w_a = Ws1; a.w_b = Ws3; a.offsets = nullptr; a.groups = 1; a.R = N;
    a.rows_single = (int)N; a.K = H; a.Nout = Is; a.out = hs; a.dev_err = err;
    MOE_CUDA(moe::launch_gemm13_swiglu(a, s));
    moe::GroupedGemmArgs b{};
    b.act = hs; b.w_a = Ws2; b.offsets = nullptr; b.groups = 1; b.R = N; b.rows_single = (int)N;
    b.K = Is; b.Nout = H; b.out = s_out; b.dev_err = err;
    MOE_CUDA(moe::launch_gemm2(b, s));
    return MOE_OK;
}

moe_status_t record(void *const *ev, int i, cudaStream_t s)
{
    if (ev && ev[i]) MOE_CUDA(cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s));
    return MOE_OK;
}

#define MOE_TRY(call)                            \
    do {                                         \
        moe_status_t st_ = (call);               \
        if (st_ != MOE_OK) return st_;           \
    } while (0)

// The layer on N rows with a workspace laid out for N rows; after_dispatch (nullable)
// runs once the permute phase is enqueued on s.
// A second stream with its fork and join events (the shared experts' side stream).
struct SideStream {
    cudaStream_t s2;
    cudaEvent_t fork, join;
};

template <typename Hook>
moe_status_t layer_run(const uint16_t *x, const float *W_gate, const float *bias, const Experts &X,
                       const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H, int I, int E,
                       int k, int Is, uint16_t *out, float *logits, void *ws, int *err, cudaStream_t s,
                       void *const *phase_events, Hook after_dispatch, const SideStream *side = nullptr)
{
    WsLayout L;
    ws_layout(N, H, I, E, k, Is, X.a8, &L);
    uint8_t *base = static_cast<uint8_t *>(ws);
    const ActQ Q{base + L.xq, reinterpret_cast<float *>(base + L.xsc), base + L.hq,
                 reinterpret_cast<float *>(base + L.hsc), base + L.xqt, reinterpret_cast<float *>(base + L.xst)};
    float *lg = logits ? logits : reinterpret_cast<float *>(base + L.logits);
    int32_t *idx = reinterpret_cast<int32_t *>(base + L.idx);
    float *w = reinterpret_cast<float *>(base + L.w);
    int32_t *counts = reinterpret_cast<int32_t *>(base + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(base + L.offsets);
    int32_t *r2t = reinterpret_cast<int32_t *>(base + L.r2t);
    int32_t *t2r = reinterpret_cast<int32_t *>(base + L.t2r);
    int32_t *perm = reinterpret_cast<int32_t *>(base + L.perm);
    uint16_t *x_perm = reinterpret_cast<uint16_t *>(base + L.x_perm);
    uint16_t *h = reinterpret_cast<uint16_t *>(base + L.h);
    uint16_t *hs = reinterpret_cast<uint16_t *>(base + L.hs);
    float *y_perm = reinterpret_cast<float *>(base + L.y_perm);
    float *sh = Is > 0 ? reinterpret_cast<float *>(base + L.s) : nullptr;
    const int64_t R = N * k;

    MOE_TRY(record(phase_events, 0, s));
    if (side && Is > 0) {
        // the shared experts need only x: they start at once on the side stream, beside the
        // router and the dispatch, and are joined before whatever adds their output
        MOE_CUDA(cudaEventRecord(side->fork, s));
        MOE_CUDA(cudaStreamWaitEvent(side->s2, side->fork, 0));
        MOE_TRY(shared_ffn_impl(x, Ws1, Ws3, Ws2, N, H, Is, hs, sh, err, side->s2));
        MOE_CUDA(cudaEventRecord(side->join, side->s2));
    }
    moe::GroupedGemmArgs a{};
    a.offsets = offsets; a.groups = E; a.R = R;
    a.K = H; a.Nout = I; a.out = h; a.dev_err = err;
    set_weights13(&a, X);
    const bool gather = !X.a8 && !X.fp8 && moe::layer_gathers(N, k, H);
    if (!X.a8 && !X.fp8 && !gather && moe::layer_decode_gemv(N, k, E, H, I)) {
        // a decode batch in bf16: the router's partial logits, then the expert FFN as two
        // GEMV kernels on CUDA cores -- the first finishes the top-k, reads x per pick (no
        // dispatch, no row copies), the second folds in the combine
        moe::RouterPartials rp{};
        MOE_CUDA(moe::launch_router_partials(x, W_gate, bias, N, H, E, k, lg, idx, w, base + L.router,
                                             L.router_bytes, &rp, s));
        for (int p : {MOE_PHASE_ROUTE, MOE_PHASE_PERMUTE}) MOE_TRY(record(phase_events, 1 + p, s));
        MOE_TRY(after_dispatch());
        MOE_CUDA(moe::launch_decode_w13(x, rp, idx, w, N, k, E, H, I, static_cast<const uint16_t *>(X.W1),
                                        static_cast<const uint16_t *>(X.W3), h, err, s));
        MOE_TRY(record(phase_events, 1 + MOE_PHASE_GEMM13, s));
        // the W2 kernel adds the shared experts' output: it must be complete (with phase
        // events, the gemm2 phase holds the shared experts and the combine)
        if (Is > 0) {
            if (side) MOE_CUDA(cudaStreamWaitEvent(s, side->join, 0));
            else MOE_TRY(shared_ffn_impl(x, Ws1, Ws3, Ws2, N, H, Is, hs, sh, err, s));
        }
        MOE_CUDA(moe::launch_decode_w2_combine(h, idx, w, sh, N, E, H, I, k, static_cast<const uint16_t *>(X.W2),
                                               out, err, s));
        for (int p : {MOE_PHASE_GEMM2, MOE_PHASE_SHARED, MOE_PHASE_COMBINE}) MOE_TRY(record(phase_events, 1 + p, s));
        return MOE_OK;
    }
    // a small batch: router, top-k, dispatch and the row copies in two kernels (the
    // route phase then holds the permute phase's work too)
    cudaError_t fused = cudaErrorNotSupported;
    if (!X.a8 && !gather) {
        fused = moe::launch_route_dispatch_small(x, W_gate, bias, N, H, E, k, lg, idx, w, base + L.router,
                                                 L.router_bytes, counts, offsets, r2t, t2r, x_perm, err, s);
        if (fused != cudaSuccess && fused != cudaErrorNotSupported) return cuda_fail(fused);
    }
    if (fused != cudaSuccess)
        MOE_CUDA(moe::launch_router(x, W_gate, bias, N, H, E, k, lg, idx, w, base + L.router, L.router_bytes, err, s));
    MOE_TRY(record(phase_events, 1 + MOE_PHASE_ROUTE, s));
    if (fused == cudaSuccess) {
        a.act = x_perm;
    } else if (X.a8) {
        // each token row is quantized once (N rows, not N*k: a permuted row is a copy of
        // its token's row, so its codes and scale are the same), then the codes and the
        // scales move to the permuted rows
        MOE_CUDA(moe::launch_quantize_fp8(x, N, H, Q.xqt, Q.xst, s));
        MOE_CUDA(moe::launch_permute(x, idx, N, H, E, k, counts, offsets, r2t, t2r, nullptr, perm, err, s));
        MOE_CUDA(moe::launch_scatter_rows(reinterpret_cast<const uint16_t *>(Q.xqt), Q.xst, t2r, N, k, H / 2,
                                          reinterpret_cast<uint16_t *>(Q.xq), R, Q.xsc, s));
        a.act = Q.xq; a.a8 = true; a.scale_act = Q.xsc;
    } else if (gather) {
        // dispatch only: W1/W3 gathers its rows from x through row_to_token
        MOE_CUDA(moe::launch_permute(x, idx, N, H, E, k, counts, offsets, r2t, t2r, nullptr, perm, err, s));
        a.act = x; a.gather_rows = r2t; a.gather_src_rows = N;
    } else {
        MOE_CUDA(moe::launch_permute(x, idx, N, H, E, k, counts, offsets, r2t, t2r, x_perm, perm, err, s));
        a.act = x_perm;
    }
    MOE_TRY(record(phase_events, 1 + MOE_PHASE_PERMUTE, s));
    MOE_TRY(after_dispatch());
    MOE_CUDA(moe::launch_gemm13_swiglu(a, s));
    const int ksplit = moe::gemm2_ksplit(R, E, I, H);
    moe::GroupedGemmArgs b{};
    b.offsets = offsets; b.groups = E; b.R = R;
    b.K = I; b.Nout = H; b.out = y_perm; b.dev_err = err;
    set_weights2(&b, X);
    b.ksplit = ksplit; b.split_stride = R * (int64_t)H;
    MOE_TRY(set_act(&b, h, R, I, Q.hq, Q.hsc, X.a8, s));
    MOE_TRY(record(phase_events, 1 + MOE_PHASE_GEMM13, s));
    MOE_CUDA(moe::launch_gemm2(b, s));
    MOE_TRY(record(phase_events, 1 + MOE_PHASE_GEMM2, s));
    if (Is > 0) {
        if (side) MOE_CUDA(cudaStreamWaitEvent(s, side->join, 0));
        else MOE_TRY(shared_ffn_impl(x, Ws1, Ws3, Ws2, N, H, Is, hs, sh, err, s));
    }
    MOE_TRY(record(phase_events, 1 + MOE_PHASE_SHARED, s));
    MOE_CUDA(moe::launch_combine(y_perm, ksplit, R * (int64_t)H, t2r, w, sh, N, H, k, out, s));
    MOE_TRY(record(phase_events, 1 + MOE_PHASE_COMBINE, s));
    return MOE_OK;
}

// A second stream and two events per device for the micro-batched layer, created on
// first use and kept for the process; the mutex makes one layer call's fork and join
// use them at a time.
struct MicroStreams {
    std::mutex mu;
    cudaStream_t s2 = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr, rows2 = nullptr, half1 = nullptr;
    void *ctx = nullptr;
};

// Creates the device's second stream and events on first use (again under a new context).
moe_status_t ensure_side_stream(MicroStreams *ms)
{
    void *ctx = moe::current_context();
    if (!ms->s2 || ctx != ms->ctx) {
        MOE_CUDA(cudaStreamCreateWithFlags(&ms->s2, cudaStreamNonBlocking));
        MOE_CUDA(cudaEventCreateWithFlags(&ms->fork, cudaEventDisableTiming));
        MOE_CUDA(cudaEventCreateWithFlags(&ms->join, cudaEventDisableTiming));
        MOE_CUDA(cudaEventCreateWithFlags(&ms->rows2, cudaEventDisableTiming));
        MOE_CUDA(cudaEventCreateWithFlags(&ms->half1, cudaEventDisableTiming));
        ms->ctx = moe::current_context();
    }
    return MOE_OK;
}

MicroStreams *micro_streams()
{
    static MicroStreams per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    return &per_dev[dev];
}

// The layer with its expert GEMMs in two micro-batches of tokens, [0, N0) and [N0, N)
// (the pages' ping-pong of micro-batches, inside one GPU).  The router and the dispatch
// run once for the whole batch; inside every expert's group the rows of the first half's
// tokens come first (the dispatch is stable), and the dispatch's per-block table at the
// block where the second half starts gives, for every expert, the row where its second
// half starts.  So the two halves' GEMMs are the same grouped kernels on complementary
// row ranges of each group, writing disjoint rows of h and y.  On the caller's stream s:
// router, dispatch, the first half's row copies, its GEMMs, then the second half's GEMMs
// and combine.  On the side stream: the second half's row copies, started after the
// dispatch, and the first half's combine, started after its GEMMs -- so HBM-bound
// copies and combines run beside the persistent GEMMs of the other half.  Every token's
// arithmetic is the one-piece layer's.
moe_status_t layer_run_micro(const uint16_t *x, const float *W_gate, const float *bias, const Experts &X, int64_t N,
                             int H, int I, int E, int k, uint16_t *out, float *logits, void *ws, int *err,
                             cudaStream_t s, MicroStreams *ms, int64_t N0)
{
    WsLayout L;
    ws_layout(N, H, I, E, k, 0, false, &L);
    uint8_t *base = static_cast<uint8_t *>(ws);
    float *lg = logits ? logits : reinterpret_cast<float *>(base + L.logits);
    int32_t *idx = reinterpret_cast<int32_t *>(base + L.idx);
    float *w = reinterpret_cast<float *>(base + L.w);
    int32_t *counts = reinterpret_cast<int32_t *>(base + L.counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(base + L.offsets);
    int32_t *r2t = reinterpret_cast<int32_t *>(base + L.r2t);
    int32_t *t2r = reinterpret_cast<int32_t *>(base + L.t2r);
    int32_t *perm = reinterpret_cast<int32_t *>(base + L.perm);
    uint16_t *x_perm = reinterpret_cast<uint16_t *>(base + L.x_perm);
    uint16_t *h = reinterpret_cast<uint16_t *>(base + L.h);
    float *y_perm = reinterpret_cast<float *>(base + L.y_perm);
    const int64_t R = N * k;
    const int64_t N1 = N - N0;
    cudaStream_t s2 = ms->s2;

    MOE_CUDA(moe::launch_router(x, W_gate, bias, N, H, E, k, lg, idx, w, base + L.router, L.router_bytes, err, s));
    MOE_CUDA(moe::launch_permute(x, idx, N, H, E, k, counts, offsets, r2t, t2r, nullptr, perm, err, s));
    const int32_t *mid = perm + (N0 * k / moe::kPermuteChunk) * E;  // second half's first row, per expert
    MOE_CUDA(moe::launch_scatter_rows(x, nullptr, t2r, N0, k, H, x_perm, R, nullptr, s));
    MOE_CUDA(cudaEventRecord(ms->fork, s));
    MOE_CUDA(cudaStreamWaitEvent(s2, ms->fork, 0));
    MOE_CUDA(moe::launch_scatter_rows(x + N0 * H, nullptr, t2r + N0 * k, N1, k, H, x_perm, R, nullptr, s2));
    MOE_CUDA(cudaEventRecord(ms->rows2, s2));

    const int ksplit = moe::gemm2_ksplit(R, E, I, H);
    auto gemms = [&](const int32_t *starts, const int32_t *ends) -> moe_status_t {
        moe::GroupedGemmArgs a{};
        a.act = x_perm; a.offsets = starts; a.ends = ends; a.groups = E; a.R = R;
        a.K = H; a.Nout = I; a.out = h; a.dev_err = err;
        set_weights13(&a, X);
        MOE_CUDA(moe::launch_gemm13_swiglu(a, s));
        moe::GroupedGemmArgs b{};
        b.act = h; b.offsets = starts; b.ends = ends; b.groups = E; b.R = R;
        b.K = I; b.Nout = H; b.out = y_perm; b.dev_err = err;
        set_weights2(&b, X);
        b.ksplit = ksplit; b.split_stride = R * (int64_t)H;
        MOE_CUDA(moe::launch_gemm2(b, s));
        return MOE_OK;
    };
    MOE_TRY(gemms(offsets, mid));                 // first half: [offsets[e], mid[e])
    MOE_CUDA(cudaEventRecord(ms->half1, s));
    MOE_CUDA(cudaStreamWaitEvent(s2, ms->half1, 0));
    MOE_CUDA(moe::launch_combine(y_perm, ksplit, R * (int64_t)H, t2r, w, nullptr, N0, H, k, out, s2));
    MOE_CUDA(cudaEventRecord(ms->join, s2));
    MOE_CUDA(cudaStreamWaitEvent(s, ms->rows2, 0));
    MOE_TRY(gemms(mid, offsets + 1));             // second half: [mid[e], offsets[e + 1])
    MOE_CUDA(moe::launch_combine(y_perm, ksplit, R * (int64_t)H, t2r + N0 * k, w + N0 * k, nullptr, N1, H, k,
                                 out + N0 * H, s));
    MOE_CUDA(cudaStreamWaitEvent(s, ms->join, 0));
    return MOE_OK;
}

moe_status_t layer_impl(const uint16_t *x, const float *W_gate, const float *bias, const Experts &X,
                        const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H, int I,
                        int E, int k, int Is, uint16_t *out, float *logits, void *ws, size_t ws_bytes,
                        void *stream, void *const *phase_events)
{
    if (!valid_rows(N, k) || !valid_hidden(H) || !valid_hidden(I) || !valid_ek(E, k)) return MOE_ERR_INVALID_ARG;
    if (Is < 0 || (Is > 0 && !valid_hidden(Is))) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (N == 0) return MOE_OK;
    if (!x || !W_gate || !X.W1 || !X.W3 || !X.W2 || !out) return MOE_ERR_INVALID_ARG;
    if (Is > 0 && (!Ws1 || !Ws3 || !Ws2)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(X.W1) || !aligned16(X.W3) || !aligned16(X.W2) || !aligned16(out))
        return MOE_ERR_UNSUPPORTED;
    if (Is > 0 && (!aligned16(Ws1) || !aligned16(Ws3) || !aligned16(Ws2))) return MOE_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < layer_ws_bytes(N, H, I, E, k, Is, X.a8) || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    int *err = device_error_word();
    if (!err) return cuda_fail(cudaGetLastError());
    auto none = [] { return MOE_OK; };
    const int64_t N0 = micro_split(N, k);
    const bool side_shared = Is > 0 && moe::layer_shared_side() && !phase_events && N0 == 0;
    if (side_shared) {
        MicroStreams *ms = micro_streams();
        if (!ms) return MOE_ERR_UNSUPPORTED;
        std::lock_guard<std::mutex> lock(ms->mu);
        MOE_TRY(ensure_side_stream(ms));
        const SideStream side{ms->s2, ms->fork, ms->join};
        return layer_run(x, W_gate, bias, X, Ws1, Ws3, Ws2, N, H, I, E, k, Is, out, logits, ws, err, s, nullptr,
                         none, &side);
    }
    const bool micro = N0 > 0 && !phase_events && !X.a8 && !X.fp8 && Is == 0 && !moe::layer_gathers(N, k, H);
    if (!micro)
        return layer_run(x, W_gate, bias, X, Ws1, Ws3, Ws2, N, H, I, E, k, Is, out, logits, ws, err, s,
                         phase_events, none);
    MicroStreams *ms = micro_streams();
    if (!ms) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(ms->mu);
    MOE_TRY(ensure_side_stream(ms));
    return layer_run_micro(x, W_gate, bias, X, N, H, I, E, k, out, logits, ws, err, s, ms, N0);
}
}  // namespace

extern "C" {

const char *moe_status_string(moe_status_t status)
{
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape, alignment or device";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_DEVICE: return "device-side fault reported by a kernel";
    }
    return "unknown status";
}

const char *moe_last_cuda_error(void) { return g_last_cuda_error; }

int moe_device_sm_count(void) { return moe::device_sm_count(); }

uint64_t moe_kernel_launches(void) { return moe::launches_so_far(); }

int moe_set_shared_stream(int on)
{
    if (on != 0 && on != 1) return -1;
    return moe::g_shared_side.exchange(on);
}

int moe_set_decode_gemv(int mode)
{
    if (mode != MOE_DECODE_AUTO && mode != MOE_DECODE_OFF && mode != MOE_DECODE_ON) return -1;
    return moe::g_decode_gemv.exchange(mode);
}

int moe_set_microbatches(int m)
{
    if (m < 1 || m > 2) return -1;
    return moe::g_microbatches.exchange(m);
}

int moe_set_gather_mode(int mode)
{
    if (mode != MOE_GATHER_AUTO && mode != MOE_GATHER_OFF && mode != MOE_GATHER_ON) return -1;
    return moe::g_gather_mode.exchange(mode);
}

size_t moe_workspace_bytes(int64_t N, int H, int I, int E, int k, int Is)
{
    if (!valid_rows(N, k) || !valid_hidden(H) || !valid_hidden(I) || !valid_ek(E, k)) return 0;
    if (Is < 0 || (Is > 0 && !valid_hidden(Is))) return 0;
    return layer_ws_bytes(N, H, I, E, k, Is, false);
}

size_t moe_workspace_bytes_w8a8(int64_t N, int H, int I, int E, int k, int Is)
{
    if (!valid_rows(N, k) || !valid_hidden(H) || !valid_hidden(I) || !valid_ek(E, k)) return 0;
    if (Is < 0 || (Is > 0 && !valid_hidden(Is))) return 0;
    return layer_ws_bytes(N, H, I, E, k, Is, true);
}

moe_status_t moe_route(const uint16_t *x, const float *W_gate, const float *bias, int64_t N, int H, int E,
                       int k, float *logits, int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes,
                       void *stream)
{
    if (!valid_rows(N, k) || !valid_hidden(H) || !valid_ek(E, k)) return MOE_ERR_INVALID_ARG;
    if (N == 0) return MOE_OK;
    if (!x || !W_gate || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || (ws && !aligned16(ws))) return MOE_ERR_UNSUPPORTED;
    int *err = device_error_word();
    if (!err) return cuda_fail(cudaGetLastError());
    MOE_CUDA(moe::launch_router(x, W_gate, bias, N, H, E, k, logits, topk_idx, topk_w, ws, ws ? ws_bytes : 0,
                                err, static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

moe_status_t moe_permute(const uint16_t *x, const int32_t *topk_idx, int64_t N, int H, int E, int k,
                         int32_t *counts, int32_t *offsets, int32_t *row_to_token, int32_t *token_to_row,
                         uint16_t *x_perm, void *ws, size_t ws_bytes, void *stream)
{
    if (!valid_rows(N, k) || !valid_hidden(H) || !valid_ek(E, k)) return MOE_ERR_INVALID_ARG;
    if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (N == 0) {
        // empty batch: the group table is still well defined (all zero)
        MOE_CUDA(cudaMemsetAsync(counts, 0, (size_t)E * 4, s));
        MOE_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * 4, s));
        return MOE_OK;
    }
    if (!x || !topk_idx || !row_to_token || !token_to_row || !x_perm) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_UNSUPPORTED;
    const size_t need = (size_t)moe::permute_scratch_ints(N * k, E) * 4;
    if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
    int *err = device_error_word();
    if (!err) return cuda_fail(cudaGetLastError());
    MOE_CUDA(moe::launch_permute(x, topk_idx, N, H, E, k, counts, offsets, row_to_token, token_to_row, x_perm,
                                 static_cast<int32_t *>(ws), err, s));
    return MOE_OK;
}

moe_status_t moe_expert_ffn(const uint16_t *x_perm, const int32_t *offsets, const uint16_t *W1,
                            const uint16_t *W3, const uint16_t *W2, int64_t R, int H, int I, int E,
                            float *y_perm, void *ws, size_t ws_bytes, void *stream)
{
    if (R < 0 || R >= (int64_t(1) << 31) || !valid_hidden(H) || !valid_hidden(I) || E < 1 || E > 256)
        return MOE_ERR_INVALID_ARG;
    if (R == 0) return MOE_OK;
    if (!x_perm || !offsets || !W1 || !W3 || !W2 || !y_perm) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_perm) || !aligned16(W1) || !aligned16(W3) || !aligned16(W2) || !aligned16(y_perm))
        return MOE_ERR_UNSUPPORTED;
    const size_t need = (size_t)R * I * 2;
    if (!ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    int *err = device_error_word();
    if (!err) return cuda_fail(cudaGetLastError());
    const Experts X{W1, W3, W2, nullptr, nullptr, nullptr, false, false};
    return expert_ffn_impl(x_perm, offsets, X, R, H, I, E, static_cast<uint16_t *>(ws), y_perm, ActQ{}, err,
                           static_cast<cudaStream_t>(stream));
}

moe_status_t moe_scatter_rows(const uint16_t *src, const int32_t *dst_row, int64_t rows, int width, uint16_t *dst,
                              int64_t dst_rows, void *stream)
{
    if (rows < 0 || dst_rows < 0 || width < 8 || width % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!src || !dst_row || !dst) return MOE_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst)) return MOE_ERR_UNSUPPORTED;
    MOE_CUDA(moe::launch_scatter_rows(src, nullptr, dst_row, rows, 1, width, dst, dst_rows, nullptr,
                                      static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

moe_status_t moe_combine(const float *y_perm, const int32_t *token_to_row, const float *topk_w,
                         const float *shared_out, int64_t N, int H, int k, uint16_t *out, void *stream)
{
    if (!valid_rows(N, k) || !valid_hidden(H) || k < 1 || k > 8) return MOE_ERR_INVALID_ARG;
    if (N == 0) return MOE_OK;
    if (!y_perm || !token_to_row || !topk_w || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(y_perm) || !aligned16(out) || (shared_out && !aligned16(shared_out)))
        return MOE_ERR_UNSUPPORTED;
    MOE_CUDA(moe::launch_combine(y_perm, 1, 0, token_to_row, topk_w, shared_out, N, H, k, out,
                                 static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

moe_status_t moe_layer_forward_ex(const uint16_t *x, const float *W_gate, const float *bias,
                                  const uint16_t *W1, const uint16_t *W3, const uint16_t *W2,
                                  const uint16_t *Ws1, const uint16_t *Ws3, const uint16_t *Ws2, int64_t N,
                                  int H, int I, int E, int k, int Is, uint16_t *out, float *logits, void *ws,
                                  size_t ws_bytes, void *stream, void *const *phase_events)
{
    const Experts X{W1, W3, W2, nullptr, nullptr, nullptr, false, false};
    return layer_impl(x, W_gate, bias, X, Ws1, Ws3, Ws2, N, H, I, E, k, Is, out, logits, ws, ws_bytes, stream,
                      phase_events);
}

moe_status_t moe_layer_forward_fp8_ex(const uint16_t *x, const float *W_gate, const float *bias,
                                      const uint8_t *W1q, const float *s1, const uint8_t *W3q, const float *s3,
                                      const uint8_t *W2q, const float *s2, const uint16_t *Ws1,
                                      const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H, int I, int E,
                                      int k, int Is, uint16_t *out, float *logits, void *ws, size_t ws_bytes,
                                      void *stream, void *const *phase_events)
{
    if (N > 0 && (!s1 || !s3 || !s2)) return MOE_ERR_INVALID_ARG;
    const Experts X{W1q, W3q, W2q, s1, s3, s2, true, false};
    return layer_impl(x, W_gate, bias, X, Ws1, Ws3, Ws2, N, H, I, E, k, Is, out, logits, ws, ws_bytes, stream,
                      phase_events);
}

moe_status_t moe_layer_forward_w8a8_ex(const uint16_t *x, const float *W_gate, const float *bias,
                                       const uint8_t *W1q, const float *s1, const uint8_t *W3q, const float *s3,
                                       const uint8_t *W2q, const float *s2, const uint16_t *Ws1,
                                       const uint16_t *Ws3, const uint16_t *Ws2, int64_t N, int H, int I, int E,
                                       int k, int Is, uint16_t *out, float *logits, void *ws, size_t ws_bytes,
                                       void *stream, void *const *phase_events)
{
    if (N > 0 && (!s1 || !s3 || !s2)) return MOE_ERR_INVALID_ARG;
    const Experts X{W1q, W3q, W2q, s1, s3, s2, true, true};
    return layer_impl(x, W_gate, bias, X, Ws1, Ws3, Ws2, N, H, I, E, k, Is, out, logits, ws, ws_bytes, stream,
                      phase_events);
}

moe_status_t moe_quantize_fp8(const uint16_t *W, int64_t rows, int K, uint8_t *q, float *scale, void *stream)
{
    if (rows < 0 || !valid_hidden(K)) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!W || !q || !scale) return MOE_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(q) || !aligned16(scale)) return MOE_ERR_UNSUPPORTED;
    MOE_CUDA(moe::launch_quantize_fp8(W, rows, K, q, scale, static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

moe_status_t moe_expert_ffn_fp8(const uint16_t *x_perm, const int32_t *offsets, const uint8_t *W1q,
                                const float *s1, const uint8_t *W3q, const float *s3, const uint8_t *W2q,
                                const float *s2, int64_t R, int H, int I, int E, float *y_perm, void *ws,
                                size_t ws_bytes, void *stream)
{
    if (R < 0 || R >= (int64_t(1) << 31) || !valid_hidden(H) || !valid_hidden(I) || E < 1 || E > 256)
        return MOE_ERR_INVALID_ARG;
    if (R == 0) return MOE_OK;
    if (!x_perm || !offsets || !W1q || !W3q || !W2q || !s1 || !s3 || !s2 || !y_perm) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_perm) || !aligned16(W1q) || !aligned16(W3q) || !aligned16(W2q) || !aligned16(y_perm))
        return MOE_ERR_UNSUPPORTED;
    const size_t need = (size_t)R * I * 2;
    if (!ws || ws_bytes < need || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    int *err = device_error_word();
    if (!err) return cuda_fail(cudaGetLastError());
    const Experts X{W1q, W3q, W2q, s1, s3, s2, true, false};
    return expert_ffn_impl(x_perm, offsets, X, R, H, I, E, static_cast<uint16_t *>(ws), y_perm, ActQ{}, err,
                           static_cast<cudaStream_t>(stream));
}

// h [R,I] bf16 (when the caller keeps none), then x_perm's and h's quantized rows and scales.
size_t moe_expert_ffn_w8a8_ws_bytes(int64_t R, int H, int I)
{
    if (R < 0 || R >= (int64_t(1) << 31) || !valid_hidden(H) || !valid_hidden(I)) return 0;
    return round_up((size_t)R * I * 2) + round_up((size_t)R * H) + round_up((size_t)R * 4) +
           round_up((size_t)R * I) + round_up((size_t)R * 4);
}

moe_status_t moe_expert_ffn_w8a8(const uint16_t *x_perm, const int32_t *offsets, const uint8_t *W1q,
                                 const float *s1, const uint8_t *W3q, const float *s3, const uint8_t *W2q,
                                 const float *s2, int64_t R, int H, int I, int E, float *y_perm, uint16_t *h,
                                 void *ws, size_t ws_bytes, void *stream)
{
    if (R < 0 || R >= (int64_t(1) << 31) || !valid_hidden(H) || !valid_hidden(I) || E < 1 || E > 256)
        return MOE_ERR_INVALID_ARG;
    if (R == 0) return MOE_OK;
    if (!x_perm || !offsets || !W1q || !W3q || !W2q || !s1 || !s3 || !s2 || !y_perm) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_perm) || !aligned16(W1q) || !aligned16(W3q) || !aligned16(W2q) || !aligned16(y_perm) ||
        (h && !aligned16(h)))
        return MOE_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < moe_expert_ffn_w8a8_ws_bytes(R, H, I) || !aligned16(ws)) return MOE_ERR_WORKSPACE;
    int *err = device_error_word();
    if (!err) return cuda_fail(cudaGetLastError());
    uint8_t *p = static_cast<uint8_t *>(ws);
    uint16_t *hb = reinterpret_cast<uint16_t *>(p);
    p += round_up((size_t)R * I * 2);
    ActQ Q{};
    Q.xq = p; p += round_up((size_t)R * H);
    Q.xsc = reinterpret_cast<float *>(p); p += round_up((size_t)R * 4);
    Q.hq = p; p += round_up((size_t)R * I);
    Q.hsc = reinterpret_cast<float *>(p);
    const Experts X{W1q, W3q, W2q, s1, s3, s2, true, true};
    return expert_ffn_impl(x_perm, offsets, X, R, H, I, E, h ? h : hb, y_perm, Q, err,
                           static_cast<cudaStream_t>(stream));
}

moe_status_t moe_layer_forward(const uint16_t *x, const float *W_gate, const uint16_t *W1, const uint16_t *W3,
                               const uint16_t *W2, int64_t N, int H, int I, int E, int k, uint16_t *out)
{
    if (!valid_rows(N, k) || !valid_hidden(H) || !valid_hidden(I) || !valid_ek(E, k)) return MOE_ERR_INVALID_ARG;
    if (N == 0) return MOE_OK;
    if (!x || !W_gate || !W1 || !W3 || !W2 || !out) return MOE_ERR_INVALID_ARG;

    // Library-owned buffers, one set per device, grown on demand.
    struct Cache { void *ws = nullptr; size_t ws_bytes = 0; void *io = nullptr; size_t io_bytes = 0; };
    static Cache cache[64];
    static std::mutex mu;
    int dev = 0;
    MOE_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(mu);
    Cache &c = cache[dev];

    auto is_device = [](const void *p) {
        cudaPointerAttributes at{};
        if (cudaPointerGetAttributes(&at, p) != cudaSuccess) { cudaGetLastError(); return false; }
        return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
    };
    const bool x_dev = is_device(x), out_dev = is_device(out);
    const size_t act_bytes = round_up((size_t)N * H * 2);
    const size_t io_need = (x_dev ? 0 : act_bytes) + (out_dev ? 0 : act_bytes);
    const size_t ws_need = moe_workspace_bytes(N, H, I, E, k, 0);
    if (c.ws_bytes < ws_need) {
        if (c.ws) MOE_CUDA(cudaFree(c.ws));
        c.ws = nullptr; c.ws_bytes = 0;
        MOE_CUDA(cudaMalloc(&c.ws, ws_need));
        c.ws_bytes = ws_need;
    }
    if (c.io_bytes < io_need) {
        if (c.io) MOE_CUDA(cudaFree(c.io));
        c.io = nullptr; c.io_bytes = 0;
        MOE_CUDA(cudaMalloc(&c.io, io_need));
        c.io_bytes = io_need;
    }
    const cudaStream_t s = 0;
    uint8_t *io = static_cast<uint8_t *>(c.io);
    const uint16_t *xd = x;
    uint16_t *outd = out;
    if (!x_dev) {
        MOE_CUDA(cudaMemcpyAsync(io, x, (size_t)N * H * 2, cudaMemcpyHostToDevice, s));
        xd = reinterpret_cast<const uint16_t *>(io);
        io += act_bytes;
    }
    if (!out_dev) outd = reinterpret_cast<uint16_t *>(io);
    MOE_TRY(moe_layer_forward_ex(xd, W_gate, nullptr, W1, W3, W2, nullptr, nullptr, nullptr, N, H, I, E, k, 0,
                                 outd, nullptr, c.ws, c.ws_bytes, s, nullptr));
    if (!out_dev) {
        MOE_CUDA(cudaMemcpyAsync(out, outd, (size_t)N * H * 2, cudaMemcpyDeviceToHost, s));
        MOE_CUDA(cudaStreamSynchronize(s));
    }
    return MOE_OK;
}

moe_status_t moe_get_device_error(void *stream, int32_t *code)
{
    if (!code) return MOE_ERR_INVALID_ARG;
    MOE_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int v = 0;
    MOE_CUDA(cudaMemcpyFromSymbol(&v, g_moe_device_error, sizeof v));
    const int zero = 0;
    MOE_CUDA(cudaMemcpyToSymbol(g_moe_device_error, &zero, sizeof zero));
    *code = v;
    return MOE_OK;
}

}  // extern "C"
