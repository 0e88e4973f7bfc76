// permute_noalloc.cu -- moe_permute without a caller workspace (see include/moe.h).
//
// For callers that cannot allocate device memory: the dispatch's per-block expert
// histograms live in a fixed array inside the library instead of a workspace, and
// the call then runs the same kernels as moe_permute.  Nothing here allocates.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace {

// 1 MiB per device, held by every GPU that loads the library until the process exits.
static __device__ __align__(256) int32_t g_permute_scratch[MOE_PERMUTE_NOALLOC_MAX_SCRATCH_INTS];

// Device address of g_permute_scratch on the current device, looked up once per
// device and context (again after a device reset, or under another context on the
// same device).  In host code the symbol itself is only a host-side stand-in: a
// kernel handed it would fault, or silently touch the wrong memory where the GPU can
// reach host memory, so kernels get this address instead.
cudaError_t scratch_address(int32_t **out)
{
    static std::mutex mu;
    static int32_t *addr[64] = {nullptr};
    static void *ctx_of[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    void *ctx = moe::current_context();
    if (!addr[dev] || !ctx || ctx != ctx_of[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = static_cast<int32_t *>(p);
        ctx_of[dev] = moe::current_context();  // bound now, if the lookup initialised it
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const uint16_t *x, const int32_t *topk_idx, int64_t N, int H,
                                            int E, int k, int32_t *counts, int32_t *offsets,
                                            int32_t *row_to_token, int32_t *token_to_row, uint16_t *x_perm,
                                            void *stream)
{
    // N * k < 2^31, checked before the product is formed (a huge N would overflow it)
    if (k < 1 || k > 8 || E < 1 || E > 256 || N < 0 || N >= ((int64_t(1) << 31) + k - 1) / k)
        return MOE_ERR_INVALID_ARG;
    if (moe::permute_scratch_ints(N * k, E) > MOE_PERMUTE_NOALLOC_MAX_SCRATCH_INTS) return MOE_ERR_UNSUPPORTED;
    int32_t *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    return moe_permute(x, topk_idx, N, H, E, k, counts, offsets, row_to_token, token_to_row, x_perm, scratch,
                       sizeof(int32_t) * (size_t)MOE_PERMUTE_NOALLOC_MAX_SCRATCH_INTS, stream);
}
