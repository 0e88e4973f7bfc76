// quantize.cu -- e4m3 expert weights with one fp32 scale per output channel (sm_100a).
//
// MoE-latency article, section "优化从测量开始": quantizing the weights cuts the bytes
// a decode step streams, and its numerical error is measured as an experiment of its
// own.  The pages fix no format; this library uses OCP e4m3 (largest finite 448) with
// one scale per weight row:
//   s[r] = max_c |W[r,c]| / 448   (fp32, correctly rounded; 1 for an all-zero row)
//   q[r,c] = e4m3(W[r,c] / s[r])  (fp32 quotient, round to nearest even, saturating)
// so that the grouped GEMM can use the weight e4m3(q) * s.  This is weight
// preparation, run once per weight set, not part of a layer step.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kWarps = 8;

// Four fp32 values -> four e4m3 bytes, the first in the lowest byte.
__device__ __forceinline__ uint32_t f32x4_to_e4m3x4(float a, float b, float c, float d)
{
    uint32_t lo, hi;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(lo) : "f"(a), "f"(b));
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(hi) : "f"(c), "f"(d));
    return lo | (hi << 16);
}

// Largest magnitude of this thread's 8-element groups c = first, first + step, ... of a row.
__device__ __forceinline__ float row_amax_part(const uint16_t *__restrict__ w, int K, int first, int step)
{
    float amax = 0.0f;
    for (int c = first; c < K; c += step) {
        const uint4 v = *reinterpret_cast<const uint4 *>(w + c);
        const uint32_t p[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = unpack_bf16x2(p[i]);
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
    return amax;
}

// Codes of this thread's 8-element groups of a row, given the row's scale.
__device__ __forceinline__ void row_codes_part(const uint16_t *__restrict__ w, int K, int first, int step, float s,
                                               uint8_t *__restrict__ qr)
{
    for (int c = first; c < K; c += step) {
        const uint4 v = *reinterpret_cast<const uint4 *>(w + c);
        const float2 f0 = unpack_bf16x2(v.x), f1 = unpack_bf16x2(v.y), f2 = unpack_bf16x2(v.z),
                     f3 = unpack_bf16x2(v.w);
        uint2 o;
        o.x = f32x4_to_e4m3x4(__fdiv_rn(f0.x, s), __fdiv_rn(f0.y, s), __fdiv_rn(f1.x, s), __fdiv_rn(f1.y, s));
        o.y = f32x4_to_e4m3x4(__fdiv_rn(f2.x, s), __fdiv_rn(f2.y, s), __fdiv_rn(f3.x, s), __fdiv_rn(f3.y, s));
        *reinterpret_cast<uint2 *>(qr + c) = o;
    }
}

__device__ __forceinline__ float row_scale(float amax) { return amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f; }

// One warp per row (many rows); K is a multiple of 64, so each lane takes whole
// 8-element groups.
__global__ void __launch_bounds__(kWarps * 32)
    quantize_rows_kernel(const uint16_t *__restrict__ W, int64_t rows, int K, uint8_t *__restrict__ q,
                         float *__restrict__ scale)
{
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
    if (row >= rows) return;
    const uint16_t *w = W + row * K;
    float amax = row_amax_part(w, K, lane * 8, 256);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = row_scale(amax);
    if (lane == 0) scale[row] = s;
    row_codes_part(w, K, lane * 8, 256, s, q + row * K);
}

// One block of eight warps per row (few rows, e.g. a decode batch's activations):
// the same codes and scale, the row spread over eight times the threads.
__global__ void __launch_bounds__(kWarps * 32)
    quantize_rows_block_kernel(const uint16_t *__restrict__ W, int K, uint8_t *__restrict__ q,
                               float *__restrict__ scale)
{
    __shared__ float part[kWarps];
    pdl_entry();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t row = blockIdx.x;
    const uint16_t *w = W + row * K;
    float amax = row_amax_part(w, K, threadIdx.x * 8, kWarps * 256);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) part[warp] = amax;
    __syncthreads();
    amax = part[0];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) amax = fmaxf(amax, part[i]);
    const float s = row_scale(amax);
    if (threadIdx.x == 0) scale[row] = s;
    row_codes_part(w, K, threadIdx.x * 8, kWarps * 256, s, q + row * K);
}

}  // namespace

cudaError_t launch_quantize_fp8(const uint16_t *W, int64_t rows, int K, uint8_t *q, float *scale, cudaStream_t s)
{
    if (rows <= 0) return cudaSuccess;
    // a warp per row only once the rows fill every SM with blocks of eight warps
    if (rows < (int64_t)device_sm_count() * kWarps * 4 && rows < (int64_t)1 << 31)
        return launch_pdl(quantize_rows_block_kernel, dim3((unsigned)rows), dim3(kWarps * 32), 0, s, W, K, q, scale);
    return launch_pdl(quantize_rows_kernel, dim3((unsigned)((rows + kWarps - 1) / kWarps)), dim3(kWarps * 32), 0, s,
                      W, rows, K, q, scale);
}

}  // namespace moe
