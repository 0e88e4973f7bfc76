// common.cuh -- small device helpers shared by the MoE kernels (sm_100a only).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

// Record a device-side fault code (first writer wins) without trapping.
__device__ __forceinline__ void set_device_error(int *err, int code)
{
    if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b)
{
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Two packed bf16 (low half first in memory) -> two floats.
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t v)
{
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    return static_cast<uint32_t>(float_to_bf16_bits(lo)) |
           (static_cast<uint32_t>(float_to_bf16_bits(hi)) << 16);
}

// Programmatic dependent launch.  Every kernel of the layer lets the next kernel in the
// stream begin launching at once, then waits until the kernels it depends on have
// finished and their writes are visible -- before touching global memory, so no
// read-after-write or write-after-read hazard can cross the overlap.  What overlaps is
// launch latency and any prologue placed before the wait.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_entry()
{
    pdl_launch_dependents();
    pdl_wait();
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

}  // namespace moe
