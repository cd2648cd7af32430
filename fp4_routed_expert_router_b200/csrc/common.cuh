// common.cuh -- shared device helpers of libmoe_fp4: error word, programmatic
// dependent launch (PDL) controls, bf16 helpers, small PTX wrappers.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace moe {

// Error word layout (device int32[4]): [0] first status latched, [1] detail
// (expert / layer / byte index), [2] kernel id, [3] reserved.
enum : int { ERR_OK = 0, ERR_EINVAL = 1, ERR_ESLOT = 4, ERR_ETIMEOUT = 5 };
enum : int { KID_ROUTE = 1, KID_LOAD = 2, KID_UP = 3, KID_DOWN = 4, KID_COMBINE = 5,
             KID_TC_UP = 6, KID_TC_DOWN = 7, KID_GATHER = 8 };

__device__ __forceinline__ void latch_error(int* err, int code, int detail, int kid) {
    if (atomicCAS(err, 0, code) == 0) {
        err[1] = detail;
        err[2] = kid;
    }
}

// Programmatic dependent launch.  Every kernel of a chain waits for its
// predecessor before touching data the predecessor wrote, and lets its own
// dependent start launching once it no longer gates it.  Without the launch
// attribute both instructions are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Coherent L2 load for data written earlier in the same grid (no L1).
__device__ __forceinline__ int ld_cg(const int* p) { return __ldcg(p); }

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace moe
