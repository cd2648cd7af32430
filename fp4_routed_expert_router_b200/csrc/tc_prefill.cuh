// tc_prefill.cuh -- tcgen05 grouped GEMM path for large batches (prefill).
#pragma once
#include "common.cuh"
#include "decode_common.cuh"
#include "../../include/moe_fp4.h"

namespace moe {

struct TcPlan {
    int ready;
};

inline cudaError_t tc_plan_create(TcPlan* p, const moe_fp4_config&) { p->ready = 0; return cudaSuccess; }
inline void tc_plan_destroy(TcPlan*) {}
inline bool tc_prefers(int, const moe_fp4_config&) { return false; }
inline cudaError_t tc_forward(TcPlan*, const GemvArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace moe
