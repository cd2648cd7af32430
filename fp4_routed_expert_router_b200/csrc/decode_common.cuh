// decode_common.cuh -- arguments of the expert kernels and the small
// kernels around them: the router-weighted combine, per-entry output norms
// and the per-expert saliency.
//
// Per active expert e with M_e routed entries the layer needs
//   a1 = x W1^T, a3 = x W3^T  (W1, W3: [I, H]),  h = bf16(silu(a1) * a3),
//   o  = h W2^T               (W2: [H, I]),       y[t] = sum_j w[t, j] o[t, j]
// with W = E2M1 * 2^(s-127) (10100.com article 151357339, section
// "moe专家的容量瓶颈"; SwiGLU is the reading of the unnamed activation, the
// weighted sum of the expert outputs the reading of the combine).
#pragma once
#include "common.cuh"

namespace moe {

struct ExpertArgs {
    const uint8_t* arena;
    size_t slot_bytes;
    const int32_t* slot_table;   // [L][E]
    int layer, E, k, H, I;
    const uint16_t* x;           // [T, H] bf16
    const int32_t* offsets;      // [E+1]
    const int32_t* perm;         // [T*k]
    float* obuf;                 // [T*k, H] fp32, entry order t*k+j
    int* err;
};

// -------------------------------------------------------------------- combine
// y[t] = sum_j w[t, j] * o[t*k + j] in fixed j order; optional residual
// x_out = bf16_rne(x + y).  Four consecutive features per thread.
__global__ void __launch_bounds__(256) combine_kernel(const float* obuf, const float* w,
                                                       const uint16_t* x, int T, int H, int k,
                                                       float* y, uint16_t* x_out) {
    pdl_wait();
    pdl_trigger();
    const int H4 = H / 4;
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= T * H4) return;
    const int t = idx / H4, n4 = idx - t * H4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
        const float wj = __ldcg(w + t * k + j);
        const float4 o = __ldcg(reinterpret_cast<const float4*>(obuf + static_cast<size_t>(t * k + j) * H) + n4);
        acc.x = fmaf(wj, o.x, acc.x);
        acc.y = fmaf(wj, o.y, acc.y);
        acc.z = fmaf(wj, o.z, acc.z);
        acc.w = fmaf(wj, o.w, acc.w);
    }
    reinterpret_cast<float4*>(y + static_cast<size_t>(t) * H)[n4] = acc;
    if (x_out) {
        const uint2 xv = *reinterpret_cast<const uint2*>(x + static_cast<size_t>(t) * H + 4 * n4);
        const float r0 = bf16_to_f32(xv.x & 0xFFFF) + acc.x, r1 = bf16_to_f32(xv.x >> 16) + acc.y;
        const float r2 = bf16_to_f32(xv.y & 0xFFFF) + acc.z, r3 = bf16_to_f32(xv.y >> 16) + acc.w;
        uint2 ov;
        ov.x = static_cast<uint32_t>(f32_to_bf16_rne(r0)) | (static_cast<uint32_t>(f32_to_bf16_rne(r1)) << 16);
        ov.y = static_cast<uint32_t>(f32_to_bf16_rne(r2)) | (static_cast<uint32_t>(f32_to_bf16_rne(r3)) << 16);
        *reinterpret_cast<uint2*>(x_out + static_cast<size_t>(t) * H + 4 * n4) = ov;
    }
}

// ||o_p||_2 of each per-entry output row: one warp per row, lanes sum
// strided squares in index order, then a fixed xor tree (deterministic).
__global__ void __launch_bounds__(256) entry_norm_kernel(const float* obuf, int n_ent, int H, float* norms) {
    pdl_wait();
    pdl_trigger();
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (row >= n_ent) return;
    const float4* r = reinterpret_cast<const float4*>(obuf + static_cast<size_t>(row) * H);
    float s = 0.f;
    for (int i = lane; i < H / 4; i += 32) {
        const float4 v = __ldcg(r + i);
        s = fmaf(v.x, v.x, s);
        s = fmaf(v.y, v.y, s);
        s = fmaf(v.z, v.z, s);
        s = fmaf(v.w, v.w, s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane == 0) norms[row] = sqrtf(s);
}

// saliency[e] += sum over e's grouped entries of w * norm, in perm order, fp64.
// Offsets or entries outside [0, n_ent) (not a grouping of this batch) add nothing.
__global__ void __launch_bounds__(128) saliency_kernel(const float* norms, const float* w, const int32_t* offsets,
                                                       const int32_t* perm, int E, int n_ent, double* sal) {
    pdl_wait();
    pdl_trigger();
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int p0 = __ldg(offsets + e), p1 = __ldg(offsets + e + 1);
    if (p1 <= p0 || p0 < 0 || p1 > n_ent) return;
    double acc = 0.0;
    for (int p = p0; p < p1; ++p) {
        const int ent = __ldg(perm + p);
        if (ent < 0 || ent >= n_ent) continue;
        acc += static_cast<double>(__ldg(w + ent)) * static_cast<double>(norms[ent]);
    }
    sal[e] += acc;
}

}  // namespace moe
