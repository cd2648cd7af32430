// decode_common.cuh -- pieces shared by the decode kernels: arguments, the
// mma.sync wrapper, the per-scale decode tables, and the combine kernel.
//
// Per active expert e with M_e routed entries the layer needs
//   a1 = x W1^T, a3 = x W3^T  (W1, W3: [I, H]),  h = bf16(silu(a1) * a3),
//   o  = h W2^T               (W2: [H, I]),
// with W = E2M1 * 2^(s-127) (10100.com article 151357339, section
// "moe专家的容量瓶颈"; SwiGLU is the reading of the unnamed activation).
// At decode the weights are read once per step and the work is bound by HBM;
// the decode kernels turn FP4 codes into exact bf16 in registers
// (fp4_decode.cuh) and let the tensor cores do the multiply-adds through
// mma.sync.m16n8k16 (bf16 in, fp32 accumulate): one MMA covers 16 weight rows
// x 16 K x 8 tokens, so up to 8 tokens of an expert share each decoded weight.
//
// K order inside an MMA is free as long as A and B agree: lane (g, c) of a
// warp takes the 32 codes K = kb+32c .. kb+32c+31 of rows g and g+8 (one
// 16-byte vector and one scale byte each) and uses codes 4i..4i+3 in MMA step
// i (i = 0..7); its B fragment is x[token g][kb+32c+4i .. +3], so a 16x128
// weight chunk and a 128-long x slice pair up element for element.
#pragma once
#include "common.cuh"
#include "fp4_decode.cuh"

namespace moe {

struct GemvArgs {
    const uint8_t* arena;
    size_t slot_bytes;
    const int32_t* slot_table;   // [L][E]
    int layer, E, k, H, I;
    const uint16_t* x;           // [T, H] bf16
    const int32_t* offsets;      // [E+1]
    const int32_t* perm;         // [T*k]
    uint16_t* hbuf;              // [T*k, I] bf16, grouped position order
    float* obuf;                 // [T*k, H] fp32, entry order t*k+j
    int* err;
};

__device__ __forceinline__ void mma_bf16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void fill_lut(Fp4Lut* lut) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lut[i] = make_fp4_lut(static_cast<uint32_t>(i));
}

__device__ __forceinline__ uint32_t word(const uint4& v, int j) {
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

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
__global__ void __launch_bounds__(128) saliency_kernel(const float* norms, const float* w, const int32_t* offsets,
                                                       const int32_t* perm, int E, double* sal) {
    pdl_wait();
    pdl_trigger();
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int p0 = __ldg(offsets + e), p1 = __ldg(offsets + e + 1);
    if (p1 <= p0) return;
    double acc = 0.0;
    for (int p = p0; p < p1; ++p) {
        const int ent = __ldg(perm + p);
        acc += static_cast<double>(__ldg(w + ent)) * static_cast<double>(norms[ent]);
    }
    sal[e] += acc;
}

}  // namespace moe
