// decode_gemv.cuh -- grouped FP4 GEMV for small batches (decode).
//
// Per active expert e with M_e routed entries the layer needs
//   a1 = x W1^T, a3 = x W3^T  (W1, W3: [I, H]),  h = bf16(silu(a1) * a3),
//   o  = h W2^T               (W2: [H, I]),
// with W = E2M1 * 2^(s-127) (10100.com article 151357339, section
// "moe专家的容量瓶颈"; SwiGLU is the reading of the unnamed activation).
// At decode the weights are read once per step and the work is bound by HBM,
// so the kernels stream 16-byte code vectors straight into registers, decode
// them exactly to bf16 (fp4_decode.cuh) and let the tensor cores do the
// multiply-adds through mma.sync.m16n8k16 (bf16 in, fp32 accumulate): one MMA
// covers 16 weight rows x 16 K x 8 tokens, so decode, not arithmetic, is the
// per-weight cost and up to 8 tokens of an expert share each decoded weight.
//
// K order inside an MMA is free as long as A and B agree: lane (g, c) of a
// warp loads the 32 codes K = kb+32c .. kb+32c+31 of rows g and g+8 (one
// 16-byte vector and one scale byte each), and uses codes 4i..4i+3 in MMA
// step i (i = 0..7); its B fragment is x[token g][kb+32c+4i .. +3], so the
// 16x128 weight tile and the 128-long x slice pair up element for element.
//
// Work split: one CTA per (16-row tile, active expert); its warps take the
// 128-wide K chunks round robin and reduce through shared memory in a fixed
// order (deterministic).  Up (w1/w3 + SwiGLU) writes h rows at the entry's
// grouped position; down (w2) writes fp32 rows of o at entry index t*k+j.
#pragma once
#include "common.cuh"
#include "fp4_decode.cuh"

namespace moe {

struct GemvArgs {
    const uint8_t* arena;
    size_t slot_bytes;
    size_t off_w3, off_w2, off_s1, off_s3, off_s2;
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

// a-th active expert (offsets[e+1] > offsets[e]) found by warp 0, or -1.
__device__ __forceinline__ int find_active_expert(const int32_t* offsets, int E, int a) {
    const int lane = threadIdx.x & 31;
    for (int base = 0; base < E; base += 32) {
        int e = base + lane;
        bool act = (e < E) && (__ldg(offsets + e + 1) > __ldg(offsets + e));
        uint32_t ball = __ballot_sync(0xFFFFFFFFu, act);
        int cnt = __popc(ball);
        if (a < cnt) {   // warp-uniform: the lane holding the a-th set bit answers
            uint32_t hit = __ballot_sync(0xFFFFFFFFu, act && __popc(ball & lanemask_lt()) == a);
            return base + __ffs(hit) - 1;
        }
        a -= cnt;
    }
    return -1;
}

struct ExpertJob {
    int e, p0, m, slot;
};

__device__ __forceinline__ ExpertJob locate_job(const GemvArgs& a, ExpertJob* sm) {
    if (threadIdx.x < 32) {
        int e = find_active_expert(a.offsets, a.E, blockIdx.y);
        if (threadIdx.x == 0) {
            ExpertJob j{e, 0, 0, -1};
            if (e >= 0) {
                j.p0 = __ldg(a.offsets + e);
                j.m = __ldg(a.offsets + e + 1) - j.p0;
                j.slot = __ldg(a.slot_table + static_cast<size_t>(a.layer) * a.E + e);
            }
            *sm = j;
        }
    }
    __syncthreads();
    return *sm;
}

__device__ __forceinline__ void fill_lut(Fp4Lut* lut) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) lut[i] = make_fp4_lut(static_cast<uint32_t>(i));
}

__device__ __forceinline__ uint32_t word(const uint4& v, int j) {
    return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// -------------------------------------------------------------------- up
template <int NW>
__global__ void __launch_bounds__(NW * 32) gemv_up_kernel(GemvArgs a) {
    __shared__ Fp4Lut lut[256];
    __shared__ float red[NW][2][16][8];
    __shared__ ExpertJob job_s;
    fill_lut(lut);
    pdl_wait();
    const ExpertJob job = locate_job(a, &job_s);
    pdl_trigger();
    if (job.e < 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int row0 = blockIdx.x * 16;
    const int H = a.H, I = a.I;
    if (job.slot < 0) {
        if (threadIdx.x == 0) latch_error(a.err, ERR_ESLOT, job.e, KID_UP);
        for (int i = threadIdx.x; i < job.m * 16; i += blockDim.x)
            a.hbuf[static_cast<size_t>(job.p0 + i / 16) * I + row0 + (i & 15)] = 0;
        return;
    }
    const uint8_t* base = a.arena + static_cast<size_t>(job.slot) * a.slot_bytes;
    const size_t rb = H / 2, sb = H / 32;
    const uint8_t* w1a = base + static_cast<size_t>(row0 + g) * rb + 16 * c;
    const uint8_t* w3a = base + a.off_w3 + static_cast<size_t>(row0 + g) * rb + 16 * c;
    const uint8_t* s1a = base + a.off_s1 + static_cast<size_t>(row0 + g) * sb + c;
    const uint8_t* s3a = base + a.off_s3 + static_cast<size_t>(row0 + g) * sb + c;
    const int nchunks = H / 128;
    __syncthreads();   // lut ready
    for (int g0 = 0; g0 < job.m; g0 += 8) {
        const int ng = min(8, job.m - g0);
        const int ent = __ldg(a.perm + job.p0 + g0 + min(g, ng - 1));
        const uint16_t* xr = a.x + static_cast<size_t>(ent / a.k) * H + 32 * c;
        float d1[4] = {0.f, 0.f, 0.f, 0.f}, d3[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ch = warp; ch < nchunks; ch += NW) {
            const int kb = ch * 128;
            const uint4 A1a = ldg_stream(w1a + kb / 2);
            const uint4 A1b = ldg_stream(w1a + 8 * rb + kb / 2);
            const uint4 A3a = ldg_stream(w3a + kb / 2);
            const uint4 A3b = ldg_stream(w3a + 8 * rb + kb / 2);
            const Fp4Lut L1a = lut[__ldg(s1a + kb / 32)];
            const Fp4Lut L1b = lut[__ldg(s1a + 8 * sb + kb / 32)];
            const Fp4Lut L3a = lut[__ldg(s3a + kb / 32)];
            const Fp4Lut L3b = lut[__ldg(s3a + 8 * sb + kb / 32)];
            uint4 X[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) X[q] = ldg_cached(xr + kb + 8 * q);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t oa[4], ob[4], pa[4], pb[4];
                fp4_decode8(word(A1a, j), L1a, oa);
                fp4_decode8(word(A1b, j), L1b, ob);
                fp4_decode8(word(A3a, j), L3a, pa);
                fp4_decode8(word(A3b, j), L3b, pb);
                const uint32_t b00 = word(X[j], 0), b01 = word(X[j], 1);
                const uint32_t b10 = word(X[j], 2), b11 = word(X[j], 3);
                mma_bf16_16816(d1, oa[0], ob[0], oa[1], ob[1], b00, b01);
                mma_bf16_16816(d1, oa[2], ob[2], oa[3], ob[3], b10, b11);
                mma_bf16_16816(d3, pa[0], pb[0], pa[1], pb[1], b00, b01);
                mma_bf16_16816(d3, pa[2], pb[2], pa[3], pb[3], b10, b11);
            }
        }
        red[warp][0][g][2 * c] = d1[0];
        red[warp][0][g][2 * c + 1] = d1[1];
        red[warp][0][g + 8][2 * c] = d1[2];
        red[warp][0][g + 8][2 * c + 1] = d1[3];
        red[warp][1][g][2 * c] = d3[0];
        red[warp][1][g][2 * c + 1] = d3[1];
        red[warp][1][g + 8][2 * c] = d3[2];
        red[warp][1][g + 8][2 * c + 1] = d3[3];
        __syncthreads();
        for (int i = threadIdx.x; i < 128; i += NW * 32) {
            const int row = i >> 3, tk = i & 7;
            if (tk < ng) {
                float a1 = 0.f, a3 = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) { a1 += red[w][0][row][tk]; a3 += red[w][1][row][tk]; }
                const float hv = a1 / (1.0f + expf(-a1)) * a3;
                a.hbuf[static_cast<size_t>(job.p0 + g0 + tk) * I + row0 + row] = f32_to_bf16_rne(hv);
            }
        }
        __syncthreads();
    }
}

// -------------------------------------------------------------------- down
template <int NW>
__global__ void __launch_bounds__(NW * 32) gemv_down_kernel(GemvArgs a) {
    __shared__ Fp4Lut lut[256];
    __shared__ float red[NW][16][8];
    __shared__ ExpertJob job_s;
    fill_lut(lut);
    pdl_wait();
    const ExpertJob job = locate_job(a, &job_s);
    pdl_trigger();
    if (job.e < 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int row0 = blockIdx.x * 16;
    const int H = a.H, I = a.I;
    if (job.slot < 0) {
        if (threadIdx.x == 0) latch_error(a.err, ERR_ESLOT, job.e, KID_DOWN);
        for (int i = threadIdx.x; i < job.m * 16; i += blockDim.x) {
            const int ent = __ldg(a.perm + job.p0 + i / 16);
            a.obuf[static_cast<size_t>(ent) * H + row0 + (i & 15)] = 0.f;
        }
        return;
    }
    const uint8_t* base = a.arena + static_cast<size_t>(job.slot) * a.slot_bytes;
    const size_t rb = I / 2, sb = I / 32;
    const uint8_t* w2a = base + a.off_w2 + static_cast<size_t>(row0 + g) * rb + 16 * c;
    const uint8_t* s2a = base + a.off_s2 + static_cast<size_t>(row0 + g) * sb + c;
    const int nchunks = I / 128;
    __syncthreads();
    for (int g0 = 0; g0 < job.m; g0 += 8) {
        const int ng = min(8, job.m - g0);
        const uint16_t* hr = a.hbuf + static_cast<size_t>(job.p0 + g0 + min(g, ng - 1)) * I + 32 * c;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        for (int ch = warp; ch < nchunks; ch += NW) {
            const int kb = ch * 128;
            const uint4 Aa = ldg_stream(w2a + kb / 2);
            const uint4 Ab = ldg_stream(w2a + 8 * rb + kb / 2);
            const Fp4Lut La = lut[__ldg(s2a + kb / 32)];
            const Fp4Lut Lb = lut[__ldg(s2a + 8 * sb + kb / 32)];
            uint4 X[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) X[q] = __ldcg(reinterpret_cast<const uint4*>(hr + kb + 8 * q));
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t oa[4], ob[4];
                fp4_decode8(word(Aa, j), La, oa);
                fp4_decode8(word(Ab, j), Lb, ob);
                mma_bf16_16816(d, oa[0], ob[0], oa[1], ob[1], word(X[j], 0), word(X[j], 1));
                mma_bf16_16816(d, oa[2], ob[2], oa[3], ob[3], word(X[j], 2), word(X[j], 3));
            }
        }
        red[warp][g][2 * c] = d[0];
        red[warp][g][2 * c + 1] = d[1];
        red[warp][g + 8][2 * c] = d[2];
        red[warp][g + 8][2 * c + 1] = d[3];
        __syncthreads();
        for (int i = threadIdx.x; i < 128; i += NW * 32) {
            const int row = i >> 3, tk = i & 7;
            if (tk < ng) {
                float o = 0.f;
#pragma unroll
                for (int w = 0; w < NW; ++w) o += red[w][row][tk];
                const int ent = __ldg(a.perm + job.p0 + g0 + tk);
                a.obuf[static_cast<size_t>(ent) * H + row0 + row] = o;
            }
        }
        __syncthreads();
    }
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

}  // namespace moe
