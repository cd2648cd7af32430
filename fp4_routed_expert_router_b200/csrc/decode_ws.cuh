// decode_ws.cuh -- warp-specialised grouped FP4 GEMV (decode) for sm_100a.
//
// Arithmetic as in decode_gemv.cuh: W = E2M1 x 2^(s-127) decoded exactly to
// bf16 in registers (fp4_decode.cuh), multiplied by mma.sync m16n8k16 (bf16,
// fp32 accumulate) with A and B paired element for element along K; up
// computes a1 = x W1^T, a3 = x W3^T and h = bf16(silu(a1) * a3) (SwiGLU, the
// reading of the unnamed activation of the 10100.com article, section
// "moe专家的容量瓶颈"); down computes o = h W2^T.
//
// Organisation (one CTA per SM, persistent):
//  - one producer warp streams whole tiles (RB*16 rows of each matrix over the
//    full K, plus their UE8M0 scale rows) into a ring of shared-memory stages
//    with cp.async.bulk (TMA engine, no multicast, L2 evict-first); a `full`
//    mbarrier per stage counts the bytes, an `empty` mbarrier per stage counts
//    the consumer warps that are done with it;
//  - RB*KS consumer warps: warp w owns row block w / KS of the tile and the
//    K chunks (128 wide) ks, ks+KS, ... (ks = w % KS); it writes its partial
//    sums to a double-buffered array, releases the stage, and one named
//    barrier per tile later every warp reduces a share of the outputs in a
//    fixed order (results do not depend on the schedule);
//  - B fragments (x for up, h for down) are read through L1, so the warps of
//    an SM fetch each row from L2 once.
// `down` builds its work list and starts streaming w2 before it waits for
// `up` (programmatic dependent launch); work items are expert-major.
#pragma once
#include "common.cuh"
#include "decode_gemv.cuh"
#include "fp4_decode.cuh"
#include "tma.cuh"

namespace moe {

struct WsPlan {
    int stages;        // ring depth
    int rs;            // padded row stride in shared memory (bytes)
    int stage_bytes;   // bytes per stage (multiple of 128)
    int off_bars, off_lut, off_red, off_act, off_stage;   // byte offsets in dynamic smem
    int smem_bytes;
    int max_active;
};

__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <bool UP, int RB, int KS, int CPW>
__global__ void __launch_bounds__((RB * KS + 1) * 32, 1) gemv_ws_kernel(GemvArgs a, WsPlan p) {
    constexpr int NCW = RB * KS;                 // consumer warps
    constexpr int MATS = UP ? 2 : 1;
    constexpr int PART = MATS * 16 * 8;          // partial sums per consumer warp
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.off_bars);
    uint64_t* empty = full + p.stages;
    Fp4Lut* lut = reinterpret_cast<Fp4Lut*>(smem + p.off_lut);
    float* red = reinterpret_cast<float*>(smem + p.off_red);        // [2][NCW][PART]
    int* act = reinterpret_cast<int*>(smem + p.off_act);             // [4][max_active] + scratch
    __shared__ int n_act_s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = UP ? a.H : a.I;
    const int rows = UP ? a.I : a.H;
    const int rb = K / 2, sb = K / 32, rs = p.rs;
    const int TR = RB * 16;                       // rows per tile
    const int n_rt = rows / TR;
    const int E = a.E;

    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCW);
        }
    }
    fill_lut(lut);
    if (UP) pdl_wait();
    {   // active experts (ascending), first grouped position, count, slot
        int* offs_s = act + 4 * p.max_active;
        int* slot_s = offs_s + E + 1;
        for (int e = tid; e <= E; e += blockDim.x) {
            offs_s[e] = __ldcg(a.offsets + e);
            if (e < E) slot_s[e] = __ldcg(a.slot_table + static_cast<size_t>(a.layer) * E + e);
        }
        __syncthreads();
        if (warp == 0) {
            int n = 0;
            for (int base = 0; base < E; base += 32) {
                const int e = base + lane;
                const int o0 = (e < E) ? offs_s[e] : 0, o1 = (e < E) ? offs_s[e + 1] : 0;
                const bool on = (e < E) && (o1 > o0);
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, on);
                const int pos = n + __popc(ball & lanemask_lt());
                if (on && pos < p.max_active) {
                    act[pos] = e;
                    act[p.max_active + pos] = o0;
                    act[2 * p.max_active + pos] = o1 - o0;
                    act[3 * p.max_active + pos] = slot_s[e];
                }
                n += __popc(ball);
            }
            if (lane == 0) n_act_s = min(n, p.max_active);
        }
        if (tid == 0) fence_barrier_init();
        __syncthreads();
    }
    if (UP) pdl_trigger();
    const int n_tiles = n_act_s * n_rt;
    const int G = gridDim.x;
    const int my_tiles = (static_cast<int>(blockIdx.x) < n_tiles) ? (n_tiles - 1 - blockIdx.x) / G + 1 : 0;

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            for (int i = 0; i < my_tiles; ++i) {
                const int st = i % p.stages;
                if (i >= p.stages && !mbar_wait(&empty[st], ((i / p.stages) - 1) & 1)) {
                    latch_error(a.err, ERR_ETIMEOUT, i, UP ? KID_UP : KID_DOWN);
                    break;   // consumers time out on `full` as well
                }
                const int tau = blockIdx.x + i * G;
                const int ai = tau / n_rt, rt = tau - ai * n_rt;
                const int slot = act[3 * p.max_active + ai];
                uint8_t* dst = smem + p.off_stage + static_cast<size_t>(st) * p.stage_bytes;
                if (slot < 0) { mbar_arrive(&full[st]); continue; }
                const uint8_t* base = a.arena + static_cast<size_t>(slot) * a.slot_bytes;
                const size_t r0 = static_cast<size_t>(rt) * TR;
                mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(MATS * TR * (rb + sb)));
                if (UP) {
                    for (int r = 0; r < TR; ++r) bulk_g2s(dst + r * rs, base + (r0 + r) * rb, rb, &full[st], pol);
                    for (int r = 0; r < TR; ++r)
                        bulk_g2s(dst + (TR + r) * rs, base + a.off_w3 + (r0 + r) * rb, rb, &full[st], pol);
                    bulk_g2s(dst + 2 * TR * rs, base + a.off_s1 + r0 * sb, TR * sb, &full[st], pol);
                    bulk_g2s(dst + 2 * TR * rs + TR * sb, base + a.off_s3 + r0 * sb, TR * sb, &full[st], pol);
                } else {
                    for (int r = 0; r < TR; ++r)
                        bulk_g2s(dst + r * rs, base + a.off_w2 + (r0 + r) * rb, rb, &full[st], pol);
                    bulk_g2s(dst + TR * rs, base + a.off_s2 + r0 * sb, TR * sb, &full[st], pol);
                }
            }
        }
        return;   // the producer reads nothing that `up` writes
    }

    // ---------------------------------------------------------------- consumers
    if (!UP) { pdl_wait(); pdl_trigger(); }      // h of `up` is complete from here on
    const int g = lane >> 2, c = lane & 3;
    const int rbw = warp / KS, ks = warp - rbw * KS;
    int phase = 0;                               // named-barrier crossings so far
    for (int i = 0; i < my_tiles; ++i) {
        const int st = i % p.stages;
        const int tau = blockIdx.x + i * G;
        const int ai = tau / n_rt, rt = tau - ai * n_rt;
        const int e = act[ai], p0 = act[p.max_active + ai], m = act[2 * p.max_active + ai];
        const int slot = act[3 * p.max_active + ai];
        const int row0 = rt * TR;
        const uint8_t* stg = smem + p.off_stage + static_cast<size_t>(st) * p.stage_bytes;
        if (!mbar_wait(&full[st], (i / p.stages) & 1)) {
            // the tile never landed: report it and carry on through the same
            // barriers as the other warps (the outputs of this tile are garbage)
            if (lane == 0) latch_error(a.err, ERR_ETIMEOUT, tau, UP ? KID_UP : KID_DOWN);
        }
        if (slot < 0) {
            if (tid == 0) latch_error(a.err, ERR_ESLOT, e, UP ? KID_UP : KID_DOWN);
            for (int q = tid; q < m * TR; q += NCW * 32) {
                if (UP) {
                    a.hbuf[static_cast<size_t>(p0 + q / TR) * a.I + row0 + (q % TR)] = 0;
                } else {
                    const int ent = __ldg(a.perm + p0 + q / TR);
                    a.obuf[static_cast<size_t>(ent) * a.H + row0 + (q % TR)] = 0.f;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
            continue;
        }
        for (int g0 = 0; g0 < m; g0 += 8) {
            const int ng = min(8, m - g0);
            const uint16_t* brow;
            if (UP) {
                const int ent = __ldg(a.perm + p0 + g0 + min(g, ng - 1));
                brow = a.x + static_cast<size_t>(ent / a.k) * a.H + 32 * c;
            } else {
                brow = a.hbuf + static_cast<size_t>(p0 + g0 + min(g, ng - 1)) * a.I + 32 * c;
            }
            float d1[2][4] = {}, d3[2][4] = {};
            const uint8_t* rbase = stg + (rbw * 16 + g) * rs + 16 * c;
            const uint8_t* sbase = stg + MATS * TR * rs + (rbw * 16 + g) * sb + c;
#pragma unroll
            for (int j = 0; j < CPW; ++j) {
                const int kb = (ks + j * KS) * 128;
                uint4 X[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) X[q] = *reinterpret_cast<const uint4*>(brow + kb + 8 * q);
                const uint8_t* ra = rbase + kb / 2;
                const uint8_t* sa = sbase + kb / 32;
                const uint4 Aa = *reinterpret_cast<const uint4*>(ra);
                const uint4 Ab = *reinterpret_cast<const uint4*>(ra + 8 * rs);
                const Fp4Lut La = lut[sa[0]];
                const Fp4Lut Lb = lut[sa[8 * sb]];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t oa[4], ob[4];
                    fp4_decode8(word(Aa, w), La, oa);
                    fp4_decode8(word(Ab, w), Lb, ob);
                    mma_bf16_16816(d1[w & 1], oa[0], ob[0], oa[1], ob[1], word(X[w], 0), word(X[w], 1));
                    mma_bf16_16816(d1[w & 1], oa[2], ob[2], oa[3], ob[3], word(X[w], 2), word(X[w], 3));
                }
                if (UP) {
                    const uint4 Ca = *reinterpret_cast<const uint4*>(ra + TR * rs);
                    const uint4 Cb = *reinterpret_cast<const uint4*>(ra + (TR + 8) * rs);
                    const Fp4Lut Lc = lut[sa[TR * sb]];
                    const Fp4Lut Ld = lut[sa[(TR + 8) * sb]];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint32_t pa[4], pb[4];
                        fp4_decode8(word(Ca, w), Lc, pa);
                        fp4_decode8(word(Cb, w), Ld, pb);
                        mma_bf16_16816(d3[w & 1], pa[0], pb[0], pa[1], pb[1], word(X[w], 0), word(X[w], 1));
                        mma_bf16_16816(d3[w & 1], pa[2], pb[2], pa[3], pb[3], word(X[w], 2), word(X[w], 3));
                    }
                }
            }
            const bool last_group = (g0 + 8 >= m);
            if (last_group) {   // this warp no longer reads the stage
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
            const int buf = phase++ & 1;
            float* rw = red + (buf * NCW + warp) * PART;
            rw[g * 8 + 2 * c] = d1[0][0] + d1[1][0];
            rw[g * 8 + 2 * c + 1] = d1[0][1] + d1[1][1];
            rw[(g + 8) * 8 + 2 * c] = d1[0][2] + d1[1][2];
            rw[(g + 8) * 8 + 2 * c + 1] = d1[0][3] + d1[1][3];
            if (UP) {
                rw[128 + g * 8 + 2 * c] = d3[0][0] + d3[1][0];
                rw[128 + g * 8 + 2 * c + 1] = d3[0][1] + d3[1][1];
                rw[128 + (g + 8) * 8 + 2 * c] = d3[0][2] + d3[1][2];
                rw[128 + (g + 8) * 8 + 2 * c + 1] = d3[0][3] + d3[1][3];
            }
            named_barrier(1, NCW * 32);
            // reduce: RB*128 outputs (row, token), KS partials each, fixed order
            for (int q = tid; q < RB * 128; q += NCW * 32) {
                const int r = q >> 7, o = q & 127, row = o >> 3, tk = o & 7;
                if (tk < ng) {
                    const float* src = red + (buf * NCW + r * KS) * PART + o;
                    float s1 = 0.f, s3 = 0.f;
#pragma unroll
                    for (int k2 = 0; k2 < KS; ++k2) {
                        s1 += src[k2 * PART];
                        if (UP) s3 += src[k2 * PART + 128];
                    }
                    if (UP) {
                        const float hv = s1 / (1.0f + expf(-s1)) * s3;
                        a.hbuf[static_cast<size_t>(p0 + g0 + tk) * a.I + row0 + r * 16 + row] = f32_to_bf16_rne(hv);
                    } else {
                        const int ent = __ldg(a.perm + p0 + g0 + tk);
                        a.obuf[static_cast<size_t>(ent) * a.H + row0 + r * 16 + row] = s1;
                    }
                }
            }
        }
    }
}

// Host-side plan; stages = 0 when the shape does not fit.
inline WsPlan make_ws_plan(bool up, int H, int I, int n_experts, int max_active, int rbk, int ncw,
                           int smem_limit) {
    WsPlan p{};
    const int K = up ? H : I;
    const int rb = K / 2, sb = K / 32, mats = up ? 2 : 1, tr = 16 * rbk;
    p.rs = (rb % 128 == 0) ? rb + 64 : rb;
    p.stage_bytes = (mats * tr * (p.rs + sb) + 127) / 128 * 128;
    p.max_active = max_active;
    p.off_bars = 0;                                   // 2 * 16 barriers at most
    p.off_lut = 256;
    p.off_red = p.off_lut + 256 * 16;
    p.off_act = p.off_red + 2 * ncw * mats * 128 * 4;
    p.off_stage = (p.off_act + 16 * max_active + 8 * (n_experts + 1) + 127) / 128 * 128;
    int stages = (smem_limit - p.off_stage) / p.stage_bytes;
    if (stages > 16) stages = 16;
    p.stages = stages >= 2 ? stages : 0;
    p.smem_bytes = p.off_stage + p.stages * p.stage_bytes;
    return p;
}

}  // namespace moe
