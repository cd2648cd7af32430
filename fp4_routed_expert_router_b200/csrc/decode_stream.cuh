// decode_stream.cuh -- persistent grouped FP4 GEMV with bulk-copy staging.
//
// Same arithmetic as decode_gemv.cuh (exact E2M1 x 2^(s-127) -> bf16 decode in
// registers, mma.sync m16n8k16 bf16 with fp32 accumulate, K order paired
// between A and B), organised for HBM streaming on B200:
//  - one CTA per SM walks a static list of (active expert, 16-row tile)
//    work items (tile = 16 rows of w1 AND of w3 for `up`, 16 rows of w2 for
//    `down`, plus the rows' UE8M0 scales);
//  - one thread streams each tile into a ring of shared-memory stages with
//    cp.async.bulk (the TMA engine, no multicast, L2 evict-first), signalled
//    by an mbarrier per stage, several tiles ahead of the math;
//  - rows land with a padded stride so that the 16-byte fragment loads of the
//    two 8-row halves hit disjoint banks;
//  - every warp prefetches its x (or h) fragments for the whole tile into
//    registers before it waits for the tile's weights;
//  - `down` builds its work list and starts streaming w2 before it waits on
//    `up` (programmatic dependent launch), so the w2 stream overlaps the tail
//    of `up`.
// Work items are ordered expert-major; the per-tile reduction across warps
// runs in a fixed order, so results do not depend on the schedule.
#pragma once
#include "common.cuh"
#include "decode_gemv.cuh"
#include "fp4_decode.cuh"
#include "tma.cuh"

namespace moe {

// Shared-memory plan of one stream kernel (computed on the host).
struct StreamPlan {
    int stages;        // ring depth
    int rs;            // padded row stride in shared memory (bytes)
    int stage_bytes;   // bytes per stage (multiple of 128)
    int off_lut, off_red, off_act, off_stage;   // byte offsets in dynamic smem
    int smem_bytes;    // total dynamic smem
    int max_active;    // capacity of the active-expert list
};

__host__ __device__ inline int stream_row_stride(int rb) {
    return (rb % 128 == 0) ? rb + 64 : rb;   // rb is a multiple of 64
}

template <bool UP, int NW, int MAXC>
__global__ void __launch_bounds__(NW * 32, 1) gemv_stream_kernel(GemvArgs a, StreamPlan p) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    Fp4Lut* lut = reinterpret_cast<Fp4Lut*>(smem + p.off_lut);
    float* red = reinterpret_cast<float*>(smem + p.off_red);   // [NW][UP?2:1][16][8]
    int* act = reinterpret_cast<int*>(smem + p.off_act);        // [4][max_active]: e, p0, m, slot; then scratch
    __shared__ int n_act_s;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int K = UP ? a.H : a.I;                 // reduction length
    const int rows = UP ? a.I : a.H;              // output rows
    const int rb = K / 2, sb = K / 32, rs = p.rs;
    const int n_rt = rows / 16, nchunks = K / 128;
    const int E = a.E;

    if (tid == 0)
        for (int s = 0; s < p.stages; ++s) mbar_init(&bars[s], 1);
    fill_lut(lut);
    if (UP) pdl_wait();
    // active experts (ascending), their first position, count and slot: the
    // offsets and the layer's slot-table row are fetched by all threads at
    // once (one memory latency), then warp 0 compacts them from shared memory
    int* offs_s = act + 4 * p.max_active;            // [E+1]
    int* slot_s = offs_s + E + 1;                    // [E]
    for (int e = tid; e <= E; e += NW * 32) {
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
    if (UP) pdl_trigger();
    const int n_act = n_act_s;
    const int n_tiles = n_act * n_rt;
    const int G = gridDim.x;
    const int my_tiles = (static_cast<int>(blockIdx.x) < n_tiles) ? (n_tiles - 1 - blockIdx.x) / G + 1 : 0;
    const uint64_t pol = policy_evict_first();

    auto stage_ptr = [&](int st) { return smem + p.off_stage + static_cast<size_t>(st) * p.stage_bytes; };
    auto issue = [&](int i) {   // thread 0: stream local tile i into stage i % stages
        const int tau = blockIdx.x + i * G;
        const int ai = tau / n_rt, rt = tau - ai * n_rt;
        const int slot = act[3 * p.max_active + ai];
        uint64_t* bar = &bars[i % p.stages];
        uint8_t* dst = stage_ptr(i % p.stages);
        if (slot < 0) { mbar_arrive(bar); return; }
        const uint8_t* base = a.arena + static_cast<size_t>(slot) * a.slot_bytes;
        const size_t r0 = static_cast<size_t>(rt) * 16;
        if (UP) {
            mbar_arrive_expect_tx(bar, 32u * rb + 32u * sb);
            for (int r = 0; r < 16; ++r) bulk_g2s(dst + r * rs, base + (r0 + r) * rb, rb, bar, pol);
            for (int r = 0; r < 16; ++r)
                bulk_g2s(dst + (16 + r) * rs, base + a.off_w3 + (r0 + r) * rb, rb, bar, pol);
            bulk_g2s(dst + 32 * rs, base + a.off_s1 + r0 * sb, 16 * sb, bar, pol);
            bulk_g2s(dst + 32 * rs + 16 * sb, base + a.off_s3 + r0 * sb, 16 * sb, bar, pol);
        } else {
            mbar_arrive_expect_tx(bar, 16u * rb + 16u * sb);
            for (int r = 0; r < 16; ++r)
                bulk_g2s(dst + r * rs, base + a.off_w2 + (r0 + r) * rb, rb, bar, pol);
            bulk_g2s(dst + 16 * rs, base + a.off_s2 + r0 * sb, 16 * sb, bar, pol);
        }
    };
    if (tid == 0)
        for (int i = 0; i < my_tiles && i < p.stages; ++i) issue(i);
    if (!UP) {
        pdl_wait();      // h of `up` is complete from here on
        pdl_trigger();
    }

    for (int i = 0; i < my_tiles; ++i) {
        const int tau = blockIdx.x + i * G;
        const int ai = tau / n_rt, rt = tau - ai * n_rt;
        const int e = act[ai], p0 = act[p.max_active + ai], m = act[2 * p.max_active + ai];
        const int slot = act[3 * p.max_active + ai];
        const int row0 = rt * 16;
        const uint8_t* stg = stage_ptr(i % p.stages);
        const bool landed = mbar_wait(&bars[i % p.stages], (i / p.stages) & 1);
        if (!__syncthreads_and(landed)) {   // CTA-uniform give-up after the bounded wait
            if (tid == 0) latch_error(a.err, ERR_ETIMEOUT, tau, UP ? KID_UP : KID_DOWN);
            return;
        }
        if (slot < 0) {
            if (tid == 0) latch_error(a.err, ERR_ESLOT, e, UP ? KID_UP : KID_DOWN);
            for (int q = tid; q < m * 16; q += NW * 32) {
                if (UP) {
                    a.hbuf[static_cast<size_t>(p0 + q / 16) * a.I + row0 + (q & 15)] = 0;
                } else {
                    const int ent = __ldg(a.perm + p0 + q / 16);
                    a.obuf[static_cast<size_t>(ent) * a.H + row0 + (q & 15)] = 0.f;
                }
            }
        } else {
            for (int g0 = 0; g0 < m; g0 += 8) {
                const int ng = min(8, m - g0);
                // B fragments for this warp's chunks: x rows (up) or h rows (down)
                const uint16_t* brow;
                if (UP) {
                    const int ent = __ldg(a.perm + p0 + g0 + min(g, ng - 1));
                    brow = a.x + static_cast<size_t>(ent / a.k) * a.H + 32 * c;
                } else {
                    brow = a.hbuf + static_cast<size_t>(p0 + g0 + min(g, ng - 1)) * a.I + 32 * c;
                }
                uint4 X[MAXC][4];
#pragma unroll
                for (int j = 0; j < MAXC; ++j) {
                    const int ch = warp + j * NW;
                    if (ch < nchunks) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            X[j][q] = __ldcg(reinterpret_cast<const uint4*>(brow + ch * 128 + 8 * q));
                    }
                }
                float d1[4] = {0.f, 0.f, 0.f, 0.f}, d3[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < MAXC; ++j) {
                    const int ch = warp + j * NW;
                    if (ch >= nchunks) break;
                    const int kb = ch * 128;
                    const uint8_t* ra = stg + g * rs + kb / 2 + 16 * c;
                    const uint8_t* sa = stg + (UP ? 32 : 16) * rs + g * sb + kb / 32 + c;
                    const uint4 Aa = *reinterpret_cast<const uint4*>(ra);
                    const uint4 Ab = *reinterpret_cast<const uint4*>(ra + 8 * rs);
                    const Fp4Lut La = lut[sa[0]];
                    const Fp4Lut Lb = lut[sa[8 * sb]];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint32_t oa[4], ob[4];
                        fp4_decode8(word(Aa, w), La, oa);
                        fp4_decode8(word(Ab, w), Lb, ob);
                        mma_bf16_16816(d1, oa[0], ob[0], oa[1], ob[1], word(X[j][w], 0), word(X[j][w], 1));
                        mma_bf16_16816(d1, oa[2], ob[2], oa[3], ob[3], word(X[j][w], 2), word(X[j][w], 3));
                    }
                    if (UP) {
                        const uint4 Ca = *reinterpret_cast<const uint4*>(ra + 16 * rs);
                        const uint4 Cb = *reinterpret_cast<const uint4*>(ra + 24 * rs);
                        const Fp4Lut Lc = lut[sa[16 * sb]];
                        const Fp4Lut Ld = lut[sa[24 * sb]];
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            uint32_t pa[4], pb[4];
                            fp4_decode8(word(Ca, w), Lc, pa);
                            fp4_decode8(word(Cb, w), Ld, pb);
                            mma_bf16_16816(d3, pa[0], pb[0], pa[1], pb[1], word(X[j][w], 0), word(X[j][w], 1));
                            mma_bf16_16816(d3, pa[2], pb[2], pa[3], pb[3], word(X[j][w], 2), word(X[j][w], 3));
                        }
                    }
                }
                float* rw = red + warp * (UP ? 256 : 128);
                rw[g * 8 + 2 * c] = d1[0];
                rw[g * 8 + 2 * c + 1] = d1[1];
                rw[(g + 8) * 8 + 2 * c] = d1[2];
                rw[(g + 8) * 8 + 2 * c + 1] = d1[3];
                if (UP) {
                    rw[128 + g * 8 + 2 * c] = d3[0];
                    rw[128 + g * 8 + 2 * c + 1] = d3[1];
                    rw[128 + (g + 8) * 8 + 2 * c] = d3[2];
                    rw[128 + (g + 8) * 8 + 2 * c + 1] = d3[3];
                }
                __syncthreads();
                for (int q = tid; q < 128; q += NW * 32) {
                    const int row = q >> 3, tk = q & 7;
                    if (tk < ng) {
                        float s1 = 0.f, s3 = 0.f;
#pragma unroll
                        for (int w = 0; w < NW; ++w) {
                            s1 += red[w * (UP ? 256 : 128) + q];
                            if (UP) s3 += red[w * 256 + 128 + q];
                        }
                        if (UP) {
                            const float hv = s1 / (1.0f + expf(-s1)) * s3;
                            a.hbuf[static_cast<size_t>(p0 + g0 + tk) * a.I + row0 + row] = f32_to_bf16_rne(hv);
                        } else {
                            const int ent = __ldg(a.perm + p0 + g0 + tk);
                            a.obuf[static_cast<size_t>(ent) * a.H + row0 + row] = s1;
                        }
                    }
                }
                __syncthreads();
            }
        }
        __syncthreads();   // every warp is done with this stage
        if (tid == 0 && i + p.stages < my_tiles) issue(i + p.stages);
    }
}

// Host-side plan for a stream kernel; stages = 0 when the shape does not fit.
inline StreamPlan make_stream_plan(bool up, int H, int I, int n_experts, int max_active, int nw,
                                   int smem_limit) {
    StreamPlan p{};
    const int K = up ? H : I;
    const int rb = K / 2, sb = K / 32;
    p.rs = stream_row_stride(rb);
    const int raw = up ? 32 * p.rs + 32 * sb : 16 * p.rs + 16 * sb;
    p.stage_bytes = (raw + 127) / 128 * 128;
    p.max_active = max_active;
    p.off_lut = 128;
    p.off_red = p.off_lut + 256 * 16;
    p.off_act = p.off_red + nw * (up ? 256 : 128) * 4;
    p.off_stage = (p.off_act + 16 * max_active + 8 * (n_experts + 1) + 127) / 128 * 128;
    int stages = (smem_limit - p.off_stage) / p.stage_bytes;
    if (stages > 12) stages = 12;
    p.stages = stages >= 2 ? stages : 0;
    p.smem_bytes = p.off_stage + p.stages * p.stage_bytes;
    return p;
}

}  // namespace moe
