// decode_tile.cuh -- grouped FP4 GEMV for decode batches: one persistent CTA
// per SM, whole 16-row tiles streamed by a producer warp, K split across the
// consumer warps.
//
// Arithmetic as in decode_common.cuh (exact FP4 -> bf16 register decode,
// mma.sync m16n8k16 bf16 / fp32 accumulate):
//   up    a1 = x W1^T, a3 = x W3^T, h = bf16(silu(a1) * a3)      (SwiGLU)
//   down  o = h W2^T
// Work items are (active expert, tile of TR = 16*RB weight rows, group of
// <= 8 of the expert's tokens), handed out round robin to the CTAs.  In the
// slot layout (slot_layout.cuh) the blocks of one tile are consecutive, so a
// tile (w1 + w3 + their scales over all of H for up: 87,040 bytes; 32 rows of
// w2 + scales for down: 39,168 bytes) is ONE cp.async.bulk (TMA engine; no
// multicast; L2 evict-first) into a ring of shared-memory stages.  A `full`
// mbarrier per stage counts its bytes; an `empty` mbarrier per stage counts
// the consumer warps done with it, which lets the producer warp refill it.
// Every consumer warp reads every tile (in order), so a wait on a stage's
// phase is never ambiguous.  Consumer warp w owns row block w / KS of the
// tile and the CPW consecutive 128-wide K chunks starting at (w % KS) * CPW;
// partial sums meet in shared memory and are reduced in a fixed order after
// one named barrier per tile (double-buffered), so results never depend on
// the schedule.  B fragments (x or h rows) are prefetched into registers
// before the tile's bytes are awaited.  Every wait is bounded; the first one
// that gives up makes the others return at once (MOE_FP4_ETIMEOUT).
#pragma once
#include "common.cuh"
#include "decode_common.cuh"
#include "fp4_decode.cuh"
#include "slot_layout.cuh"
#include "tma.cuh"

namespace moe {

struct TilePlan {
    int stages;
    int stage_bytes;
    int off_lut, off_red, off_act, off_stage;
    int smem_bytes;
    int max_active;
};

__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <bool UP, int RB, int KS, int CPW>
__global__ void __launch_bounds__((RB * KS + 1) * 32, 1) gemv_tile_kernel(GemvArgs a, SlotLayout L, TilePlan p) {
    constexpr int NCW = RB * KS;                 // consumer warps
    constexpr int MATS = UP ? 2 : 1;
    constexpr int PART = MATS * 128;             // partial sums per consumer warp (16 rows x 8 tokens each)
    constexpr int TR = 16 * RB;                  // weight rows per tile
    extern __shared__ __align__(128) uint8_t smem[];   // 128-byte alignment is all the row swizzle needs
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + p.stages;
    Fp4Lut* lut = reinterpret_cast<Fp4Lut*>(smem + p.off_lut);
    float* red = reinterpret_cast<float*>(smem + p.off_red);             // [2][NCW][PART]
    int* act_e = reinterpret_cast<int*>(smem + p.off_act);
    int* act_p0 = act_e + p.max_active;
    int* act_m = act_p0 + p.max_active;
    int* act_slot = act_m + p.max_active;
    int* wprefix = act_slot + p.max_active;                              // [max_active + 1]
    int* scratch = wprefix + p.max_active + 1;                           // [2E + 1]
    __shared__ int n_act_s, n_work_s, abort_s;
    volatile int* abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E;
    const int rows = UP ? a.I : a.H;
    const int tiles_per_expert = rows / TR;
    const int KBb = UP ? L.KBu : L.KBd;          // K extent of one slot block
    const int cpb = KBb / 128;                   // chunks per block
    const int nfb = UP ? L.nfu : L.nfd;          // blocks per 16 rows
    const size_t BB = UP ? L.UB : L.DB;          // bytes per block
    const int rbb = KBb / 2, sbb = KBb / 32;     // code / scale bytes per block row
    const uint32_t tile_bytes = static_cast<uint32_t>(static_cast<size_t>(RB) * nfb * BB);

    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCW);
        }
        abort_s = 0;
    }
    fill_lut(lut);
    if (UP) pdl_wait();
    {   // active experts with their positions, counts, slots; prefix of work items
        int* offs_s = scratch;
        int* slot_s = scratch + E + 1;
        for (int e = tid; e <= E; e += blockDim.x) {
            offs_s[e] = __ldcg(a.offsets + e);
            if (e < E) slot_s[e] = __ldcg(a.slot_table + static_cast<size_t>(a.layer) * E + e);
        }
        __syncthreads();
        if (warp == 0) {
            int n = 0, work = 0;
            for (int base = 0; base < E; base += 32) {
                const int e = base + lane;
                const int o0 = (e < E) ? offs_s[e] : 0, o1 = (e < E) ? offs_s[e + 1] : 0;
                const bool on = (e < E) && (o1 > o0);
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, on);
                const int pos = n + __popc(ball & lanemask_lt());
                const int mine = on ? tiles_per_expert * ((o1 - o0 + 7) >> 3) : 0;
                int incl = mine;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += v;
                }
                if (on) {
                    act_e[pos] = e;
                    act_p0[pos] = o0;
                    act_m[pos] = o1 - o0;
                    act_slot[pos] = slot_s[e];
                    wprefix[pos] = work + incl - mine;
                }
                n += __popc(ball);
                work += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
            if (lane == 0) {
                n_act_s = n;
                n_work_s = work;
                wprefix[n] = work;
            }
        }
        if (tid == 0) fence_barrier_init();
        __syncthreads();
    }
    if (UP) pdl_trigger();
    const int n_act = n_act_s, n_work = n_work_s;
    const int G = gridDim.x;
    const int my_items = (static_cast<int>(blockIdx.x) < n_work) ? (n_work - 1 - blockIdx.x) / G + 1 : 0;
    // work item -> (active expert, tile, token group); groups of a tile are adjacent
    auto item_of = [&](int i, int& ai, int& tile, int& grp) {
        const int w = blockIdx.x + i * G;
        int lo = 0, hi = n_act - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (wprefix[mid] <= w) lo = mid; else hi = mid - 1;
        }
        const int v = w - wprefix[lo];
        const int groups = (act_m[lo] + 7) >> 3;
        ai = lo;
        tile = v / groups;
        grp = v - tile * groups;
    };

    if (warp == NCW) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            for (int i = 0; i < my_items; ++i) {
                const int st = i % p.stages;
                if (i >= p.stages && !mbar_wait(&empty[st], ((i / p.stages) - 1) & 1, abort_flag)) {
                    latch_error(a.err, ERR_ETIMEOUT, i, UP ? KID_UP : KID_DOWN);
                    break;
                }
                int ai, tile, grp;
                item_of(i, ai, tile, grp);
                const int slot = act_slot[ai];
                if (slot < 0) { mbar_arrive(&full[st]); continue; }
                const size_t src = (UP ? 0 : L.up_bytes) + static_cast<size_t>(tile) * RB * nfb * BB;
                mbar_arrive_expect_tx(&full[st], tile_bytes);
                bulk_g2s(smem + p.off_stage + static_cast<size_t>(st) * p.stage_bytes,
                         a.arena + static_cast<size_t>(slot) * a.slot_bytes + src, tile_bytes, &full[st], pol);
            }
            if (*abort_flag) {   // let copies still in flight land before the CTA may exit
                volatile int fresh = 0;
                for (int st = 0; st < p.stages && st < my_items; ++st) {
                    const int il = st + ((my_items - 1 - st) / p.stages) * p.stages;
                    fresh = 0;
                    mbar_wait(&full[st], (il / p.stages) & 1, &fresh);
                }
            }
        }
        return;   // reads nothing that `up` writes
    }

    // -------------------------------------------------------------------- consumers
    if (!UP) { pdl_wait(); pdl_trigger(); }     // h complete from here on (w2 already streams)
    const int g = lane >> 2, c = lane & 3;
    const int rbw = warp / KS, ks = warp - rbw * KS;
    int phase = 0;
    for (int i = 0; i < my_items; ++i) {
        const int st = i % p.stages;
        int ai, tile, grp;
        item_of(i, ai, tile, grp);
        const int p0 = act_p0[ai], m = act_m[ai], slot = act_slot[ai];
        const int g0 = grp * 8, ng = min(8, m - g0);
        const int row0 = tile * TR;
        // B fragments of this warp's chunks, before waiting for the weights
        const uint16_t* brow = UP ? a.x + static_cast<size_t>(__ldg(a.perm + p0 + g0 + min(g, ng - 1)) / a.k) * a.H
                                  : a.hbuf + static_cast<size_t>(p0 + g0 + min(g, ng - 1)) * a.I;
        uint4 X[CPW][4];
#pragma unroll
        for (int j = 0; j < CPW; ++j) {
            const int ch = ks * CPW + j;
#pragma unroll
            for (int q = 0; q < 4; ++q) X[j][q] = *reinterpret_cast<const uint4*>(brow + ch * 128 + 32 * c + 8 * q);
        }
        if (!mbar_wait(&full[st], (i / p.stages) & 1, abort_flag) && lane == 0)
            latch_error(a.err, ERR_ETIMEOUT, i, UP ? KID_UP : KID_DOWN);
        const uint8_t* stg = smem + p.off_stage + static_cast<size_t>(st) * p.stage_bytes;
        // two accumulators per matrix (even / odd MMA of each code word) halve
        // the chain of dependent mma.sync; summed once per item
        float d1[4] = {0.f, 0.f, 0.f, 0.f}, d3[4] = {0.f, 0.f, 0.f, 0.f};
        float e1[4] = {0.f, 0.f, 0.f, 0.f}, e3[4] = {0.f, 0.f, 0.f, 0.f};
        if (slot >= 0) {
#pragma unroll
            for (int j = 0; j < CPW; ++j) {
                const int ch = ks * CPW + j;
                const int f = ch / cpb, jj = ch - f * cpb;
                const uint8_t* blk = stg + static_cast<size_t>(rbw * nfb + f) * BB;
                const int qs = swizzle_chunk(jj * 4 + c, g, rbb) * 16;
                const uint8_t* ra = blk + g * rbb + qs;
                const uint8_t* sa = blk + MATS * 16 * rbb + g * sbb + jj * 4 + c;
                const uint4 Aa = *reinterpret_cast<const uint4*>(ra);
                const uint4 Ab = *reinterpret_cast<const uint4*>(ra + 8 * rbb);
                const Fp4Lut La = lut[sa[0]];
                const Fp4Lut Lb = lut[sa[8 * sbb]];
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    uint32_t oa[4], ob[4];
                    fp4_decode8(word(Aa, w), La, oa);
                    fp4_decode8(word(Ab, w), Lb, ob);
                    mma_bf16_16816(d1, oa[0], ob[0], oa[1], ob[1], word(X[j][w], 0), word(X[j][w], 1));
                    mma_bf16_16816(e1, oa[2], ob[2], oa[3], ob[3], word(X[j][w], 2), word(X[j][w], 3));
                }
                if (UP) {
                    const uint4 Ca = *reinterpret_cast<const uint4*>(ra + 16 * rbb);
                    const uint4 Cb = *reinterpret_cast<const uint4*>(ra + 24 * rbb);
                    const Fp4Lut Lc = lut[sa[16 * sbb]];
                    const Fp4Lut Ld = lut[sa[24 * sbb]];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        uint32_t pa[4], pb[4];
                        fp4_decode8(word(Ca, w), Lc, pa);
                        fp4_decode8(word(Cb, w), Ld, pb);
                        mma_bf16_16816(d3, pa[0], pb[0], pa[1], pb[1], word(X[j][w], 0), word(X[j][w], 1));
                        mma_bf16_16816(e3, pa[2], pb[2], pa[3], pb[3], word(X[j][w], 2), word(X[j][w], 3));
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                d1[q] += e1[q];
                d3[q] += e3[q];
            }
        } else if (tid == 0) {
            latch_error(a.err, ERR_ESLOT, act_e[ai], UP ? KID_UP : KID_DOWN);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);   // this warp is done reading the stage
        const int buf = phase++ & 1;
        float* rw = red + (buf * NCW + warp) * PART;
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
        named_barrier(1, NCW * 32);
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
                    const float hv = (slot >= 0) ? s1 / (1.0f + expf(-s1)) * s3 : 0.0f;
                    a.hbuf[static_cast<size_t>(p0 + g0 + tk) * a.I + row0 + r * 16 + row] = f32_to_bf16_rne(hv);
                } else {
                    const int ent = __ldg(a.perm + p0 + g0 + tk);
                    a.obuf[static_cast<size_t>(ent) * a.H + row0 + r * 16 + row] = (slot >= 0) ? s1 : 0.0f;
                }
            }
        }
    }
}

// Host-side plan; stages = 0 when the shape does not fit.
inline TilePlan make_tile_plan(bool up, const SlotLayout& L, int rbk, int ncw, int n_experts, int max_active,
                               int smem_limit) {
    TilePlan p{};
    const size_t tile = static_cast<size_t>(rbk) * (up ? L.nfu * L.UB : L.nfd * L.DB);
    p.stage_bytes = static_cast<int>((tile + 127) / 128 * 128);
    p.max_active = max_active;
    p.off_lut = 256;                                   // barriers before (16 stages at most)
    p.off_red = p.off_lut + 256 * 16;
    p.off_act = p.off_red + 2 * ncw * (up ? 2 : 1) * 128 * 4;
    p.off_stage = (p.off_act + 4 * (5 * max_active + 1 + 2 * n_experts + 1) + 127) / 128 * 128;
    int stages = (smem_limit - p.off_stage) / p.stage_bytes;
    if (stages > 16) stages = 16;
    p.stages = stages >= 2 ? stages : 0;
    p.smem_bytes = p.off_stage + p.stages * p.stage_bytes;
    return p;
}

}  // namespace moe
