// tc_prefill.cuh -- grouped expert GEMM on the 5th-generation tensor cores
// (tcgen05 + TMEM) for batches where experts see many tokens (prefill).
//
// Per active expert e with M_e tokens (10100.com article 151357339, section
// "moe专家的容量瓶颈"; SwiGLU reading of the unnamed activation):
//   up    D1 = W1 X^T, D3 = W3 X^T  (128 weight rows x N tokens, K = H)
//         h  = bf16(silu(D1) * D3)
//   down  D  = W2 H^T               (128 weight rows x N tokens, K = I)  -> o
// Weights are the M side (M = 128 rows per tile) and tokens the N side
// (N <= 128, rounded up to 16), so a work item is (expert, 128-row tile,
// chunk of <= 128 of the expert's tokens).
//
// One persistent CTA per SM, warp roles:
//   warps 0-7  dequantisers: thread r (+128) decodes row r of the tile for
//              half of a 64-wide K step straight from the slot (exact E2M1 x
//              2^(s-127) -> bf16, fp4_decode.cuh) into the A stage, stored in
//              the 128-byte-swizzled K-major layout the MMA reads; warps 0-3
//              then run the epilogue from TMEM (lane r = weight row r).
//   warp 8     TMA producer: the step's 16-row boxes of gathered token rows
//              (x grouped by expert, or h) into the B stage, 128-byte swizzle.
//   warp 9     MMA issuer: tcgen05.mma.cta_group::1.kind::f16 (bf16 x bf16 ->
//              fp32 in TMEM), four K=16 instructions per matrix per step;
//              tcgen05.commit frees the stage and, after the last step,
//              hands the accumulators to the epilogue.
// Stages are a ring of {A1, (A3), B} buffers with `a_full` (dequant warps),
// `b_full` (TMA bytes) and `free` (MMA commit) mbarriers; the accumulators
// have `acc_full` / `acc_empty`.  Every party walks the same sequence of
// steps, so each parity wait is unambiguous; every wait is bounded and the
// first one that gives up aborts the CTA's remaining waits.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "../../include/moe_fp4.h"
#include "common.cuh"
#include "decode_common.cuh"
#include "fp4_decode.cuh"
#include "slot_layout.cuh"
#include "tma.cuh"

namespace moe {

constexpr int kTcM = 128;          // weight rows per tile
constexpr int kTcBK = 64;          // K per step (one 128-byte swizzle atom of bf16)
constexpr int kTcNmax = 128;       // tokens per item
constexpr int kTcDequantWarps = 8;
constexpr int kTcThreads = (kTcDequantWarps + 2) * 32;

struct TcArgs {
    GemvArgs g;
    SlotLayout L;
    int T;
    int stages;
    int stage_bytes;       // A (1 or 2 x 16 KB) + B (16 KB)
    int off_stage;         // dynamic smem offset of stage 0 (1024-aligned)
    int max_active;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
    // K-major, 128-byte swizzle: start >> 4, LBO (unused) 1, SBO 1024 >> 4,
    // descriptor version 1 (bits 46-47), layout SWIZZLE_128B = 2 (bits 61-63).
    return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ uint32_t umma_idesc_bf16(int m, int n) {
    // D fp32 (bits 4-5 = 1), A bf16 (7-9 = 1), B bf16 (10-12 = 1), both
    // K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------------ gather
// x rows in grouped (expert-major) order: xg[p] = x[perm[p] / k].
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* x, const int32_t* perm, int k, int H,
                                                          int n_rows, uint16_t* xg) {
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x;
    if (row >= n_rows) return;
    const int src = __ldg(perm + row) / k;
    const uint4* s = reinterpret_cast<const uint4*>(x + static_cast<size_t>(src) * H);
    uint4* d = reinterpret_cast<uint4*>(xg + static_cast<size_t>(row) * H);
    for (int i = threadIdx.x; i < H / 8; i += blockDim.x) d[i] = s[i];
}

// ------------------------------------------------------------------ GEMM
template <bool UP>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_gemm_kernel(TcArgs t, const __grid_constant__ CUtensorMap bmap) {
    constexpr int MATS = UP ? 2 : 1;
    constexpr int A_BYTES = kTcM * 128;          // one matrix, one step: 128 rows x 64 bf16
    extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
    // the 128-byte swizzle of the operand tiles is defined on 1024-byte atoms
    // of the shared address space: align the working base explicitly
    uint8_t* smem = tc_smem_raw + ((1024u - (smem_u32(tc_smem_raw) & 1023u)) & 1023u);
    const GemvArgs& a = t.g;
    const SlotLayout& L = t.L;
    uint64_t* a_full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* b_full = a_full + t.stages;
    uint64_t* sfree = b_full + t.stages;
    uint64_t* acc_full = sfree + t.stages;
    uint64_t* acc_empty = acc_full + 1;
    Fp4Lut* lut = reinterpret_cast<Fp4Lut*>(smem + 1024);              // 4 KB, 16-byte aligned
    int* act_e = reinterpret_cast<int*>(smem + 1024 + 256 * 16);
    int* act_p0 = act_e + t.max_active;
    int* act_m = act_p0 + t.max_active;
    int* act_slot = act_m + t.max_active;
    int* wprefix = act_slot + t.max_active;
    int* scratch = wprefix + t.max_active + 1;                          // [2E + 1]
    __shared__ uint32_t tmem_base_s;
    __shared__ int n_act_s, n_work_s, abort_s;
    volatile int* abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E;
    const int K = UP ? a.H : a.I;
    const int rows = UP ? a.I : a.H;
    const int n_mt = rows / kTcM;
    const int n_steps = K / kTcBK;

    if (tid == 0) {
        for (int s = 0; s < t.stages; ++s) {
            mbar_init(&a_full[s], kTcDequantWarps);
            mbar_init(&b_full[s], 1);
            mbar_init(&sfree[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 4);
        abort_s = 0;
    }
    if (warp == 0) {   // TMEM for the accumulators: 128 (or 256) columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base_s)),
                     "r"(static_cast<uint32_t>(MATS * kTcNmax)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    for (int i = tid; i < 256; i += blockDim.x) lut[i] = make_fp4_lut(static_cast<uint32_t>(i));
    pdl_wait();
    {   // active experts and the prefix of their work items
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
                const int mine = on ? n_mt * ((o1 - o0 + kTcNmax - 1) / kTcNmax) : 0;
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
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    pdl_trigger();
    const uint32_t tmem = tmem_base_s;
    const int n_act = n_act_s, n_work = n_work_s, G = gridDim.x;
    const int my_items = (static_cast<int>(blockIdx.x) < n_work) ? (n_work - 1 - blockIdx.x) / G + 1 : 0;
    auto item_of = [&](int i, int& ai, int& mt, int& n0) {
        const int w = blockIdx.x + i * G;
        int lo = 0, hi = n_act - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (wprefix[mid] <= w) lo = mid; else hi = mid - 1;
        }
        const int v = w - wprefix[lo];
        const int chunks = (act_m[lo] + kTcNmax - 1) / kTcNmax;
        ai = lo;
        mt = v / chunks;
        n0 = (v - mt * chunks) * kTcNmax;
    };
    auto stage_a = [&](int st, int mat) { return smem + t.off_stage + static_cast<size_t>(st) * t.stage_bytes + mat * A_BYTES; };
    auto stage_b = [&](int st) { return smem + t.off_stage + static_cast<size_t>(st) * t.stage_bytes + MATS * A_BYTES; };

    if (warp < kTcDequantWarps) {
        // ------------------------------------------------------------ dequantisers
        const int r = tid & 127, hf = tid >> 7;     // row of the tile, half of the K step
        int gstep = 0;                              // steps walked so far (all items)
        int items_done = 0;
        for (int i = 0; i < my_items; ++i) {
            int ai, mt, n0;
            item_of(i, ai, mt, n0);
            const int slot = act_slot[ai];
            const int grow = mt * kTcM + r;          // weight row
            const int rt = grow >> 4, rr = grow & 15;
            const uint8_t* sbase = a.arena + static_cast<size_t>(slot < 0 ? 0 : slot) * a.slot_bytes;
            if (slot < 0 && tid == 0) latch_error(a.err, ERR_ESLOT, act_e[ai], UP ? KID_TC_UP : KID_TC_DOWN);
            for (int s = 0; s < n_steps; ++s, ++gstep) {
                const int st = gstep % t.stages;
                if (gstep >= t.stages && !mbar_wait(&sfree[st], ((gstep / t.stages) - 1) & 1, abort_flag) && lane == 0)
                    latch_error(a.err, ERR_ETIMEOUT, gstep, UP ? KID_TC_UP : KID_TC_DOWN);
                const int k0 = s * kTcBK + hf * 32;  // first K of this thread's 32
#pragma unroll
                for (int mat = 0; mat < MATS; ++mat) {
                    uint32_t o[16];
                    if (slot >= 0) {
                        const uint8_t* cp;
                        const uint8_t* sp;
                        if (UP) {
                            const int f = k0 / L.KBu, q = (k0 - f * L.KBu) / 32;
                            const uint8_t* blk = sbase + (static_cast<size_t>(rt) * L.nfu + f) * L.UB;
                            cp = blk + mat * 16 * (L.KBu / 2) + rr * (L.KBu / 2) + swizzle_chunk(q, rr, L.KBu / 2) * 16;
                            sp = blk + 32 * (L.KBu / 2) + mat * 16 * (L.KBu / 32) + rr * (L.KBu / 32) + q;
                        } else {
                            const int f = k0 / L.KBd, q = (k0 - f * L.KBd) / 32;
                            const uint8_t* blk = sbase + L.up_bytes + (static_cast<size_t>(rt) * L.nfd + f) * L.DB;
                            cp = blk + rr * (L.KBd / 2) + swizzle_chunk(q, rr, L.KBd / 2) * 16;
                            sp = blk + 16 * (L.KBd / 2) + rr * (L.KBd / 32) + q;
                        }
                        const uint4 v = ldg_stream(cp);
                        const Fp4Lut lt = lut[__ldg(sp)];
                        fp4_decode8(v.x, lt, o);
                        fp4_decode8(v.y, lt, o + 4);
                        fp4_decode8(v.z, lt, o + 8);
                        fp4_decode8(v.w, lt, o + 12);
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) o[q] = 0;
                    }
                    // row r, K chunks 4hf..4hf+3 of the 128-byte row, swizzled by r & 7
                    uint8_t* arow = stage_a(st, mat) + r * 128;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int j = (4 * hf + c) ^ (r & 7);
                        *reinterpret_cast<uint4*>(arow + j * 16) = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
                    }
                }
                fence_async_smem();                    // generic stores -> tensor core reads
                __syncwarp();
                if (lane == 0) mbar_arrive(&a_full[st]);
            }
            // epilogue (warps 0-3: TMEM lanes 0-127)
            if (warp < 4) {
                const int p0 = act_p0[ai], m = act_m[ai];
                const int nvalid = min(kTcNmax, m - n0);
                if (!mbar_wait(acc_full, items_done & 1, abort_flag) && lane == 0)
                    latch_error(a.err, ERR_ETIMEOUT, i, UP ? KID_TC_UP : KID_TC_DOWN);
                tc_fence_after();
                const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
                for (int c16 = 0; c16 * 16 < nvalid; ++c16) {
                    uint32_t v1[16], v3[16];
                    tmem_ld16(tmem + lane_base + c16 * 16, v1);
                    if (UP) tmem_ld16(tmem + lane_base + kTcNmax + c16 * 16, v3);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int j = c16 * 16 + q;
                        if (j < nvalid) {
                            const float s1 = __uint_as_float(v1[q]);
                            if (UP) {
                                const float s3 = __uint_as_float(v3[q]);
                                const float hv = (slot >= 0) ? s1 / (1.0f + expf(-s1)) * s3 : 0.0f;
                                a.hbuf[static_cast<size_t>(p0 + n0 + j) * a.I + mt * kTcM + r] = f32_to_bf16_rne(hv);
                            } else {
                                const int ent = __ldg(a.perm + p0 + n0 + j);
                                a.obuf[static_cast<size_t>(ent) * a.H + mt * kTcM + r] = (slot >= 0) ? s1 : 0.0f;
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty);
            }
            ++items_done;
        }
    } else if (warp == kTcDequantWarps) {
        // ------------------------------------------------------------ TMA producer (B)
        if (lane == 0) {
            int gstep = 0;
            for (int i = 0; i < my_items; ++i) {
                int ai, mt, n0;
                item_of(i, ai, mt, n0);
                const int nvalid = min(kTcNmax, act_m[ai] - n0);
                const int nb = (nvalid + 15) / 16;
                const int row0 = act_p0[ai] + n0;
                for (int s = 0; s < n_steps; ++s, ++gstep) {
                    const int st = gstep % t.stages;
                    if (gstep >= t.stages && !mbar_wait(&sfree[st], ((gstep / t.stages) - 1) & 1, abort_flag))
                        latch_error(a.err, ERR_ETIMEOUT, gstep, UP ? KID_TC_UP : KID_TC_DOWN);
                    mbar_arrive_expect_tx(&b_full[st], static_cast<uint32_t>(nb * 16 * 128));
                    for (int b = 0; b < nb; ++b)
                        tma_load_2d(stage_b(st) + b * 2048, &bmap, s * kTcBK, row0 + 16 * b, &b_full[st]);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int gstep = 0;
            for (int i = 0; i < my_items; ++i) {
                int ai, mt, n0;
                item_of(i, ai, mt, n0);
                const int nvalid = min(kTcNmax, act_m[ai] - n0);
                const int n = (nvalid + 15) / 16 * 16;
                const uint32_t idesc = umma_idesc_bf16(kTcM, n);
                if (i > 0 && !mbar_wait(acc_empty, (i - 1) & 1, abort_flag))
                    latch_error(a.err, ERR_ETIMEOUT, i, UP ? KID_TC_UP : KID_TC_DOWN);
                tc_fence_after();
                for (int s = 0; s < n_steps; ++s, ++gstep) {
                    const int st = gstep % t.stages;
                    const uint32_t ph = (gstep / t.stages) & 1;
                    if (!mbar_wait(&a_full[st], ph, abort_flag) || !mbar_wait(&b_full[st], ph, abort_flag))
                        latch_error(a.err, ERR_ETIMEOUT, gstep, UP ? KID_TC_UP : KID_TC_DOWN);
                    tc_fence_after();
                    const uint64_t bdesc = umma_desc_sw128(smem_u32(stage_b(st)));
#pragma unroll
                    for (int mat = 0; mat < MATS; ++mat) {
                        const uint64_t adesc = umma_desc_sw128(smem_u32(stage_a(st, mat)));
#pragma unroll
                        for (int kk = 0; kk < kTcBK / 16; ++kk)   // +32 bytes per K=16 inside the atom
                            umma_bf16(tmem + mat * kTcNmax, adesc + 2 * kk, bdesc + 2 * kk, idesc,
                                      (s > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&sfree[st]);                  // stage reusable once these MMAs are done
                }
                umma_commit(acc_full);                        // accumulators complete
            }
            if (my_items > 0) {   // the last commits must land before TMEM is released
                volatile int fresh = 0;
                mbar_wait(acc_full, (my_items - 1) & 1, &fresh);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(static_cast<uint32_t>(MATS * kTcNmax)));
}

// ------------------------------------------------------------------ host side
struct TcPlan {
    int ready;
    uint16_t* xg;          // gathered x rows [max_tokens * k, H]
    CUtensorMap map_x;     // bf16 [rows, H], box {64, 16}, 128-byte swizzle
    CUtensorMap map_h;     // bf16 [rows, I], box {64, 16}, 128-byte swizzle
    int rows;
    int smem_limit;
    int sm_count;
};

inline bool tc_encode_map(CUtensorMap* map, void* base, int rows, int cols) {
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    if (!encode) {
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", reinterpret_cast<void**>(&encode), cudaEnableDefault,
                                    &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
    }
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcBK), 16};
    const cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline cudaError_t tc_plan_create(TcPlan* p, const moe_fp4_config& cfg, uint16_t* hbuf, int sm_count,
                                  int smem_limit) {
    *p = TcPlan{};
    p->rows = cfg.max_tokens * cfg.top_k;
    p->sm_count = sm_count;
    p->smem_limit = smem_limit;
    cudaError_t e = cudaMalloc(&p->xg, sizeof(uint16_t) * static_cast<size_t>(p->rows) * cfg.hidden);
    if (e != cudaSuccess) return e;
    if (!tc_encode_map(&p->map_x, p->xg, p->rows, cfg.hidden) || !tc_encode_map(&p->map_h, hbuf, p->rows, cfg.inter))
        return cudaErrorInvalidValue;
    auto set = [&](const void* f) {
        return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_limit);
    };
    if ((e = set(reinterpret_cast<const void*>(tc_gemm_kernel<true>))) != cudaSuccess) return e;
    if ((e = set(reinterpret_cast<const void*>(tc_gemm_kernel<false>))) != cudaSuccess) return e;
    p->ready = 1;
    return cudaSuccess;
}

inline void tc_plan_destroy(TcPlan* p) {
    if (p->xg) cudaFree(p->xg);
    p->xg = nullptr;
    p->ready = 0;
}

// The tcgen05 path pays off once experts see several tokens on average.
inline bool tc_prefers(int T, const moe_fp4_config& cfg) {
    return static_cast<long long>(T) * cfg.top_k >= 4LL * cfg.n_experts;
}

inline TcArgs tc_args(const TcPlan& p, const GemvArgs& g, const SlotLayout& L, int T, bool up) {
    TcArgs t{};
    t.g = g;
    t.L = L;
    t.T = T;
    const int ent = T * g.k;
    t.max_active = ent < g.E ? ent : g.E;
    const int mats = up ? 2 : 1;
    t.stage_bytes = mats * kTcM * 128 + kTcNmax * 128;
    const int head = 1024 + 256 * 16 + 4 * (5 * t.max_active + 1 + 2 * g.E + 1);
    t.off_stage = (head + 1023) / 1024 * 1024;
    int stages = (p.smem_limit - 1024 - t.off_stage) / t.stage_bytes;
    if (stages > 8) stages = 8;
    t.stages = stages >= 2 ? stages : 0;
    return t;
}

inline size_t tc_smem_bytes(const TcArgs& t) {
    return static_cast<size_t>(t.off_stage) + t.stages * t.stage_bytes + 1024;   // + alignment slack
}

}  // namespace moe
