// tc_prefill.cuh -- grouped expert GEMM on the 5th-generation tensor cores
// (tcgen05 + TMEM) for batches where experts see many tokens (prefill).
//
// Per active expert e with M_e tokens (10100.com article 151357339, section
// "moe专家的容量瓶颈"; SwiGLU reading of the unnamed activation):
//   up    a1 = W1 X^T, a3 = W3 X^T, h = bf16(silu(a1) * a3)   (K = H)
//   down  o  = W2 H^T                                         (K = I)
// Weights are the M side of tcgen05.mma (M = 128 TMEM lanes) and tokens the
// N side (N <= NMAX, rounded up to 16; NMAX = 128, or 64 with a deeper ring
// for batches of at most 64 tokens).  A work item is (expert, row group,
// chunk of <= NMAX of the expert's tokens):
//   up    64 output rows: TMEM lane 32g + l holds w1 row 16g + l (l < 16) or
//         w3 row 16g + l - 16 (l >= 16) of the item's 64 rows (half of a
//         128-row unit of each) -- so silu(a1) * a3 pairs lanes l and l + 16
//         of one warp (a shuffle, no shared memory);
//   down  128 output rows, lane r = row r.
// Both GEMMs therefore run the same pipeline on a 128 x 128 bf16 A tile per
// stage (128 K, two 128-byte swizzle atoms).  One persistent CTA per SM, warp
// roles:
//   warps 0-15   dequantisers: warp w works in TMEM lane group w % 4 and
//                takes 32-K block c = w / 4 of every 128-K stage: each
//                thread reads its row's 16-byte chunk of block c (32 codes,
//                slot_layout.cuh) and the block's scale byte, converts the
//                codes to f16 (exact E2M1), multiplies them by 2^(s - s_ref) with
//                s_ref the row's largest scale (exact while the row's scales
//                span at most 23: 0.5 * 2^-23 is f16's 2^-24), and writes them
//                to the stage's A columns in TMEM with tcgen05.st (lane =
//                row, two f16 per column, K in natural order).
//   warps 16-19  epilogue: tcgen05.ld of the finished accumulator (double
//                buffered), times 2^(s_ref - 127) of the row and the
//                column's 2^-sigma (B is prescaled f16), SwiGLU -> h (bf16) or
//                o (fp32, scattered back to token-expert order), overlapping
//                the next item's MMAs.
//   warp 20      B producer: TMA tensor loads of the stage's 16-row boxes of
//                gathered token rows (x grouped by expert, or h, both as f16
//                with an exact power-of-two prescale per row), 128-byte
//                swizzle, into shared memory.
//   warp 21      code producer: cp.async.bulk of the item's rows of two
//                128-K units (one when K / 128 is odd) per ring entry (up:
//                rows 64h.. of the w1 and the w3 unit and both scale atoms;
//                down: the whole w2 unit); the dequantisers free an entry
//                once, after both of its stages.
//   warp 22      MMA issuer: tcgen05.mma.cta_group::1.kind::f16 (f16 x f16)
//                with A from TMEM and B from shared memory (fp32 accumulate
//                in TMEM), eight
//                K=16 instructions per stage; tcgen05.commit frees the stage
//                and, after the last stage, hands the accumulator over.
// A stage is "full" when all 16 dequant warps have arrived and the B bytes
// have landed (one mbarrier: 16 arrivals + the producer's expect-tx).
// Every party walks the same sequence of stages and items, so each parity wait
// is unambiguous; every wait is bounded and the first one that gives up
// aborts the CTA's remaining waits (MOE_FP4_ETIMEOUT), after producers have
// let their copies in flight land.  The pipeline's waits poll the barrier
// (mbar_poll: a non-blocking probe every ~32 ns) instead of suspending in
// try_wait: measured on B200, polling made the w1/w3 GEMM 7 % faster at 2,048
// tokens and 10 % faster at 64, the stage hand-offs being the critical path.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

#include "../../include/moe_fp4.h"
#include "common.cuh"
#include "decode_common.cuh"
#include "fp4_cvt.cuh"
#include "slot_layout.cuh"
#include "tma.cuh"

namespace moe {

constexpr int kTcM = 128;          // TMEM lanes = A rows per MMA
constexpr int kTcBK = 64;          // K of one 128-byte swizzle atom of bf16 (four K=16 MMAs)
constexpr int kTcSK = 128;         // K per pipeline stage (two atoms, eight MMAs)
constexpr int kTcDequantWarps = 16;
constexpr int kTcEpiWarps = 4;
constexpr int kTcThreads = (kTcDequantWarps + kTcEpiWarps + 3) * 32;   // + B producer, code producer, MMA
constexpr int kTcMaxEntries = 8;   // code ring entries at most
// Tile shapes.  NMAX = tokens per item (columns of each of the two fp32
// accumulators); the rest of the 512 TMEM columns holds the A stages (64
// columns each), and the B ring in shared memory has as many stages
// (2 atoms x NMAX rows x 128 bytes each):
//   NMAX 128: 4 stages -- an expert's tokens are read in chunks of 128;
//   NMAX  64: 6 stages -- chosen when no expert can hold more than 64 tokens
//             (batch <= 64: a token names an expert at most once), where the
//             deeper ring is faster (decode batch 64: 1.13 ms against 1.22 ms
//             on B200) and no weight is read twice.  At 2048 tokens the extra
//             chunks of hot experts cost as much as the stages gain.
constexpr int kTcNmaxWide = 128;
constexpr int kTcNmaxNarrow = 64;
__host__ __device__ constexpr int tc_stages(int nmax) { return (512 - 2 * nmax) / 64; }
static_assert(tc_stages(kTcNmaxWide) == 4 && tc_stages(kTcNmaxNarrow) == 6, "TMEM: 2 NMAX + 64 S = 512 columns");

struct TcArgs {
    ExpertArgs g;
    const uint8_t* rowref;  // [n_slots][2I + H]: largest scale byte of each w1, w3, w2 row
    const float* colscale;  // [T*k] 2^-sigma of each B row (gathered x, or h)
    uint16_t* hb;           // [T*k, I] bf16 h (up output, grouped order)
    SlotLayout L;
    int T;
    int nmax;              // tile shape: kTcNmaxWide or kTcNmaxNarrow (tokens per item)
    int off_b;             // dynamic smem offset of the B ring (1024-aligned), stages x 2 atoms x nmax rows x 128 bytes
    int off_code;          // offset of the code ring: centries x entry_bytes
    int entry_bytes;       // one code ring entry: spe units' worth of the item's rows
    int spe;               // 128-K units (= stages) per code entry: 2 when K / 128 is even, else 1
    int centries;          // 0 when the shape does not fit
    int max_active;
    unsigned long long timeout_ns;   // limit of each bounded wait
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
    // K-major, 128-byte swizzle: start >> 4, LBO (unused) 1, SBO 1024 >> 4,
    // descriptor version 1 (bits 46-47), layout SWIZZLE_128B = 2 (bits 61-63).
    return static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ uint32_t umma_idesc_f16(int m, int n) {
    // D fp32 (bits 4-5 = 1), A f16 (7-9 = 0), B f16 (10-12 = 0), both
    // K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
    return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// One tcgen05.mma (kind::f16, f16 x f16 -> fp32, M = 128) with A read from
// tensor memory (lane = row, two f16 per column) and B from shared memory.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t r[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane, then wait for the stores.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t r[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// f16x2 product (exact here: a power of two times an E2M1 value).
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// ------------------------------------------------------------------ gather
// Token rows in grouped (expert-major) order as prescaled f16 (fp4_cvt.cuh):
// xg[p] = x[perm[p] / k] * 2^sigma, colscale[p] = 2^-sigma, sigma from the
// row's largest |x|.  One CTA per grouped row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* x, const int32_t* perm, int k, int H,
                                                          int n_rows, uint16_t* xg, float* colscale) {
    __shared__ uint32_t red[8];
    pdl_wait();
    pdl_trigger();
    const int row = blockIdx.x;
    if (row >= n_rows) return;
    const int ent = __ldg(perm + row);
    if (ent < 0 || ent >= n_rows) {   // not an entry of this batch (an invalid routing): a zero row
        uint32_t* d = reinterpret_cast<uint32_t*>(xg + static_cast<size_t>(row) * H);
        for (int i = threadIdx.x; i < H / 2; i += blockDim.x) d[i] = 0u;
        if (threadIdx.x == 0) colscale[row] = 0.0f;
        return;
    }
    const int src = ent / k;
    const uint32_t* s = reinterpret_cast<const uint32_t*>(x + static_cast<size_t>(src) * H);
    uint32_t mx = 0;
    for (int i = threadIdx.x; i < H / 2; i += blockDim.x) mx = max(mx, bf16x2_absmax(s[i]));
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    uint32_t tot = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) tot = max(tot, red[w]);
    const int sg = prescale_sigma(tot);
    const float mult = pow2i(sg);
    uint32_t* d = reinterpret_cast<uint32_t*>(xg + static_cast<size_t>(row) * H);
    for (int i = threadIdx.x; i < H / 2; i += blockDim.x) d[i] = bf16x2_scaled_to_f16x2(s[i], mult);
    if (threadIdx.x == 0) colscale[row] = pow2i(-sg);
}

// h rows (bf16, grouped order) -> prescaled f16 for the down GEMM: one warp
// per row, sigma from the row's largest |h|.
__global__ void __launch_bounds__(256) h_convert_kernel(const uint16_t* hb, int I, int n_rows, uint16_t* hh,
                                                        float* colscale) {
    pdl_wait();
    pdl_trigger();
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (row >= n_rows) return;
    const uint32_t* s = reinterpret_cast<const uint32_t*>(hb + static_cast<size_t>(row) * I);
    uint32_t mx = 0;
    for (int i = lane; i < I / 2; i += 32) mx = max(mx, bf16x2_absmax(__ldcg(s + i)));
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    const int sg = prescale_sigma(mx);
    const float mult = pow2i(sg);
    uint32_t* d = reinterpret_cast<uint32_t*>(hh + static_cast<size_t>(row) * I);
    for (int i = lane; i < I / 2; i += 32) d[i] = bf16x2_scaled_to_f16x2(__ldcg(s + i), mult);
    if (lane == 0) colscale[row] = pow2i(-sg);
}

// ------------------------------------------------------------------ GEMM
template <bool UP, int NMAX>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_gemm_kernel(TcArgs t, const __grid_constant__ CUtensorMap bmap) {
    constexpr int ROWT = UP ? 4 : 8;             // 16-row groups per item
    constexpr int OUT_ROWS = UP ? 64 : 128;      // output rows per item
    constexpr int ACOLS = kTcSK / 2;             // TMEM columns of one stage's A (bf16 pairs)
    constexpr int BATOM = NMAX * 128;            // bytes of one B swizzle atom (N rows x 64 K)
    constexpr int S = tc_stages(NMAX);
    constexpr int ACC_COLS = 2 * NMAX;           // two accumulators of NMAX fp32 columns, then the A stages
    extern __shared__ __align__(1024) uint8_t tc_smem_raw[];
    // the 128-byte swizzle of the B tiles is defined on 1024-byte atoms of the
    // shared address space: align the working base explicitly
    uint8_t* smem = tc_smem_raw + ((1024u - (smem_u32(tc_smem_raw) & 1023u)) & 1023u);
    const ExpertArgs& a = t.g;
    const SlotLayout& L = t.L;
    const int CE = t.centries;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);   // A decoded + B landed
    uint64_t* sfree = full + S;
    uint64_t* cfull = sfree + S;
    uint64_t* cfree = cfull + CE;
    uint64_t* acc_full = cfree + CE;             // [2]
    uint64_t* acc_empty = acc_full + 2;          // [2]
    uint32_t* mtab = reinterpret_cast<uint32_t*>(smem + 1024);          // f16x2 2^-i, i = 0..255 (4 KB reserved)
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
    const int n_mt = (UP ? a.I : a.H) / OUT_ROWS;
    const int n_stg = K / kTcSK;                 // stages per item: one 128-K unit each
    const int spe = t.spe;                       // stages per code entry
    const int nfb = n_stg / spe;                 // code entries per item
    const int ustride = t.entry_bytes / spe;     // bytes of one unit inside an entry

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], kTcDequantWarps + 1);   // dequant warps + the B producer's expect_tx
            mbar_init(&sfree[s], 1);
        }
        for (int c = 0; c < CE; ++c) {
            mbar_init(&cfull[c], 1);
            mbar_init(&cfree[c], kTcDequantWarps);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(&acc_full[q], 1);
            mbar_init(&acc_empty[q], kTcEpiWarps);
        }
        abort_s = 0;
    }
    if (warp == 0) {   // all 512 TMEM columns: two accumulators, then the A stages
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base_s)),
                     "r"(512u));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    for (int i = tid; i < 256; i += blockDim.x) {   // 2^-i as f16 (subnormal from 2^-15 to 2^-24, then 0)
        const uint32_t hb16 = i <= 14 ? static_cast<uint32_t>(15 - i) << 10 : (i <= 24 ? 1u << (24 - i) : 0u);
        mtab[i] = hb16 | (hb16 << 16);
    }
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
                bool on = (e < E) && (o1 > o0);
                if (on && (o0 < 0 || o1 > t.T * a.k)) {   // not a grouping of these T*k entries
                    latch_error(a.err, ERR_EINVAL, e, UP ? KID_TC_UP : KID_TC_DOWN);
                    on = false;
                }
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, on);
                const int pos = n + __popc(ball & lanemask_lt());
                const int mine = on ? n_mt * ((o1 - o0 + NMAX - 1) / NMAX) : 0;
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
    const uint32_t tmem_a = tmem + ACC_COLS;   // A stage st at + st * ACOLS
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
        const int chunks = (act_m[lo] + NMAX - 1) / NMAX;
        ai = lo;
        mt = v / chunks;
        n0 = (v - mt * chunks) * NMAX;
    };
    auto code_entry = [&](int ce) { return smem + t.off_code + static_cast<size_t>(ce) * t.entry_bytes; };
    auto stage_b = [&](int st) { return smem + t.off_b + static_cast<size_t>(st) * (2 * BATOM); };
    const int kid = UP ? KID_TC_UP : KID_TC_DOWN;
    const int lg = warp & 3;                                   // TMEM lane group of this warp
    const uint32_t lane_addr = static_cast<uint32_t>(32 * lg) << 16;

    if (warp < kTcDequantWarps) {
        // ------------------------------------------------------------ dequantisers
        // Warp w works in TMEM lane group w % 4 and takes 32-K block c = w / 4
        // of every 128-K stage: each thread converts its row's 32 codes of
        // block c (one 16-byte chunk of the unit, slot_layout.cuh), scales
        // them by 2^(s - s_ref) and stores 16 columns (K in natural order).
        const int cc = warp >> 2;                              // 32-K block of the stage
        // up: lanes 0-15 w1 rows, 16-31 w3 rows of the item's 64; down: row 32 lg + lane
        const int mat = UP ? (lane >> 4) : 0;
        const int rloc = UP ? 16 * lg + (lane & 15) : 32 * lg + lane;
        int gstg = 0, gent = 0;
        for (int i = 0; i < my_items; ++i) {
            int ai, mt, n0;
            item_of(i, ai, mt, n0);
            const int slot = act_slot[ai];
            if (slot < 0 && tid == 0) latch_error(a.err, ERR_ESLOT, act_e[ai], kid);
            // entry layout, per unit j at j * ustride:
            //   up   [w1 rows 64h.. codes 4096][w3 codes 4096][w1 scale atom][w3 scale atom]
            //   down [the unit, 8704]
            const int urow = UP ? 64 * (mt & 1) + rloc : rloc;       // row inside the 128-row unit
            const int code_off = UP ? mat * 4096 + unit_code_chunk(rloc, cc) : unit_code_chunk(rloc, cc);
            const int scale_off = UP ? 2 * 4096 + mat * kUnitScaleBytes + unit_scale_byte(urow, cc) - kUnitCodeBytes
                                     : unit_scale_byte(urow, cc);
            // the row's largest scale (load-time table)
            const int wrow = mt * OUT_ROWS + rloc;
            const int sref = slot < 0 ? 0
                                      : __ldg(t.rowref + static_cast<size_t>(slot) * (2 * a.I + a.H) +
                                              (UP ? mat * a.I : 2 * a.I) + wrow);
            for (int f = 0; f < nfb; ++f, ++gent) {
                const int ce = gent % CE;
                if (!mbar_poll(&cfull[ce], (gent / CE) & 1, abort_flag, t.timeout_ns) && lane == 0)
                    latch_error(a.err, ERR_ETIMEOUT, gent, kid);
                const uint8_t* ent = code_entry(ce);
                for (int j = 0; j < spe; ++j, ++gstg) {
                    const int st = gstg % S;
                    if (gstg >= S && !mbar_poll(&sfree[st], ((gstg / S) - 1) & 1, abort_flag, t.timeout_ns) &&
                        lane == 0)
                        latch_error(a.err, ERR_ETIMEOUT, gstg, kid);
                    tc_fence_after();
                    const uint4 w = *reinterpret_cast<const uint4*>(ent + j * ustride + code_off);
                    const int sq = ent[j * ustride + scale_off];
                    const uint32_t mult = (slot < 0) ? 0u : mtab[(sref - sq) & 255];
                    uint32_t o[16];
                    e2m1x8_to_f16x2(w.x, o);
                    e2m1x8_to_f16x2(w.y, o + 4);
                    e2m1x8_to_f16x2(w.z, o + 8);
                    e2m1x8_to_f16x2(w.w, o + 12);
#pragma unroll
                    for (int q = 0; q < 16; ++q) o[q] = hmul2_u32(o[q], mult);
                    tmem_st16(tmem_a + lane_addr + st * ACOLS + 16 * cc, o);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&full[st]);
                }
                if (lane == 0) mbar_arrive(&cfree[ce]);
            }
        }
    } else if (warp < kTcDequantWarps + kTcEpiWarps) {
        // ------------------------------------------------------------ epilogue
        for (int i = 0; i < my_items; ++i) {
            int ai, mt, n0;
            item_of(i, ai, mt, n0);
            const int p0 = act_p0[ai], m = act_m[ai], slot = act_slot[ai];
            const int nvalid = min(NMAX, m - n0);
            const int ab = i & 1;
            if (!mbar_poll(&acc_full[ab], (i >> 1) & 1, abort_flag, t.timeout_ns) && lane == 0)
                latch_error(a.err, ERR_ETIMEOUT, i, kid);
            tc_fence_after();
            // this lane's weight row and its 2^(s_ref - 127)
            const int erow = UP ? (mt * ROWT + lg) * 16 + (lane & 15) : mt * OUT_ROWS + 32 * lg + lane;
            const int emat = UP ? (lane >> 4) : 2;
            const float rowmul = slot < 0 ? 0.0f
                                          : pow2i(static_cast<int>(__ldg(t.rowref + static_cast<size_t>(slot) *
                                                                                        (2 * a.I + a.H) +
                                                                         emat * a.I + erow)) - 127);
            for (int c16 = 0; c16 * 16 < nvalid; ++c16) {
                uint32_t v[16];
                tmem_ld16(tmem + lane_addr + ab * NMAX + c16 * 16, v);
                if (UP) {
                    // lanes 0-15: a1 of rows 16 lg + lane; lanes 16-31 hold the matching a3
#pragma unroll
                    for (int qq = 0; qq < 16; ++qq) {
                        const int jt = c16 * 16 + qq;
                        const float cs = (jt < nvalid) ? __ldg(t.colscale + p0 + n0 + jt) : 0.0f;
                        const float mine = __uint_as_float(v[qq]) * rowmul * cs;
                        const float a3 = __shfl_down_sync(0xFFFFFFFFu, mine, 16);
                        if (lane < 16 && jt < nvalid) {
                            const float a1 = mine;
                            const float hv = (slot >= 0) ? a1 / (1.0f + expf(-a1)) * a3 : 0.0f;
                            t.hb[static_cast<size_t>(p0 + n0 + jt) * a.I + mt * OUT_ROWS + 16 * lg + lane] =
                                f32_to_bf16_rne(hv);
                        }
                    }
                } else {
#pragma unroll
                    for (int qq = 0; qq < 16; ++qq) {
                        const int jt = c16 * 16 + qq;
                        if (jt < nvalid) {
                            const int entn = __ldg(a.perm + p0 + n0 + jt);
                            if (entn < 0 || entn >= t.T * a.k) continue;   // not an entry of this batch
                            const float cs = __ldg(t.colscale + p0 + n0 + jt);
                            a.obuf[static_cast<size_t>(entn) * a.H + mt * OUT_ROWS + 32 * lg + lane] =
                                (slot >= 0) ? __uint_as_float(v[qq]) * rowmul * cs : 0.0f;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
    } else if (warp == kTcDequantWarps + kTcEpiWarps) {
        // ------------------------------------------------------------ B producer
        // The whole warp walks the loop (warp-uniform waits); lane 0 issues.
        // After a wait gives up no further copy is issued (a stage is never
        // the target of two copies at once); the decision is warp-uniform.
        int gstg = 0;
        bool stop = false;
        for (int i = 0; i < my_items && !stop; ++i) {
            int ai, mt, n0;
            item_of(i, ai, mt, n0);
            const int nvalid = min(NMAX, act_m[ai] - n0);
            const int nb = (nvalid + 15) / 16;
            const int row0 = act_p0[ai] + n0;
            for (int s = 0; s < n_stg; ++s, ++gstg) {
                const int st = gstg % S;
                int ok = 1;
                if (gstg >= S && lane == 0) ok = mbar_poll(&sfree[st], ((gstg / S) - 1) & 1, abort_flag, t.timeout_ns);
                if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
                    if (lane == 0) latch_error(a.err, ERR_ETIMEOUT, gstg, kid);
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(2 * nb * 16 * 128));
                    for (int at = 0; at < 2; ++at)
                        for (int b = 0; b < nb; ++b)
                            tma_load_2d(stage_b(st) + at * BATOM + b * 2048, &bmap, s * kTcSK + at * kTcBK,
                                        row0 + 16 * b, &full[st]);
                }
                __syncwarp();
            }
        }
        if (*abort_flag && lane == 0) {   // copies still in flight land before the CTA may exit
            volatile int fresh = 0;
            for (int st = 0; st < S && st < gstg; ++st) {
                const int last = st + ((gstg - 1 - st) / S) * S;
                fresh = 0;
                mbar_wait(&full[st], (last / S) & 1, &fresh);
            }
        }
    } else if (warp == kTcDequantWarps + kTcEpiWarps + 1) {
        // ------------------------------------------------------------ code producer (FP4 blocks)
        const uint64_t pol = policy_evict_first();
        int gentry = 0;
        bool stop = false;
        for (int i = 0; i < my_items && !stop; ++i) {
            int ai, mt, n0;
            item_of(i, ai, mt, n0);
            const int slot = act_slot[ai];
            const uint8_t* src = a.arena + static_cast<size_t>(slot < 0 ? 0 : slot) * a.slot_bytes +
                                 (UP ? 0 : L.up_bytes);
            for (int f = 0; f < nfb; ++f, ++gentry) {
                const int ce = gentry % CE;
                int ok = 1;
                if (gentry >= CE && lane == 0)
                    ok = mbar_poll(&cfree[ce], ((gentry / CE) - 1) & 1, abort_flag, t.timeout_ns);
                if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) {
                    if (lane == 0) latch_error(a.err, ERR_ETIMEOUT, gentry, kid);
                    stop = true;
                    break;
                }
                if (lane == 0) {
                    if (slot < 0) {
                        mbar_arrive(&cfull[ce]);
                    } else {
                        mbar_arrive_expect_tx(&cfull[ce], static_cast<uint32_t>(t.entry_bytes));
                        for (int j = 0; j < spe; ++j) {
                            uint8_t* dst = code_entry(ce) + j * ustride;
                            const int ku = f * spe + j;
                            if (UP) {   // rows 64h .. 64h+63 of the w1 and w3 units (rt, ku), and both scale atoms
                                const int rt = mt >> 1, hh = mt & 1;
                                const uint8_t* u1 = src + up_unit_offset(L, 0, rt, ku);
                                const uint8_t* u3 = src + up_unit_offset(L, 1, rt, ku);
                                bulk_g2s(dst, u1 + 4096 * hh, 4096u, &cfull[ce], pol);
                                bulk_g2s(dst + 4096, u3 + 4096 * hh, 4096u, &cfull[ce], pol);
                                bulk_g2s(dst + 8192, u1 + kUnitCodeBytes, kUnitScaleBytes, &cfull[ce], pol);
                                bulk_g2s(dst + 8192 + kUnitScaleBytes, u3 + kUnitCodeBytes, kUnitScaleBytes,
                                         &cfull[ce], pol);
                            } else {
                                bulk_g2s(dst, src + down_unit_offset(L, mt, ku) - L.up_bytes, kUnitBytes,
                                         &cfull[ce], pol);
                            }
                        }
                    }
                }
                __syncwarp();
            }
        }
        if (*abort_flag && lane == 0) {
            volatile int fresh = 0;
            for (int ce = 0; ce < CE && ce < gentry; ++ce) {
                const int last = ce + ((gentry - 1 - ce) / CE) * CE;
                fresh = 0;
                mbar_wait(&cfull[ce], (last / CE) & 1, &fresh);
            }
        }
    } else {
        // ------------------------------------------------------------ MMA issuer
        int gstg = 0;
        for (int i = 0; i < my_items; ++i) {
            int ai, mt, n0;
            item_of(i, ai, mt, n0);
            const int nvalid = min(NMAX, act_m[ai] - n0);
            const int n = (nvalid + 15) / 16 * 16;
            const uint32_t idesc = umma_idesc_f16(kTcM, n);
            const int ab = i & 1;
            if (i >= 2 && !mbar_poll(&acc_empty[ab], ((i >> 1) - 1) & 1, abort_flag, t.timeout_ns) && lane == 0)
                latch_error(a.err, ERR_ETIMEOUT, i, kid);
            tc_fence_after();
            const uint32_t dacc = tmem + ab * NMAX;
            for (int s = 0; s < n_stg; ++s, ++gstg) {
                const int st = gstg % S;
                if (!mbar_poll(&full[st], (gstg / S) & 1, abort_flag, t.timeout_ns) && lane == 0)
                    latch_error(a.err, ERR_ETIMEOUT, gstg, kid);
                tc_fence_after();
                const uint64_t bdesc = umma_desc_sw128(smem_u32(stage_b(st)));
                const uint32_t acol = tmem_a + st * ACOLS;
                if (lane == 0) {
#pragma unroll
                    for (int at = 0; at < 2; ++at)
#pragma unroll
                        for (int kk = 0; kk < kTcBK / 16; ++kk)   // K = 16: 8 TMEM columns of A, +32 bytes of B
                            umma_f16_ts(dacc, acol + at * (kTcBK / 2) + 8 * kk,
                                         bdesc + static_cast<uint64_t>((at * BATOM) >> 4) + 2 * kk, idesc,
                                         (s > 0 || at > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sfree[st]);                  // stage reusable once these MMAs are done
                }
                __syncwarp();
            }
            if (lane == 0) umma_commit(&acc_full[ab]);        // accumulator complete
            __syncwarp();
        }
        if (my_items > 0 && lane == 0) {   // the last commits must land before TMEM is released
            volatile int fresh = 0;
            mbar_wait(&acc_full[(my_items - 1) & 1], ((my_items - 1) >> 1) & 1, &fresh);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u));
}

// ------------------------------------------------------------------ host side
struct TcPlan {
    int ready;
    uint16_t* xg;          // gathered x rows, prescaled f16 [max_tokens * k, H]
    float* xcs;            // [max_tokens * k] 2^-sigma of each gathered x row
    uint16_t* hb;          // h, bf16 [max_tokens * k, I] (up output)
    uint16_t* hh;          // h, prescaled f16 [max_tokens * k, I] (down input; owned by the context)
    float* hcs;            // [max_tokens * k] 2^-sigma of each h row
    CUtensorMap map_x;     // f16 [rows, H], box {64, 16}, 128-byte swizzle
    CUtensorMap map_h;     // f16 [rows, I], box {64, 16}, 128-byte swizzle
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
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline cudaError_t tc_plan_create(TcPlan* p, const moe_fp4_config& cfg, uint16_t* hh, int sm_count,
                                  int smem_limit) {
    *p = TcPlan{};
    p->rows = cfg.max_tokens * cfg.top_k;
    p->sm_count = sm_count;
    p->smem_limit = smem_limit;
    p->hh = hh;
    const size_t rows = static_cast<size_t>(p->rows);
    cudaError_t e;
    if ((e = cudaMalloc(&p->xg, sizeof(uint16_t) * rows * cfg.hidden)) != cudaSuccess ||
        (e = cudaMalloc(&p->xcs, sizeof(float) * rows)) != cudaSuccess ||
        (e = cudaMalloc(&p->hb, sizeof(uint16_t) * rows * cfg.inter)) != cudaSuccess ||
        (e = cudaMalloc(&p->hcs, sizeof(float) * rows)) != cudaSuccess)
        return e;
    if (!tc_encode_map(&p->map_x, p->xg, p->rows, cfg.hidden) || !tc_encode_map(&p->map_h, hh, p->rows, cfg.inter))
        return cudaErrorInvalidValue;
    auto set = [&](const void* f) {
        return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_limit);
    };
    if ((e = set(reinterpret_cast<const void*>(tc_gemm_kernel<true, kTcNmaxWide>))) != cudaSuccess) return e;
    if ((e = set(reinterpret_cast<const void*>(tc_gemm_kernel<false, kTcNmaxWide>))) != cudaSuccess) return e;
    if ((e = set(reinterpret_cast<const void*>(tc_gemm_kernel<true, kTcNmaxNarrow>))) != cudaSuccess) return e;
    if ((e = set(reinterpret_cast<const void*>(tc_gemm_kernel<false, kTcNmaxNarrow>))) != cudaSuccess) return e;
    p->ready = 1;
    return cudaSuccess;
}

inline void tc_plan_destroy(TcPlan* p) {
    if (p->xg) cudaFree(p->xg);
    if (p->xcs) cudaFree(p->xcs);
    if (p->hb) cudaFree(p->hb);
    if (p->hcs) cudaFree(p->hcs);
    p->xg = p->hb = nullptr;
    p->xcs = p->hcs = nullptr;
    p->ready = 0;
}

// The tcgen05 path pays off once the batch holds about as many token-expert
// pairs as there are experts (measured crossover on B200: between 8 and 64
// tokens at k = 6, E = 384).
inline bool tc_prefers(int T, const moe_fp4_config& cfg) {
    return 4LL * T * cfg.top_k >= 3LL * cfg.n_experts;
}

// Tile shape for a batch of T tokens: an expert holds at most T of them.
inline int tc_nmax_for(int T) { return T <= kTcNmaxNarrow ? kTcNmaxNarrow : kTcNmaxWide; }

inline TcArgs tc_args(const TcPlan& p, const ExpertArgs& g, const SlotLayout& L, int T, bool up,
                      const uint8_t* rowref, int nmax) {
    TcArgs t{};
    t.nmax = nmax;
    t.g = g;
    t.rowref = rowref;
    t.colscale = up ? p.xcs : p.hcs;
    t.hb = p.hb;
    t.L = L;
    t.T = T;
    const int ent = T * g.k;
    t.max_active = ent < g.E ? ent : g.E;
    const int head = 1024 + 256 * 16 + 4 * (5 * t.max_active + 1 + 2 * g.E + 1);
    t.off_b = (head + 1023) / 1024 * 1024;
    t.off_code = t.off_b + tc_stages(nmax) * 2 * nmax * 128;
    const int K = up ? g.H : g.I, rows = up ? g.I : g.H;
    t.spe = (K / kTcSK) % 2 == 0 ? 2 : 1;
    t.entry_bytes = t.spe * (up ? 2 * (4096 + kUnitScaleBytes) : kUnitBytes);
    int ce = (p.smem_limit - 1024 - t.off_code) / t.entry_bytes;
    if (ce > kTcMaxEntries) ce = kTcMaxEntries;
    const bool shape_ok = (K % kTcSK == 0) && (rows % kTcM == 0);
    t.centries = (ce >= 2 && shape_ok) ? ce : 0;
    return t;
}

inline size_t tc_smem_bytes(const TcArgs& t) {
    return static_cast<size_t>(t.off_code) + static_cast<size_t>(t.centries) * t.entry_bytes + 1024;   // + alignment slack
}

}  // namespace moe
