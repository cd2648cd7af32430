// decode_fused.cuh -- the whole routed-expert layer for decode batches in one
// persistent kernel: route -> x prescale -> w1/w3 GEMV + SwiGLU -> w2 GEMV ->
// router-weighted combine.
//
// Per active expert e with M_e routed entries (10100.com article 151357339,
// section "moe专家的容量瓶颈"; SwiGLU is the reading of the unnamed
// activation):
//   a1 = x W1^T, a3 = x W3^T, h = bf16(silu(a1) * a3),  o = h W2^T,
//   y[t] = sum_j w[t, j] o[t, j]   (fixed j order).
// In decode every expert weight is read once per step and the layer is bound
// by HBM: one layer at batch 1 streams 6 x 18,800,640 bytes.
//
// Arithmetic.  FP4 codes are decoded by the hardware E2M1 -> f16 convert and
// multiplied on the tensor cores with mma.sync m16n8k16 (f16 in, fp32 out):
// one MMA = 16 weight rows x 16 K of ONE 32-K scale block x 8 tokens, so the
// UE8M0 scale multiplies the fp32 block result exactly (fp4_cvt.cuh).  The
// activations enter as f16 with an exact power-of-two prescale: x per token
// row, h per (entry, 32-K block).  With at most 8 tokens per expert an MMA
// column holds one token; K order inside an MMA is free as long as A and B
// agree, and the slot layout (slot_layout.cuh) hands lane column c the eight
// codes 8c .. 8c+7 of every block, matched by eight consecutive activations.
//
// Work.  An up item is (token group of <= 8 entries of one expert, 32 rows of
// w1/w3); a down item is (group, 32 rows of w2).  A unit is one 16-byte
// aligned bulk copy of 4,352 bytes (V4.1): 16 rows x 256 K of both w1 and w3
// (up) or 32 rows x 256 K of w2 (down), codes and scales together.  Items are
// split contiguously over the CTAs (one per SM).  Inside a CTA, consumer warp
// w takes units w, w + 14, w + 28, ... and owns 2 or 3 ring slots for them;
// a producer warp streams the units (bulk copies, L2 evict-first, no
// multicast) into whichever warp's slot is free, so one slow warp never holds
// back the others' copies.  A warp accumulates its units of an item in
// registers and writes one partial; the last warp to finish an item sums the
// partials in a fixed order (results do not depend on timing) and runs the
// epilogue: SwiGLU, the f16 prescale of h and its store (up), or the
// per-entry output o (down).  For a single token the activations (x, and the
// CTA's h rows after phase 1) are staged in shared memory.
//
// Phases, separated by grid-wide barriers (all CTAs are co-resident: a
// cooperative launch of one CTA per SM); only the consumer warps wait, so the
// producer keeps streaming weights through every barrier:
//   0  route the tokens (every CTA, identically; CTA 0 writes the routing
//      outputs) or read a given routing; x rows -> f16 (one token: every CTA
//      converts x into its own shared memory and no barrier follows)
//   1  w1/w3 items; combine counters := 0
//   2  w2 items; the CTA that completes the last item of a 32-row output tile
//      combines it for every token (y, and x_out = bf16(x + y)).
// Every wait is bounded (%globaltimer); the first that gives up latches
// MOE_FP4_ETIMEOUT and makes the CTA's later waits return at once, the
// producer lets its copies in flight land before the CTA exits, and every CTA
// still arrives at every barrier, so the barrier state is consistent for the
// next launch.
#pragma once
#include "common.cuh"
#include "fp4_cvt.cuh"
#include "router.cuh"
#include "slot_layout.cuh"
#include "tma.cuh"

namespace moe {

constexpr int kDecNW = 14;                       // consumer warps (15 warps: <= 4 per SM sub-partition)
constexpr int kDecThreads = (kDecNW + 1) * 32;   // + one producer warp
constexpr int kDecMaxSpw = 3;                    // ring slots per consumer warp at most
constexpr int kDecNBufMax = 8;                   // item partial buffers (8 for one token, else 4)
constexpr int kDecRouteMax = 64;                 // T*k routed inside the kernel at most
constexpr int kDecRouteExperts = 384;            // E routed inside the kernel at most (12 logits per lane)
constexpr int kDecCombineMax = 16;               // tokens combined inside the kernel at most
constexpr int kDecStageRows = 4;                 // h rows staged in shared memory (one token)

struct DecodeArgs {
    const uint8_t* arena;
    size_t slot_bytes;
    const int32_t* slot_table;   // [L][E]
    int layer, E, k, H, I, T;    // T rows of x; T*k entries
    const float* logits;         // [T,E]: route inside the kernel; NULL: the routing below is given
    const uint8_t* keep;         // [E] or NULL
    int32_t* ids;                // [T*k]  written when routing, else unused
    float* weights;              // [T*k]  written when routing, else read (combine)
    int32_t* counts;             // [E]    written when routing
    int32_t* offsets;            // [E+1]  written when routing, else read
    int32_t* perm;               // [T*k]  written when routing, else read
    const uint16_t* x;           // [T,H] bf16
    uint16_t* xh;                // [T,H] f16 workspace: x * 2^sigma_t (more than one token)
    float* xs;                   // [T]   2^-sigma_t
    uint16_t* hh;                // [T*k, I] f16 workspace (grouped order): h * 2^sigma
    uint8_t* hs;                 // [T*k, I/32] 127 - sigma per (entry, 32-K block): h = hh * 2^(hs-127)
    float* obuf;                 // [T*k, H] fp32 per-entry outputs, entry order t*k+j
    int* tile_cnt;               // [H/16] combine arrival counters
    unsigned int* gbar;          // [4] grid barriers: {count, generation} x 2
    float* y;                    // [T,H] or NULL (per-entry outputs only)
    uint16_t* x_out;             // [T,H] or NULL
    int* err;
    unsigned long long timeout_ns;
};

struct DecodePlan {
    int ok;
    int tp;             // token columns kept in partials (1 or 8)
    int nb;             // item partial buffers in flight
    int spw;            // ring slots per consumer warp (2 or 3)
    int small;          // one token: x and the CTA's h rows in shared memory
    int max_ent, max_act, max_gs;
    int unit_bytes;
    int off_tab, off_part, off_xs, off_hs, off_ring, smem_bytes;
};

__device__ __forceinline__ void dec_named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid barrier among the CTAs' consumer warps, run by one thread per CTA
// (after the consumers' named barrier).  The last arriver resets the count
// and releases the generation; the count is 0 again after every use.
__device__ __forceinline__ void dec_grid_barrier(unsigned int* cnt, unsigned int* gen, unsigned int gen_start,
                                                 unsigned int n_cta, unsigned long long timeout_ns, int* err,
                                                 volatile int* abort_flag, int which) {
    __threadfence();
    const unsigned int old = atomicAdd(cnt, 1u);
    if (old == n_cta - 1) {
        *reinterpret_cast<volatile unsigned int*>(cnt) = 0u;
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(gen) : "memory");
        return;
    }
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_u32(gen) == gen_start) {
        if (global_timer_ns() - t0 > timeout_ns) {
            latch_error(err, ERR_ETIMEOUT, 100 + which, KID_UP);
            *abort_flag = 1;
            break;
        }
    }
}

// One unit of MMAs: two 16-row x 256 (or 128) K A tiles -- w1 and w3 rows
// of one row block (up), or two consecutive K blocks of the same w2 rows
// (down; the second may be absent: code1 == NULL) -- against B fragments.
// bfrag(m, q, j) returns this lane's B fragment for 32-K block j of 128-K
// group q of tile m; bscale(m, q, j, col) the block's activation scale of
// accumulator column 2c + col (down GEMM; 1 for the up GEMM).  Adds each
// 32-K block's fp32 result, times 2^(s-127) of its row and the activation
// scale, into acc[m*4 ..].  The two MMAs of a block (K 0-15, 16-31)
// accumulate separately, so they do not wait for each other.
template <int NTOK, int Q, typename BF, typename BS>
__device__ __forceinline__ void dec_unit_mma(const uint8_t* code0, const uint8_t* scl0, const uint8_t* code1,
                                             const uint8_t* scl1, int rowbytes, int sb, int g, int c, BF&& bfrag,
                                             BS&& bscale, float (&acc)[8]) {
    const int ntile = code1 == nullptr ? 1 : 2;
    const int off_g = g * rowbytes, off_g8 = (g + 8) * rowbytes;
    auto group = [&](int q) {
        const int chunk = swizzle_chunk(4 * q + c, g, rowbytes) * 16;   // same for rows g and g + 8
        uint4 A[2][2];
        uint32_t sg[2][2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const uint8_t* codes = (m == 0 || ntile == 1) ? code0 : code1;
            const uint8_t* scl = (m == 0 || ntile == 1) ? scl0 : scl1;
            A[m][0] = *reinterpret_cast<const uint4*>(codes + off_g + chunk);
            A[m][1] = *reinterpret_cast<const uint4*>(codes + off_g8 + chunk);
            sg[m][0] = *reinterpret_cast<const uint32_t*>(scl + g * sb + 4 * q);
            sg[m][1] = *reinterpret_cast<const uint32_t*>(scl + (g + 8) * sb + 4 * q);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                if (m >= ntile) break;
                const uint4 xb = bfrag(m, q, j);
                const float c0 = bscale(m, q, j, 0);
                const float c1 = NTOK > 1 ? bscale(m, q, j, 1) : 0.0f;
                const uint4& A0 = A[m][0];
                const uint4& A1 = A[m][1];
                uint32_t pa[4], pb[4];
                e2m1x8_to_f16x2(j == 0 ? A0.x : j == 1 ? A0.y : j == 2 ? A0.z : A0.w, pa);
                e2m1x8_to_f16x2(j == 0 ? A1.x : j == 1 ? A1.y : j == 2 ? A1.z : A1.w, pb);
                float e[4], f[4];
                mma_f16_zero(e, pa[0], pb[0], pa[1], pb[1], xb.x, xb.y);
                mma_f16_zero(f, pa[2], pb[2], pa[3], pb[3], xb.z, xb.w);
                const float s0 = ue8m0_mult(sg[m][0], j), s8 = ue8m0_mult(sg[m][1], j);
                acc[m * 4 + 0] = fmaf(e[0] + f[0], s0 * c0, acc[m * 4 + 0]);
                acc[m * 4 + 2] = fmaf(e[2] + f[2], s8 * c0, acc[m * 4 + 2]);
                if (NTOK > 1) {
                    acc[m * 4 + 1] = fmaf(e[1] + f[1], s0 * c1, acc[m * 4 + 1]);
                    acc[m * 4 + 3] = fmaf(e[3] + f[3], s8 * c1, acc[m * 4 + 3]);
                }
            }
        }
    };
    if (NTOK == 1) {   // B read from shared memory as needed: keep the code small
#pragma unroll 1
        for (int q = 0; q < Q; ++q) group(q);
    } else {           // B prefetched into registers: compile-time indices
#pragma unroll
        for (int q = 0; q < Q; ++q) group(q);
    }
}

template <int NTOK, int QU, int QD>
__global__ void __launch_bounds__(kDecThreads, 1)
moe_fp4_decode_layer(DecodeArgs a, SlotLayout L, DecodePlan p) {
    constexpr int NW = kDecNW;
    constexpr int TP = (NTOK == 1) ? 1 : 8;          // token columns kept per partial row
    constexpr int PART = 2 * 16 * TP;                // partial floats per warp per item
    extern __shared__ __align__(128) uint8_t smem[];
    const int spw = p.spw, S = p.spw * NW, NB = p.nb;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kDecMaxSpw * NW;
    int* tab = reinterpret_cast<int*>(smem + p.off_tab);
    int* act_e = tab;
    int* act_p0 = act_e + p.max_act;
    int* act_m = act_p0 + p.max_act;
    int* act_slot = act_m + p.max_act;
    int* gs_a = act_slot + p.max_act;
    int* gs_p0 = gs_a + p.max_gs;
    int* gs_n = gs_p0 + p.max_gs;
    int* slot_s = gs_n + p.max_gs;                   // this layer's row of the slot table [E]
    int* scratch = slot_s + a.E;
    // routing inside the kernel: ids, weights (entry order), perm, sorted experts
    int* r_ids = scratch;
    float* r_w = reinterpret_cast<float*>(scratch + kDecRouteMax);
    int* r_perm = scratch + 2 * kDecRouteMax;
    int* r_se = scratch + 3 * kDecRouteMax;
    int* offs_s = scratch;                           // given routing: offsets [E+1]
    float* part = reinterpret_cast<float*>(smem + p.off_part);
    uint16_t* xsm = reinterpret_cast<uint16_t*>(smem + p.off_xs);           // one token: x * 2^sigma (f16)
    float* xsig = reinterpret_cast<float*>(smem + p.off_xs + 2 * a.H);       // its 2^-sigma
    uint16_t* hsm = reinterpret_cast<uint16_t*>(smem + p.off_hs);           // staged h rows (f16)
    float* hsig = reinterpret_cast<float*>(smem + p.off_hs + kDecStageRows * 2 * a.I);   // their block scales
    // one token: B fragments of lanes without a token (g >= 1) read zeros here (512 bytes)
    const uint16_t* zrow = reinterpret_cast<const uint16_t*>(smem + p.off_hs + kDecStageRows * (2 * a.I + 4 * (a.I / 32)));
    uint8_t* ring = smem + p.off_ring;
    __shared__ int n_act_s, n_gs_s, abort_s;
    __shared__ int bcnt[kDecNBufMax], btag[kDecNBufMax];
    __shared__ unsigned int gen_start[2];
    __shared__ uint32_t red_s[NW];
    volatile int* abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, k = a.k, H = a.H, I = a.I;
    const int G = gridDim.x, b = blockIdx.x;
    const bool routed = a.logits != nullptr;
    const bool small = p.small != 0;
    const int n_ent = a.T * k;

    // the producer warp sets up the barriers while the others fetch and route
    if (warp == NW && lane == 0) {
        const unsigned int g0 = __ldcg(a.gbar + 1), g1 = __ldcg(a.gbar + 3);
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int q = 0; q < NB; ++q) {
            bcnt[q] = 0;
            btag[q] = q;
        }
        abort_s = 0;
        gen_start[0] = g0;
        gen_start[1] = g1;
        fence_barrier_init();
    }
    if (warp == NW)   // the producer warp fetches this layer's slot table row while the others route
        for (int e = lane; e < E; e += 32) slot_s[e] = __ldg(a.slot_table + static_cast<size_t>(a.layer) * E + e);
    // one token: this thread's words of x, fetched now and converted after routing
    constexpr int XW = 8;                              // words of x per consumer thread (H <= 8 * 2 * 448)
    uint32_t xw[XW];
    if (NTOK == 1 && warp < NW) {
        const uint32_t* xr = reinterpret_cast<const uint32_t*>(a.x);
#pragma unroll
        for (int q = 0; q < XW; ++q) {
            const int i = tid + q * NW * 32;
            xw[q] = i < H / 2 ? __ldg(xr + i) : 0u;
        }
    }

    // ------------------------------------------------------------ routing
    if (routed) {
        if (warp < a.T)
            route_one<kDecRouteExperts / 32>(a.logits + static_cast<size_t>(warp) * E, a.keep, E, k, warp, lane,
                                             r_ids + warp * k, r_w + warp * k, a.err);
        __syncthreads();
        if (warp == 0) {
            // stable grouping of the <= 64 entries by expert: rank of key (expert, entry)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int i = lane + 32 * h2;
                if (i < n_ent) {
                    const int key = r_ids[i] * kDecRouteMax + i;
                    int rank = 0;
                    for (int m = 0; m < n_ent; ++m) rank += (r_ids[m] * kDecRouteMax + m) < key;
                    r_perm[rank] = i;
                }
            }
            __syncwarp();
            int n = 0;
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int r = lane + 32 * h2;
                const int e = (r < n_ent) ? r_ids[r_perm[r]] : -1;
                if (r < n_ent) r_se[r] = e;
                const int prev = (r > 0 && r < n_ent) ? r_ids[r_perm[r - 1]] : -1;
                const bool start = (r < n_ent) && (r == 0 || prev != e);
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, start);
                if (start) {
                    const int pos = n + __popc(ball & lanemask_lt());
                    act_e[pos] = e;
                    act_p0[pos] = r;
                }
                n += __popc(ball);
            }
            __syncwarp();
            for (int q = lane; q < n; q += 32) act_m[q] = ((q + 1 < n) ? act_p0[q + 1] : n_ent) - act_p0[q];
            if (lane == 0) n_act_s = n;
        }
        __syncthreads();
        if (b == 0) {   // the routing outputs of the layer
            for (int i = tid; i < n_ent; i += blockDim.x) {
                a.ids[i] = r_ids[i];
                a.weights[i] = r_w[i];
                a.perm[i] = r_perm[i];
            }
            for (int e = tid; e <= E; e += blockDim.x) {
                int lo = 0;   // entries with expert < e
                for (int m = 0; m < n_ent; ++m) lo += r_se[m] < e;
                a.offsets[e] = lo;
                if (e < E) {
                    int cn = 0;
                    for (int m = 0; m < n_ent; ++m) cn += r_se[m] == e;
                    a.counts[e] = cn;
                }
            }
        }
    } else {
        for (int e = tid; e <= E; e += blockDim.x) offs_s[e] = __ldg(a.offsets + e);
        __syncthreads();
        if (warp == 0) {
            int n = 0;
            for (int base = 0; base < E; base += 32) {
                const int e = base + lane;
                const int o0 = (e < E) ? offs_s[e] : 0, o1 = (e < E) ? offs_s[e + 1] : 0;
                bool on = (e < E) && (o1 > o0);
                if (on && (o0 < 0 || o1 > n_ent)) {   // not a routing of these T*k entries
                    latch_error(a.err, ERR_EINVAL, e, KID_UP);
                    on = false;
                }
                const uint32_t ball = __ballot_sync(0xFFFFFFFFu, on);
                const int pos = n + __popc(ball & lanemask_lt());
                if (on && pos < p.max_act) {
                    act_e[pos] = e;
                    act_p0[pos] = o0;
                    act_m[pos] = o1 - o0;
                }
                n += __popc(ball);
            }
            if (lane == 0) n_act_s = min(n, p.max_act);
        }
        __syncthreads();
    }
    const int n_act = n_act_s;
    for (int q = tid; q < n_act; q += blockDim.x) act_slot[q] = slot_s[act_e[q]];
    if (warp == 0) {   // token groups of <= 8 entries
        int base = 0;
        for (int q0 = 0; q0 < n_act; q0 += 32) {
            const int q = q0 + lane;
            const int ng = (q < n_act) ? (act_m[q] + 7) >> 3 : 0;
            int incl = ng;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += v;
            }
            for (int gq = 0; gq < ng; ++gq) {
                const int s = base + incl - ng + gq;
                if (s < p.max_gs) {
                    gs_a[s] = q;
                    gs_p0[s] = act_p0[q] + 8 * gq;
                    gs_n[s] = min(8, act_m[q] - 8 * gq);
                }
            }
            base += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) n_gs_s = min(base, p.max_gs);
    }
    __syncthreads();

    const int n_gs = n_gs_s;
    const int tiles_up = I / 32, tiles_dn = H / 16;  // up items: 32 rows of w1/w3; down items: 16 rows of w2
    const int upi = 2 * L.nfu;                       // units per up item (shared by the CTA's warps)
    const int dpi = (L.nfd + 1) / 2;                 // units per down item (one warp): two K blocks each
    const int N_up = n_gs * tiles_up, N_dn = n_gs * tiles_dn;
    const int up0 = static_cast<int>((static_cast<long long>(N_up) * b) / G);
    const int up1 = static_cast<int>((static_cast<long long>(N_up) * (b + 1)) / G);
    const int dn0 = static_cast<int>((static_cast<long long>(N_dn) * b) / G);
    const int dn1 = static_cast<int>((static_cast<long long>(N_dn) * (b + 1)) / G);
    const int n_up_units = (up1 - up0) * upi;
    const int n_dn_items = dn1 - dn0;                // local down item d goes to warp d % NW
    // grouped position -> entry t*k+j (and its token row of x); -1 for an
    // entry outside [0, T*k) (a routing that is not of these tokens)
    auto entry_of = [&](int pos) -> int {
        const int ent = routed ? r_perm[pos] : __ldg(a.perm + pos);
        return (ent >= 0 && ent < n_ent) ? ent : -1;
    };
    auto token_of = [&](int pos) -> int {
        const int ent = entry_of(pos);
        return ent < 0 ? -1 : ent / k;
    };

    if (warp == NW) {
        // ---------------------------------------------------------------- producer
        // Lane w serves consumer warp w: that warp's i-th unit (unit w + 14 i)
        // goes to its slot w + 14 (i % spw) once the slot's previous unit has
        // been consumed.  The lanes issue their bulk copies in parallel and
        // independently, so one slow warp never holds back another's copies.
        const uint64_t pol = policy_evict_first();
        const int w = lane;
        const bool serve = w < NW;
        int i = 0, u = w;                                   // up: unit u = w + 14 i
        int li = u / upi, r = u - li * upi;                 // up unit: item, unit in item
        int dl = w, dv = 0;                                 // down: local item dl of this warp, unit dv in it
        bool stop = false;
        uint64_t idle_since = 0;
        for (;;) {
            const bool down = u >= n_up_units;
            const bool more = serve && !stop && (down ? dl < n_dn_items : true);
            if (!__any_sync(0xFFFFFFFFu, more)) break;
            bool progress = false;
            if (more) {
                const int ring_i = i % spw;
                const int sl = w + NW * ring_i;
                if (i < spw || mbar_test(&empty[sl], ((i / spw) - 1) & 1)) {
                    uint8_t* dst = ring + static_cast<size_t>(sl) * p.unit_bytes;
                    if (!down) {
                        const int gi = up0 + li, gs = gi / tiles_up, tile = gi - gs * tiles_up;
                        const int slot = act_slot[gs_a[gs]];
                        if (slot < 0) {
                            mbar_arrive(&full[sl]);
                        } else {
                            const size_t src = static_cast<size_t>((2 * tile + (r & 1)) * L.nfu + (r >> 1)) * L.UB;
                            mbar_arrive_expect_tx(&full[sl], static_cast<uint32_t>(L.UB));
                            bulk_g2s(dst, a.arena + static_cast<size_t>(slot) * a.slot_bytes + src,
                                     static_cast<uint32_t>(L.UB), &full[sl], pol);
                        }
                        u += NW;
                        r += NW;
                        while (r >= upi) { r -= upi; ++li; }
                    } else {
                        const int gi = dn0 + dl, gs = gi / tiles_dn, tile = gi - gs * tiles_dn;
                        const int slot = act_slot[gs_a[gs]];
                        const int nb = min(2, L.nfd - 2 * dv);   // K blocks of this unit
                        if (slot < 0) {
                            mbar_arrive(&full[sl]);
                        } else {
                            const uint8_t* src = a.arena + static_cast<size_t>(slot) * a.slot_bytes + L.up_bytes +
                                                 static_cast<size_t>(tile * L.nfd + 2 * dv) * L.DB;
                            mbar_arrive_expect_tx(&full[sl], static_cast<uint32_t>(nb * L.DB));
                            bulk_g2s(dst, src, static_cast<uint32_t>(nb * L.DB), &full[sl], pol);
                        }
                        if (++dv == dpi) { dv = 0; dl += NW; }
                    }
                    ++i;
                    progress = true;
                    idle_since = 0;
                } else if (*abort_flag) {
                    stop = true;
                } else {
                    const uint64_t now = global_timer_ns();
                    if (idle_since == 0) {
                        idle_since = now;
                    } else if (now - idle_since > a.timeout_ns) {
                        latch_error(a.err, ERR_ETIMEOUT, i, KID_UP);
                        *abort_flag = 1;
                        stop = true;
                    }
                }
            }
            if (!__any_sync(0xFFFFFFFFu, progress)) __nanosleep(64);
        }
        if (serve && *abort_flag) {   // this lane's copies in flight land before the CTA may exit
            volatile int fresh = 0;
            for (int j = 0; j < spw; ++j) {
                if (i <= j) continue;                      // uses of slot (w, j): i' = j, j + spw, ... < i
                const int last = j + ((i - 1 - j) / spw) * spw;
                fresh = 0;
                mbar_wait(&full[w + NW * j], (last / spw) & 1, &fresh);
            }
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int ctid = tid;                                  // 0 .. NW*32-1
    const int g = lane >> 2, c = lane & 3;
    // phase 0: x rows -> f16 with a per-row power-of-two prescale
    if (NTOK == 1) {   // one token: every CTA converts x into its own shared memory
        uint32_t mx = 0;
#pragma unroll
        for (int q = 0; q < XW; ++q) mx = max(mx, bf16x2_absmax(xw[q]));
        mx = __reduce_max_sync(0xFFFFFFFFu, mx);
        if (lane == 0) red_s[warp] = mx;
        dec_named_barrier(1, NW * 32);
        uint32_t tot = 0;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) tot = max(tot, red_s[w2]);
        const int sg = prescale_sigma(tot);
        const float mult = pow2i(sg);
        uint32_t* xo = reinterpret_cast<uint32_t*>(xsm);
#pragma unroll
        for (int q = 0; q < XW; ++q) {
            const int i = ctid + q * NW * 32;
            if (i < H / 2) xo[i] = bf16x2_scaled_to_f16x2(xw[q], mult);
        }
        if (ctid == 0) *xsig = pow2i(-sg);
        if (ctid < 128) reinterpret_cast<uint32_t*>(const_cast<uint16_t*>(zrow))[ctid] = 0u;
        dec_named_barrier(1, NW * 32);
    } else {
        for (int t = b; t < a.T; t += G) {
            const uint32_t* xr = reinterpret_cast<const uint32_t*>(a.x + static_cast<size_t>(t) * H);
            uint32_t mx = 0;
            for (int i = ctid; i < H / 2; i += NW * 32) mx = max(mx, bf16x2_absmax(__ldg(xr + i)));
            mx = __reduce_max_sync(0xFFFFFFFFu, mx);
            if (lane == 0) red_s[warp] = mx;
            dec_named_barrier(1, NW * 32);
            uint32_t tot = 0;
#pragma unroll
            for (int w2 = 0; w2 < NW; ++w2) tot = max(tot, red_s[w2]);
            const int sg = prescale_sigma(tot);
            const float mult = pow2i(sg);
            uint32_t* xo = reinterpret_cast<uint32_t*>(a.xh + static_cast<size_t>(t) * H);
            for (int i = ctid; i < H / 2; i += NW * 32) xo[i] = bf16x2_scaled_to_f16x2(__ldg(xr + i), mult);
            if (ctid == 0) a.xs[t] = pow2i(-sg);
            dec_named_barrier(1, NW * 32);
        }
        if (ctid == 0)
            dec_grid_barrier(a.gbar, a.gbar + 1, gen_start[0], G, a.timeout_ns, a.err, abort_flag, 0);
        dec_named_barrier(1, NW * 32);
    }

    // ---------------------------------------------------------------- item partials
    // flush: warp's partial of CTA item `seq` (buffer seq % NB), the last of
    // the item's `expected` warps reduces it and runs `epi(buffer)`.
    auto flush = [&](int seq, const float* acc, int expected, auto&& epi) {
        const int bi = seq % NB;
        if (lane == 0) {
            const uint64_t t0 = global_timer_ns();
            while (*reinterpret_cast<volatile int*>(&btag[bi]) != seq) {
                __nanosleep(32);
                if (*abort_flag) break;
                if (global_timer_ns() - t0 > a.timeout_ns) {
                    latch_error(a.err, ERR_ETIMEOUT, seq, KID_UP);
                    *abort_flag = 1;
                    break;
                }
            }
        }
        __syncwarp();
        float* pw = part + (static_cast<size_t>(bi) * NW + warp) * PART;
        // acc[m*4 + 0..3]: (row g, col 2c), (row g, col 2c+1), (row g+8, col 2c), (row g+8, col 2c+1)
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            if (TP == 1) {
                if (c == 0) {
                    pw[m * 16 + g] = acc[m * 4 + 0];
                    pw[m * 16 + g + 8] = acc[m * 4 + 2];
                }
            } else {
                pw[(m * 16 + g) * TP + 2 * c] = acc[m * 4 + 0];
                pw[(m * 16 + g) * TP + 2 * c + 1] = acc[m * 4 + 1];
                pw[(m * 16 + g + 8) * TP + 2 * c] = acc[m * 4 + 2];
                pw[(m * 16 + g + 8) * TP + 2 * c + 1] = acc[m * 4 + 3];
            }
        }
        __syncwarp();
        int last = 0;
        if (lane == 0) {
            __threadfence_block();
            last = (atomicAdd(&bcnt[bi], 1) == expected - 1);
        }
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (last) {
            __threadfence_block();
            epi(bi);
            __syncwarp();
            if (lane == 0) {
                bcnt[bi] = 0;
                __threadfence_block();
                *reinterpret_cast<volatile int*>(&btag[bi]) = seq + NB;
            }
        }
    };

    // ---------------------------------------------------------------- phase 1: w1 / w3
    {
        constexpr int Q = QU;
        const int rowbytes = L.KBu / 2, sb = L.KBu / 32;
        const int expected = min(upi, NW);
        int cur = -1;
        float acc[8];
        int slot = -1, p0 = 0, ng = 0, tile = 0, gsi = 0;
        const uint16_t* brow = nullptr;
        auto epi = [&](int bi) {
            // lane = (rb, row) of the 32 output rows; contributors r = 0..expected-1
            const int rb = lane >> 4, row = lane & 15;
            const int u_first = cur * upi;
            for (int t = 0; t < ng; ++t) {
                float a1 = 0.f, a3 = 0.f;
                for (int r = rb; r < expected; r += 2) {
                    const int w2 = (u_first + r) % NW;
                    const float* pw = part + (static_cast<size_t>(bi) * NW + w2) * PART;
                    a1 += pw[(0 * 16 + row) * TP + (TP == 1 ? 0 : t)];
                    a3 += pw[(1 * 16 + row) * TP + (TP == 1 ? 0 : t)];
                }
                const int tt = token_of(p0 + t);
                const float sx = tt < 0 ? 0.0f : (small ? *xsig : __ldcg(a.xs + tt));
                a1 *= sx;
                a3 *= sx;
                const float hv = (slot >= 0) ? a1 / (1.0f + expf(-a1)) * a3 : 0.0f;
                const uint32_t hb = f32_to_bf16_rne(hv);
                const uint32_t mx = __reduce_max_sync(0xFFFFFFFFu, hb & 0x7FFFu);
                const int sg = prescale_sigma(mx);
                const float hq = __uint_as_float(hb << 16) * pow2i(sg);
                const uint32_t h16 = f32x2_to_f16x2(hq, 0.0f) & 0xFFFFu;
                a.hh[static_cast<size_t>(p0 + t) * I + tile * 32 + lane] = static_cast<uint16_t>(h16);
                if (lane == 0) a.hs[static_cast<size_t>(p0 + t) * (I / 32) + tile] = static_cast<uint8_t>(127 - sg);
            }
            if (slot < 0 && lane == 0) latch_error(a.err, ERR_ESLOT, act_e[gs_a[gsi]], KID_UP);
        };
        int i = 0, li = warp / upi, r = warp - (warp / upi) * upi, ring_i = 0, par = 0;
        for (int u = warp; u < n_up_units; u += NW) {
            if (li != cur) {
                if (cur >= 0) flush(cur, acc, expected, epi);
                cur = li;
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = 0.f;
                const int gi = up0 + li;
                gsi = gi / tiles_up;
                tile = gi - gsi * tiles_up;
                slot = act_slot[gs_a[gsi]];
                p0 = gs_p0[gsi];
                ng = gs_n[gsi];
                const int tg = (g < ng) ? token_of(p0 + g) : -1;
                if (NTOK == 1)
                    brow = tg < 0 ? zrow : xsm;                  // zero row: no f offset below
                else
                    brow = tg < 0 ? nullptr : a.xh + static_cast<size_t>(tg) * H;
            }
            const int f = r >> 1;
            const int sl = warp + NW * ring_i;
            const uint16_t* bsrc = NTOK == 1 ? brow + (brow == zrow ? 0 : f * L.KBu) + 8 * c
                                             : (brow == nullptr ? nullptr : brow + f * L.KBu + 8 * c);
            uint4 xb[NTOK == 1 ? 1 : Q][4];
            if (NTOK > 1) {   // prefetch B (L2) before waiting for the weights
#pragma unroll
                for (int q = 0; q < Q; ++q)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        xb[NTOK == 1 ? 0 : q][j] = bsrc == nullptr ? make_uint4(0u, 0u, 0u, 0u)
                                                                   : __ldcg(reinterpret_cast<const uint4*>(bsrc + 128 * q + 32 * j));
            }
            if (!mbar_wait(&full[sl], par, abort_flag, a.timeout_ns) && lane == 0)
                latch_error(a.err, ERR_ETIMEOUT, u, KID_UP);
            if (slot >= 0) {
                const uint8_t* stg = ring + static_cast<size_t>(sl) * p.unit_bytes;
                auto bfrag = [&](int, int q, int j) -> uint4 {
                    if (NTOK == 1)   // one token: x (or the zero row) in shared memory, read as needed
                        return *reinterpret_cast<const uint4*>(bsrc + 128 * q + 32 * j);
                    return xb[NTOK == 1 ? 0 : q][j];
                };
                auto bscale = [](int, int, int, int) -> float { return 1.0f; };
                dec_unit_mma<NTOK, Q>(stg, stg + 32 * rowbytes, stg + 16 * rowbytes, stg + 32 * rowbytes + 16 * sb,
                                      rowbytes, sb, g, c, bfrag, bscale, acc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[sl]);
            ++i;
            if (++ring_i == spw) { ring_i = 0; par ^= 1; }
            r += NW;
            while (r >= upi) { r -= upi; ++li; }
        }
        if (cur >= 0) flush(cur, acc, expected, epi);
    }

    // ---------------------------------------------------------------- barrier: h complete
    if (a.y != nullptr && ctid == 0)
        for (int i2 = b; i2 < H / 16; i2 += G) a.tile_cnt[i2] = 0;
    dec_named_barrier(1, NW * 32);
    if (ctid == 0)
        dec_grid_barrier(a.gbar + 2, a.gbar + 3, gen_start[1], G, a.timeout_ns, a.err, abort_flag, 1);
    dec_named_barrier(1, NW * 32);

    // ---------------------------------------------------------------- phase 2: w2 (+ combine)
    // Warp w takes local down items w, w + 14, ...: (group, 16 rows of w2)
    // over all of I, in units of two K blocks, accumulated in registers (no
    // other warp takes part in an item).
    {
        constexpr int Q = QD;
        const int rowbytes = L.KBd / 2, sb = L.KBd / 32;
        const int nblk = I / 32;
        const int kbpb = L.KBd / 32;                      // 32-K scale blocks per K block
        // one token: stage the h rows of this CTA's groups (one entry each) in shared memory
        const int gs_first = dn0 / tiles_dn;
        const int n_stage = (dn1 > dn0) ? (dn1 - 1) / tiles_dn - gs_first + 1 : 0;
        if (NTOK == 1) {
            for (int rr = 0; rr < n_stage && rr < kDecStageRows; ++rr) {
                const int pr = gs_p0[gs_first + rr];
                const uint4* sh = reinterpret_cast<const uint4*>(a.hh + static_cast<size_t>(pr) * I);
                uint4* dh = reinterpret_cast<uint4*>(hsm + static_cast<size_t>(rr) * I);
                for (int q = ctid; q < I / 8; q += NW * 32) dh[q] = __ldcg(sh + q);
                for (int q = ctid; q < nblk; q += NW * 32)
                    hsig[rr * nblk + q] = __uint_as_float(static_cast<uint32_t>(a.hs[static_cast<size_t>(pr) * nblk + q]) << 23);
            }
            dec_named_barrier(1, NW * 32);
        }
        int pend_tile = -1;                 // tile whose combine add is in flight
        unsigned int pend_old = 0;          // its result (lane 0)
        // combine of tile pend_tile if this warp's add was the tile's last:
        // y[t] over the tile's 16 rows for every token, in fixed j order
        auto combine_pending = [&]() {
            if (pend_tile < 0) return;
            const int lastt = __shfl_sync(0xFFFFFFFFu, pend_old == static_cast<unsigned int>(n_gs - 1) ? 1 : 0, 0);
            const int tile = pend_tile;
            pend_tile = -1;
            if (!lastt) return;
            __syncwarp();   // lane 0's acquire before every lane's loads
            const int n0 = tile * 16 + (lane & 15);
            for (int t = lane >> 4; t < a.T; t += 2) {
                float yv = 0.f;
                for (int j = 0; j < k; ++j) {
                    const float wj = routed ? r_w[t * k + j] : __ldg(a.weights + t * k + j);
                    yv = fmaf(wj, __ldcg(a.obuf + static_cast<size_t>(t * k + j) * H + n0), yv);
                }
                a.y[static_cast<size_t>(t) * H + n0] = yv;
                if (a.x_out) {
                    const float xv = bf16_to_f32(a.x[static_cast<size_t>(t) * H + n0]);
                    a.x_out[static_cast<size_t>(t) * H + n0] = f32_to_bf16_rne(xv + yv);
                }
            }
        };
        int i = (n_up_units - warp + NW - 1) / NW;       // this warp's up units: its ring position now
        if (i < 0) i = 0;
        int ring_i = i % spw, par = (i / spw) & 1;
        for (int dl = warp; dl < n_dn_items; dl += NW) {
            const int gi = dn0 + dl;
            const int gsi = gi / tiles_dn, tile = gi - gsi * tiles_dn;
            const int slot = act_slot[gs_a[gsi]];
            const int p0 = gs_p0[gsi], ng = gs_n[gsi];
            const uint16_t* brow;
            const float* hrow0 = nullptr;       // one token: block scales of the entry (shared memory)
            const uint8_t* hr0 = nullptr;       // block scale exponents of column 2c
            const uint8_t* hr1 = nullptr;       // and of column 2c + 1
            if (NTOK == 1) {
                brow = (g < ng) ? hsm + static_cast<size_t>(gsi - gs_first) * I : zrow;
                hrow0 = hsig + (gsi - gs_first) * nblk;
            } else {
                brow = (g < ng) ? a.hh + static_cast<size_t>(p0 + g) * I : nullptr;
                hr0 = (2 * c < ng) ? a.hs + static_cast<size_t>(p0 + 2 * c) * nblk : nullptr;
                hr1 = (2 * c + 1 < ng) ? a.hs + static_cast<size_t>(p0 + 2 * c + 1) * nblk : nullptr;
            }
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
            for (int dv = 0; dv < dpi; ++dv) {
                const int sl = warp + NW * ring_i;
                const bool two = 2 * dv + 1 < L.nfd;     // second K block present
                const int kbase = 2 * dv * L.KBd;         // K of this unit's first block
                uint4 xb[NTOK == 1 ? 1 : 2][NTOK == 1 ? 1 : Q][4];
                uint32_t hw0[NTOK == 1 ? 1 : 2][NTOK == 1 ? 1 : Q], hw1[NTOK == 1 ? 1 : 2][NTOK == 1 ? 1 : Q];
                if (NTOK > 1) {   // prefetch B and its block scales (L2) before waiting for the weights
#pragma unroll
                    for (int m = 0; m < 2; ++m)
#pragma unroll
                        for (int q = 0; q < Q; ++q) {
                            const int kk = kbase + m * L.KBd + 128 * q;
                            const bool ok = m == 0 || two;
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                xb[NTOK == 1 ? 0 : m][NTOK == 1 ? 0 : q][j] =
                                    (brow == nullptr || !ok) ? make_uint4(0u, 0u, 0u, 0u)
                                                             : __ldcg(reinterpret_cast<const uint4*>(brow + kk + 32 * j + 8 * c));
                            const int kb = kk / 32;   // a multiple of 4 (I/32 too): four exponents in one word
                            hw0[NTOK == 1 ? 0 : m][NTOK == 1 ? 0 : q] =
                                (hr0 == nullptr || !ok) ? 0u : __ldcg(reinterpret_cast<const unsigned int*>(hr0 + kb));
                            hw1[NTOK == 1 ? 0 : m][NTOK == 1 ? 0 : q] =
                                (hr1 == nullptr || !ok) ? 0u : __ldcg(reinterpret_cast<const unsigned int*>(hr1 + kb));
                        }
                }
                if (!mbar_wait(&full[sl], par, abort_flag, a.timeout_ns) && lane == 0)
                    latch_error(a.err, ERR_ETIMEOUT, dl, KID_DOWN);
                if (slot >= 0) {
                    const uint8_t* stg = ring + static_cast<size_t>(sl) * p.unit_bytes;
                    const uint16_t* bsrc = NTOK == 1 ? brow + (brow == zrow ? 0 : kbase) + 8 * c : nullptr;
                    auto bfrag = [&](int m, int q, int j) -> uint4 {
                        if (NTOK == 1)   // one token: staged h row (or the zero row) in shared memory
                            return *reinterpret_cast<const uint4*>(bsrc + (brow == zrow ? 0 : m * L.KBd) + 128 * q +
                                                                   32 * j);
                        return xb[NTOK == 1 ? 0 : m][NTOK == 1 ? 0 : q][j];
                    };
                    auto bscale = [&](int m, int q, int j, int col) -> float {
                        if (NTOK == 1) return hrow0[kbase / 32 + m * kbpb + 4 * q + j];
                        return ue8m0_mult(col == 0 ? hw0[NTOK == 1 ? 0 : m][NTOK == 1 ? 0 : q]
                                                   : hw1[NTOK == 1 ? 0 : m][NTOK == 1 ? 0 : q], j);
                    };
                    dec_unit_mma<NTOK, Q>(stg, stg + 16 * rowbytes, two ? stg + L.DB : nullptr,
                                          two ? stg + L.DB + 16 * rowbytes : nullptr, rowbytes, sb, g, c, bfrag,
                                          bscale, acc);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[sl]);
                if (a.y != nullptr) combine_pending();
                ++i;
                if (++ring_i == spw) { ring_i = 0; par ^= 1; }
            }
            // epilogue of the item: o rows of the entries (rows g, g+8 of the tile; columns 2c, 2c+1)
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const int col = 2 * c + cc;
                if (col >= ng || (NTOK == 1 && cc == 1)) continue;
                const int ent = entry_of(p0 + col);
                if (ent < 0) continue;
                float* orow = a.obuf + static_cast<size_t>(ent) * H + tile * 16;
                orow[g] = slot >= 0 ? acc[cc] + acc[4 + cc] : 0.0f;
                orow[g + 8] = slot >= 0 ? acc[2 + cc] + acc[6 + cc] : 0.0f;
            }
            if (slot < 0 && lane == 0) latch_error(a.err, ERR_ESLOT, act_e[gs_a[gsi]], KID_DOWN);
            if (a.y != nullptr) {
                // lane 0's acquire-release add orders the warp's o stores before it
                // (the warp barrier orders them before lane 0) and the last arriver's
                // loads after every other arriver's stores; its result is looked at
                // after the warp's next unit (combine_pending)
                if (pend_tile >= 0) combine_pending();
                __syncwarp();
                if (lane == 0) {
                    unsigned int old;
                    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                                 : "=r"(old) : "l"(a.tile_cnt + tile) : "memory");
                    pend_old = old;
                }
                pend_tile = tile;
            }
        }
        if (a.y != nullptr) combine_pending();
    }
}

// Host-side plan; ok = 0 when the shape or the batch does not fit.
inline DecodePlan make_decode_plan(const SlotLayout& L, int T, int k, int E, bool routed, int smem_limit, int grid) {
    DecodePlan p{};
    const int ent = T * k;
    if (T <= 0 || (routed && (ent > kDecRouteMax || T > kDecNW || E > kDecRouteExperts))) return p;
    if ((L.KBu != 128 && L.KBu != 256) || (L.KBd != 128 && L.KBd != 256) || L.I % 32 || L.H % 32) return p;
    // one token: x held 8 words per consumer thread, and the h rows of a CTA's
    // down items (at most k / grid + 2 groups) fit the staging rows
    p.small = (T == 1 && L.H <= 2 * 8 * kDecNW * 32 && (k + grid - 1) / grid + 2 <= kDecStageRows);
    p.tp = p.small ? 1 : 8;
    p.nb = p.small ? kDecNBufMax : 4;
    p.max_ent = ent;
    p.max_act = ent < E ? ent : E;
    p.max_gs = ent < ent / 8 + p.max_act ? ent : ent / 8 + p.max_act;   // sum of ceil(m/8) over active experts
    const size_t ub = L.UB > 2 * L.DB ? L.UB : 2 * L.DB;
    p.unit_bytes = static_cast<int>((ub + 127) / 128 * 128);
    p.off_tab = 2 * kDecMaxSpw * kDecNW * 8;
    const int scratch = routed ? 4 * kDecRouteMax : E + 1;
    const int tab_ints = 4 * p.max_act + 3 * p.max_gs + E + scratch;
    p.off_part = (p.off_tab + 4 * tab_ints + 127) / 128 * 128;
    p.off_xs = p.off_part + 4 * p.nb * kDecNW * 2 * 16 * p.tp;
    p.off_xs = (p.off_xs + 127) / 128 * 128;
    p.off_hs = p.off_xs + (p.small ? (2 * L.H + 4 + 127) / 128 * 128 : 0);
    const int hs_bytes = p.small ? kDecStageRows * (2 * L.I + 4 * (L.I / 32)) + 512 : 0;
    p.off_ring = (p.off_hs + hs_bytes + 127) / 128 * 128;
    for (int spw = kDecMaxSpw; spw >= 2; --spw) {
        p.spw = spw;
        p.smem_bytes = p.off_ring + spw * kDecNW * p.unit_bytes;
        if (p.smem_bytes <= smem_limit) break;
    }
    p.ok = p.smem_bytes <= smem_limit;
    return p;
}

}  // namespace moe
