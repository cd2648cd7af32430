// decode_mx.cuh -- the whole routed-expert layer for decode batches in one
// persistent kernel on the block-scaled FP4 tensor cores:
// route -> x digit planes -> w1/w3 (tcgen05.mma kind::mxf4) + SwiGLU ->
// h digit planes -> w2 (kind::mxf4) -> router-weighted combine.
//
// Per active expert e with M_e routed entries (10100.com article 151357339,
// section "moe专家的容量瓶颈"; SwiGLU is the reading of the unnamed
// activation):
//   a1 = x W1^T, a3 = x W3^T, h = bf16(silu(a1) * a3),  o = h W2^T,
//   y[t] = sum_j w[t, j] o[t, j]   (fixed j order).
// In decode every expert weight is read once per step and the layer is bound
// by HBM: one layer at batch 1 streams 6 x 18,800,640 bytes.
//
// Arithmetic.  The weights stay in their storage format: the tensor core
// multiplies E2M1 codes with their UE8M0 block scales itself (kind::mxf4,
// M = 128 weight rows, K = 64 per instruction, fp32 accumulate in TMEM), so
// no instruction of this kernel decodes a weight.  That MMA wants B in E2M1
// as well, so every bf16 activation row (x, and h for the second GEMM) is
// split exactly into 8 E2M1 "digit planes" per 32-element block: with
// 2^E0 < max|v| <= 2^(E0+1), plane p holds digits d in {0, +-0.5 .. +-2} at
// scale 2^(E0 - 2p) (a UE8M0 block scale), chosen greedily by rounding the
// remainder to the nearest half; each remainder is at most a quarter of the
// plane's unit, so after 8 planes it is below 2^(E0-16) < max|v| * 2^-16,
// and every element within 2^9 of the block maximum is represented exactly
// (bf16 has 8 significant bits).  The planes are the N columns of the MMA
// (8 per entry); the epilogue adds them in fp32.  Power-of-two rescalings of
// a row rescale its planes exactly (the digits depend on v / 2^E0 only).
//
// Work.  A unit is one 128-row x 128-K tile of one weight matrix (8,704
// bytes: codes and block scales, slot_layout.cuh) plus the B tile of its
// token group (<= 4 entries x 8 planes x 128 K, and their scale bytes).  An
// up item is (token group, 128 rows of w1 and w3) over all of H; a down item
// (group, 128 rows of w2) over all of I.  The up units of all items form one
// sequence split contiguously over the CTAs (one per SM), the down units
// another; an item cut by a range boundary is finished by whichever of its
// CTAs completes last, which adds the fp32 partials in CTA order (results do
// not depend on timing).  Inside a CTA:
//   warps 7-15, lane 0  producers: bulk copies of unit i (A + scales from the
//                       arena, B + B scales from the plane buffers) into ring
//                       slot i % S, warp 7 + i % 9 per unit (S a multiple of
//                       9, so a slot always has the same producer and issuer);
//   warps 4-6, lane 0   MMA issuers: issuer i % 3 takes unit i -- tcgen05.cp
//                       of both scale atoms into its own TMEM columns, two
//                       K = 64 MMAs into its own double-buffered accumulator,
//                       tcgen05.commit frees the slot.  One thread's tcgen05
//                       stream stalls at every commit (measured on B200: one
//                       issuer 307 ns per unit, three keep the pipe ahead of
//                       HBM), so three issuers take turns;
//   warps 0-3           epilogue (TMEM lane quadrant = warp): planes and the
//                       issuers' accumulators summed (fixed order), then a partial, or the item's finish: SwiGLU, bf16 h
//                       and its digit planes (up), per-entry o and the
//                       combine of a 128-row output tile by the CTA that
//                       completes its last item (down);
//   all warps           prologue: routing, and a share of the x planes.
// Ordering across CTAs has no grid barrier: the x planes are counted, every
// up item raises a flag once its h planes are stored, and a producer lane
// checks the flag (acquire) before it copies the h planes of a down unit --
// the weights of down units stream while h is still being made.  Flags carry
// the launch's sequence number (advanced by the last CTA to exit); counters
// come in two banks, launch n counting in bank n % 2 and clearing the other
// one for launch n + 1, so nothing is reset between launches, not even after
// a launch that gave up.  Every wait is bounded
// (%globaltimer); the first that gives up latches MOE_FP4_ETIMEOUT and makes
// the CTA's other waits return at once; copies and MMAs in flight complete
// before the CTA exits.
#pragma once
#include "common.cuh"
#include "router.cuh"
#include "slot_layout.cuh"
#include "tma.cuh"

namespace moe {

constexpr int kMxWarps = 16;
constexpr int kMxThreads = kMxWarps * 32;
constexpr int kMxEpiWarps = 4;                    // warps 0-3: TMEM lane quadrant = warp
constexpr int kMxMmaWarp = 4;                     // warps 4 .. 9: one MMA issuer lane each
constexpr int kMxIssuers = 6;
constexpr int kMxProdWarp = kMxMmaWarp + kMxIssuers;   // warps 10 .. 15: one producer lane each
constexpr int kMxProducers = kMxWarps - kMxProdWarp;
// Ring slots come in multiples of this: slot s is then always filled by
// producer s % 6 and drained by issuer s % 6, so each thread sees the uses of
// its slots in order and every mbarrier parity wait is unambiguous.
constexpr int kMxSlotQuantum = 6;
static_assert(kMxSlotQuantum % kMxProducers == 0 && kMxSlotQuantum % kMxIssuers == 0, "slot ownership");
constexpr int kMxGroup = 2;                       // entries per token group: N = 8 * entries <= 16
constexpr int kMxPlanes = 8;                      // E2M1 digit planes per activation row
constexpr int kMxPlaneTile = 512;                 // one row's planes for 128 K: [4 blocks][8 planes][16 B]
constexpr int kMxPlaneScale = 128;                // their scales: [8 planes][16 B], byte b = block b
constexpr int kMxOffB = kUnitBytes;               // slot: A codes | A scales | B (g x 512) | B scale rows (g x 128)
constexpr int kMxMaxSlots = 24;
constexpr int kMxRouteMax = 64;                   // T*k routed inside the kernel at most
constexpr int kMxRouteExperts = 384;              // E routed inside the kernel at most
constexpr int kMxCombineMax = 16;                 // tokens combined inside the kernel at most
constexpr int kMxMaxEntries = 768;                // token-expert entries of one launch at most (workspace)
constexpr int kMxPartFloats = 3 * 2 * kMxGroup * 128;   // per CTA: up 2 sides x 2 mats, down 2 sides
constexpr int kMxPartUp = 2 * kMxGroup * 128;            // floats of one up side (w1 then w3)
constexpr int kMxPartDown = kMxGroup * 128;              // floats of one down side
constexpr uint32_t kMxTmemCols = 512;             // accumulators [2][issuer][16 g] columns, scale atoms at 384 + 8 w

struct MxArgs {
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
    uint8_t* xp;                 // [T][H/128][512] digit planes of x
    uint8_t* xsf;                // [T][H/128][128] their block scales
    uint8_t* hp;                 // [T*k][I/128][512] digit planes of h (grouped entry order)
    uint8_t* hsf;                // [T*k][I/128][128]
    float* part;                 // [grid][kMxPartFloats] split-item partial sums
    unsigned int* seq;           // [2] launch sequence number, CTAs exited
    unsigned int* cnt;           // [2][cnt_cap] counter banks: x planes, up items, down items, output tiles
    int cnt_cap;                 // counters per bank (>= 1 + max up items + max down items + H/128)
    unsigned int* ready;         // [max up items] h planes of an up item stored (tag)
    const uint8_t* zero;         // >= 512 zero bytes: the B tile of an entry without a token
    float* obuf;                 // [T*k, H] fp32 per-entry outputs, entry order t*k+j
    float* y;                    // [T,H] or NULL (per-entry outputs only)
    uint16_t* x_out;             // [T,H] or NULL
    int* err;
    unsigned long long timeout_ns;
};

struct MxPlan {
    int ok;
    int gmax;                    // entries per token group (1 for one token, else kMxGroup)
    int slot_bytes;              // kUnitBytes + gmax * (512 + 128)
    int slots;                   // ring slots (a multiple of kMxSlotQuantum)
    int max_ent, max_act, max_gs;
    int max_up_items, max_dn_items;
    int off_tab, off_ring, smem_bytes;
};

// ------------------------------------------------------------------ PTX helpers
// Shared-memory operand descriptor, K-major without swizzle: core matrices of
// 8 rows x 16 bytes, `lbo` bytes apart along K and `sbo` bytes apart along M/N.
__device__ __forceinline__ uint64_t mx_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32) | (static_cast<uint64_t>(1) << 46);
}

// Instruction descriptor of tcgen05.mma kind::mxf4 (block scale): A, B E2M1
// (format 1), K-major, UE8M0 scales (bit 23), M = 128, N = n; sf_id selects
// the scale bytes sf_id, sf_id + 1 of each TMEM scale column.
__host__ __device__ inline uint32_t mx_idesc(int n, int sf_id) {
    return (static_cast<uint32_t>(sf_id) << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (1u << 23) | (static_cast<uint32_t>(128 >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}

__device__ __forceinline__ void mx_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// 32 rows x 16 bytes of shared memory -> TMEM lanes 0-31 of every lane quadrant, 4 columns.
__device__ __forceinline__ void mx_cp_atom(uint32_t taddr, uint32_t saddr) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(mx_desc(saddr, 16, 128))
                 : "memory");
}

__device__ __forceinline__ void mx_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mx_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void mx_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Sum of 8 consecutive fp32 TMEM columns of this thread's lane (one entry's planes).
__device__ __forceinline__ float mx_ld8_sum(uint32_t taddr) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    float s = 0.0f;
#pragma unroll
    for (int q = 0; q < 8; ++q) s += __uint_as_float(r[q]);
    return s;
}

__device__ __forceinline__ void mx_named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ unsigned int mx_ld_acquire(const unsigned int* p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Arrival on a counter (acquire-release); returns the count after it.
__device__ __forceinline__ unsigned int mx_arrive(unsigned int* c) {
    unsigned int old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(c) : "memory");
    return old + 1u;
}
__device__ __forceinline__ void mx_st_release(unsigned int* p, unsigned int v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Generic-proxy writes (by any thread, ordered before this point) become
// visible to the async proxy (bulk copies) issued after it.
__device__ __forceinline__ void mx_fence_proxy_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Split one 32-element block (v = this lane's element, a bf16 value held in
// fp32) into kMxPlanes E2M1 digit planes: plane p -> 16 bytes at pc + 16 p
// (element 2j in the low nibble of byte j) and its UE8M0 scale at sf[16 p].
// A zero block gets zero planes; a block holding inf/NaN gets scale byte 255
// (NaN) in plane 0, which the tensor core propagates.
__device__ __forceinline__ void mx_split_block(float v, int lane, uint8_t* pc, uint8_t* sf) {
    const uint32_t mb = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(v) & 0x7FFFFFFFu);
    int e0 = 0;
    bool live = mb != 0u && mb < 0x7F800000u;
    if (live) {
        const int field = static_cast<int>(mb >> 23);
        const uint32_t frac = mb & 0x7FFFFFu;
        if (field == 0) {   // subnormal maximum: 2^lz <= frac < 2^(lz+1), value = frac * 2^-149
            const int lz = 31 - __clz(frac);
            e0 = (lz - 149) - ((frac & (frac - 1u)) == 0u ? 1 : 0);
        } else {
            e0 = (field - 127) - (frac == 0u ? 1 : 0);
        }
    }
    float r = v;
#pragma unroll
    for (int p = 0; p < kMxPlanes; ++p) {
        const int s = e0 - 2 * p;               // plane scale 2^s
        uint32_t code = 0u;
        int sbyte = 0;
        if (live && s >= -127) {
            const float d = rintf(2.0f * ldexpf(r, -s)) * 0.5f;   // nearest half: |d| <= 2
            const float ad = fabsf(d);
            code = static_cast<uint32_t>(2.0f * ad) | (d < 0.0f ? 8u : 0u);
            r -= ldexpf(d, s);                  // exact: |r| shrinks below 2^(s-2)
            sbyte = s + 127;
        } else if (!live && p == 0 && mb != 0u) {
            sbyte = 255;
        }
        uint32_t w = code << (4 * (lane & 7));
        w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
        w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
        w |= __shfl_xor_sync(0xFFFFFFFFu, w, 4);
        if ((lane & 7) == 0) *reinterpret_cast<uint32_t*>(pc + 16 * p + 4 * (lane >> 3)) = w;
        if (lane == 0) sf[16 * p] = static_cast<uint8_t>(sbyte);
    }
}

// Contiguous split of n units over G CTAs: CTA b takes [n b / G, n (b+1) / G).
__device__ __forceinline__ int mx_range_start(int n, int G, int b) {
    return static_cast<int>((static_cast<long long>(n) * b) / G);
}
// The CTA whose range holds unit u (the largest b with start(b) <= u).
__device__ __forceinline__ int mx_cta_of(int n, int G, int u) {
    return static_cast<int>(((static_cast<long long>(u) + 1) * G + n - 1) / n) - 1;
}

// ------------------------------------------------------------------ kernel
__global__ void __launch_bounds__(kMxThreads, 1) moe_fp4_decode_mx(MxArgs a, SlotLayout L, MxPlan p) {
    extern __shared__ __align__(1024) uint8_t mx_smem_raw[];
    uint8_t* smem = mx_smem_raw + ((1024u - (smem_u32(mx_smem_raw) & 1023u)) & 1023u);
    const int S = p.slots;
    const int SB = p.slot_bytes, GM = p.gmax;
    const int off_sfb = kMxOffB + GM * kMxPlaneTile;   // B scale rows; tcgen05.cp reads 512 bytes from there
    const int acc_cols = 16 * GM;                      // one issuer's accumulator: w1 (or w2) at +0, w3 at +8 g
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);            // unit landed in slot s
    uint64_t* empty = full + kMxMaxSlots;                          // slot s consumed by the MMAs
    uint64_t* accf = empty + kMxMaxSlots;                          // [2] accumulator complete
    uint64_t* acce = accf + 2;                                     // [2] accumulator read by the epilogue
    uint64_t* fin = acce + 2;                                      // [kMxIssuers] last MMAs done
    int* tab = reinterpret_cast<int*>(smem + p.off_tab);
    int* act_e = tab;
    int* act_p0 = act_e + p.max_act;
    int* act_m = act_p0 + p.max_act;
    int* act_slot = act_m + p.max_act;
    int* gs_a = act_slot + p.max_act;
    int* gs_p0 = gs_a + p.max_gs;
    int* gs_n = gs_p0 + p.max_gs;
    int* slot_s = gs_n + p.max_gs;                                 // this layer's row of the slot table [E]
    int* scratch = slot_s + a.E;
    int* r_ids = scratch;                                          // routing inside the kernel
    float* r_w = reinterpret_cast<float*>(scratch + kMxRouteMax);
    int* r_perm = scratch + 2 * kMxRouteMax;
    int* r_se = scratch + 3 * kMxRouteMax;
    int* offs_s = scratch;                                         // given routing: offsets [E+1]
    uint8_t* ring = smem + p.off_ring;
    __shared__ uint32_t tmem_s;
    __shared__ int n_act_s, n_gs_s, abort_s, last_s;
    __shared__ unsigned int tag_s;
    __shared__ int last_issue[kMxMaxSlots];                        // last unit copied into each slot
    volatile int* abort_flag = &abort_s;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, k = a.k, H = a.H;
    const int G = gridDim.x, b = blockIdx.x;
    const bool routed = a.logits != nullptr;
    const int n_ent = a.T * k;
    const int KU = L.KU, KD = L.KD, RT = L.RT, NT = L.NT;

    if (tid == 0) {
        tag_s = mx_ld_acquire(a.seq) + 1u;   // this launch's tag (never 0 for 2^32 launches)
        for (int s = 0; s < kMxMaxSlots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int q = 0; q < 2; ++q) {
            mbar_init(&accf[q], kMxIssuers);
            mbar_init(&acce[q], kMxEpiWarps);
        }
        for (int q = 0; q < kMxIssuers; ++q) mbar_init(&fin[q], 1);
        for (int s = 0; s < kMxMaxSlots; ++s) last_issue[s] = -1;
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == kMxMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_s)),
                     "r"(kMxTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (warp == kMxProdWarp)   // this layer's slot table row
        for (int e = lane; e < E; e += 32) slot_s[e] = __ldg(a.slot_table + static_cast<size_t>(a.layer) * E + e);

    // the counter bank of the next launch starts at zero
    {
        const unsigned int nb = (mx_ld_acquire(a.seq) + 2u) & 1u;   // bank of launch seq + 1
        unsigned int* other = a.cnt + static_cast<size_t>(nb) * a.cnt_cap;
        for (int i = b * kMxThreads + tid; i < a.cnt_cap; i += G * kMxThreads) other[i] = 0u;
    }

    // ------------------------------------------------------------ x digit planes (a share per warp)
    {
        const int nblk = a.T * (H / 32);
        // blocks are dealt across CTAs first, highest warp first (low warps route)
        for (int q = (kMxWarps - 1 - warp) * G + b; q < nblk; q += kMxWarps * G) {
            const int t = q / (H / 32), kb = q - t * (H / 32);
            const float v = bf16_to_f32(__ldg(a.x + static_cast<size_t>(t) * H + 32 * kb + lane));
            const size_t tile = static_cast<size_t>(t) * KU + (kb >> 2);
            mx_split_block(v, lane, a.xp + tile * kMxPlaneTile + (kb & 3) * 128, a.xsf + tile * kMxPlaneScale + (kb & 3));
        }
    }

    // ------------------------------------------------------------ routing
    if (routed) {
        for (int t = warp; t < a.T; t += kMxWarps)
            route_one<kMxRouteExperts / 32>(a.logits + static_cast<size_t>(t) * E, a.keep, E, k, t, lane,
                                           r_ids + t * k, r_w + t * k, a.err);
        __syncthreads();
        if (warp == 0) {
            // stable grouping of the <= 64 entries by expert: rank of key (expert, entry)
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int i = lane + 32 * h2;
                if (i < n_ent) {
                    const int key = r_ids[i] * kMxRouteMax + i;
                    int rank = 0;
                    for (int m = 0; m < n_ent; ++m) rank += (r_ids[m] * kMxRouteMax + m) < key;
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
    // x planes of this CTA stored: count it (the copies of x planes wait for every CTA)
    if (tid == 0) {
        __threadfence();
        mx_fence_proxy_global();
        atomicAdd(a.cnt + static_cast<size_t>(tag_s & 1u) * a.cnt_cap, 1u);
    }
    const int n_act = n_act_s;
    for (int q = tid; q < n_act; q += blockDim.x) act_slot[q] = slot_s[act_e[q]];
    if (warp == 0) {   // token groups of <= kMxGroup entries
        int base = 0;
        for (int q0 = 0; q0 < n_act; q0 += 32) {
            const int q = q0 + lane;
            const int ng = (q < n_act) ? (act_m[q] + GM - 1) / GM : 0;
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
                    gs_p0[s] = act_p0[q] + GM * gq;
                    gs_n[s] = min(GM, act_m[q] - GM * gq);
                }
            }
            base += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) n_gs_s = min(base, p.max_gs);
    }
    mx_fence_before();
    __syncthreads();
    mx_fence_after();

    // ------------------------------------------------------------ work
    const int n_gs = n_gs_s;
    const unsigned int tag = tag_s;
    const int upi = 2 * KU, dpi = KD;                       // units per up / down item
    const int NU = n_gs * RT * upi, ND = n_gs * NT * dpi;   // units of all items
    const int u0 = mx_range_start(NU, G, b), u1 = mx_range_start(NU, G, b + 1);
    const int d0 = mx_range_start(ND, G, b), d1 = mx_range_start(ND, G, b + 1);
    const int nu = u1 - u0, n_units = nu + (d1 - d0);
    const int up_first = nu > 0 ? u0 / upi : 0, n_up_parts = nu > 0 ? (u1 - 1) / upi - up_first + 1 : 0;
    const int dn_first = d1 > d0 ? d0 / dpi : 0, n_dn_parts = d1 > d0 ? (d1 - 1) / dpi - dn_first + 1 : 0;
    const int n_parts = n_up_parts + n_dn_parts;
    unsigned int* x_cnt = a.cnt + static_cast<size_t>(tag & 1u) * a.cnt_cap;   // this launch's bank
    unsigned int* up_cnt = x_cnt + 1;
    unsigned int* dn_cnt = up_cnt + p.max_up_items;
    unsigned int* tile_cnt = dn_cnt + p.max_dn_items;
    // grouped position -> entry t*k+j; -1 for an entry outside [0, T*k)
    auto entry_of = [&](int pos) -> int {
        const int ent = routed ? r_perm[pos] : __ldg(a.perm + pos);
        return (ent >= 0 && ent < n_ent) ? ent : -1;
    };
    // part j of this CTA: its item and its unit range (global unit indices)
    auto part_of = [&](int j, bool& up, int& item, int& ua, int& ub) {
        up = j < n_up_parts;
        if (up) {
            item = up_first + j;
            ua = max(item * upi, u0);
            ub = min((item + 1) * upi, u1);
        } else {
            item = dn_first + (j - n_up_parts);
            ua = max(item * dpi, d0);
            ub = min((item + 1) * dpi, d1);
        }
    };
    const uint32_t ring_base = smem_u32(ring);

    if (warp >= kMxProdWarp) {
        // ------------------------------------------------------------ producers
        // Lane 0 of producer warp w copies units w, w + 11, ...: unit i to slot
        // i % S once the slot's previous unit has been consumed.  x planes are
        // copied once every CTA has stored its share; h planes once their up
        // item is done.
        if (lane == 0) {
            const int pw = warp - kMxProdWarp;
            const uint64_t pol = policy_evict_first();
            bool x_ok = false;
            int ready_item = -1;
            int i = pw;
            for (; i < n_units; i += kMxProducers) {
                const int s = i % S;
                if (i >= S && !mbar_poll(&empty[s], ((i / S) - 1) & 1, abort_flag, a.timeout_ns)) {
                    latch_error(a.err, ERR_ETIMEOUT, i, KID_UP);
                    *abort_flag = 1;
                    break;
                }
                const bool up = i < nu;
                const int gu = up ? u0 + i : d0 + (i - nu);
                const int item = up ? gu / upi : gu / dpi, v = up ? gu - item * upi : gu - item * dpi;
                const int gs = up ? item / RT : item / NT, tile = up ? item - gs * RT : item - gs * NT;
                const int mat = up ? v / KU : 0, ku = up ? v - mat * KU : v;
                const int slot = act_slot[gs_a[gs]];
                const int ng = gs_n[gs], p0 = gs_p0[gs];
                if (slot < 0) {   // expert not resident: nothing to copy (the epilogue writes zeros)
                    mbar_arrive(&full[s]);
                    continue;
                }
                // the weights first (they depend on the routing only), then the B
                // operand once its producers are done: expect_tx without an arrive
                // keeps the phase open until the B copies are issued too
                uint8_t* dst = ring + static_cast<size_t>(s) * SB;
                const size_t uoff = up ? up_unit_offset(L, mat, tile, ku) : down_unit_offset(L, tile, ku);
                mbar_expect_tx(&full[s], static_cast<uint32_t>(kUnitBytes));
                bulk_g2s(dst, a.arena + static_cast<size_t>(slot) * a.slot_bytes + uoff, kUnitBytes, &full[s], pol);
                reinterpret_cast<volatile int*>(last_issue)[s] = i;
                bool ok = true;
                const uint64_t t0 = global_timer_ns();
                if (up && !x_ok) {
                    while (mx_ld_acquire(x_cnt) < static_cast<unsigned int>(G)) {
                        if (*abort_flag || global_timer_ns() - t0 > a.timeout_ns) { ok = false; break; }
                        __nanosleep(64);
                    }
                    x_ok = ok;
                } else if (!up && ready_item != gs * RT + ku) {
                    while (mx_ld_acquire(a.ready + gs * RT + ku) != tag) {
                        if (*abort_flag || global_timer_ns() - t0 > a.timeout_ns) { ok = false; break; }
                        __nanosleep(64);
                    }
                    if (ok) ready_item = gs * RT + ku;
                }
                if (!ok) {
                    latch_error(a.err, ERR_ETIMEOUT, 200 + (up ? 0 : 1), up ? KID_UP : KID_DOWN);
                    *abort_flag = 1;
                    mbar_arrive(&full[s]);   // the phase now completes once the weights have landed
                    break;
                }
                mx_fence_proxy_global();
                mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(ng * (kMxPlaneTile + kMxPlaneScale)));
                for (int e = 0; e < ng; ++e) {
                    const uint8_t* pb;
                    const uint8_t* ps;
                    if (up) {
                        const int ent = entry_of(p0 + e);
                        const size_t tt = ent < 0 ? 0 : static_cast<size_t>(ent / k) * KU + ku;
                        pb = ent < 0 ? a.zero : a.xp + tt * kMxPlaneTile;
                        ps = ent < 0 ? a.zero : a.xsf + tt * kMxPlaneScale;
                    } else {
                        const size_t tt = static_cast<size_t>(p0 + e) * KD + ku;
                        pb = a.hp + tt * kMxPlaneTile;
                        ps = a.hsf + tt * kMxPlaneScale;
                    }
                    bulk_g2s_nohint(dst + kMxOffB + e * kMxPlaneTile, pb, kMxPlaneTile, &full[s]);
                    bulk_g2s_nohint(dst + off_sfb + e * kMxPlaneScale, ps, kMxPlaneScale, &full[s]);
                }
            }
            if (*abort_flag) {   // this warp's copies in flight land before the CTA may exit
                volatile int fresh = 0;
                for (int j = pw; j < i && j < n_units; j += kMxProducers) {
                    // a later unit in the same slot was only copied after unit j had been consumed
                    if (reinterpret_cast<volatile int*>(last_issue)[j % S] != j) continue;
                    fresh = 0;
                    mbar_wait(&full[j % S], (j / S) & 1, &fresh);
                }
            }
        }
    } else if (warp >= kMxMmaWarp) {
        // ------------------------------------------------------------ MMA issuers (one thread each)
        const int w = warp - kMxMmaWarp;
        if (lane == 0) {
            const uint32_t tmem = tmem_s;
            const uint32_t t_sfa = tmem + 384 + 8 * w, t_sfb = t_sfa + 4;
            const uint32_t w3off = 8 * GM;
            int i = 0;   // CTA-local unit index
            bool alive = true;
            for (int j = 0; j < n_parts && alive; ++j) {
                bool up;
                int item, ua, ub;
                part_of(j, up, item, ua, ub);
                const int gs = up ? item / RT : item / NT;
                const int slot = act_slot[gs_a[gs]];
                const uint32_t idesc0 = mx_idesc(8 * gs_n[gs], 0), idesc1 = mx_idesc(8 * gs_n[gs], 2);
                const int db = j & 1;
                if (j >= 2 && !mbar_poll(&acce[db], ((j >> 1) - 1) & 1, abort_flag, a.timeout_ns)) {
                    latch_error(a.err, ERR_ETIMEOUT, j, up ? KID_UP : KID_DOWN);
                    break;
                }
                mx_fence_after();
                bool started0 = false, started1 = false;
                for (int gu = ua; gu < ub; ++gu, ++i) {
                    if (i % kMxIssuers != w) continue;
                    const int s = i % S;
                    if (!mbar_poll(&full[s], (i / S) & 1, abort_flag, a.timeout_ns)) {
                        latch_error(a.err, ERR_ETIMEOUT, i, up ? KID_UP : KID_DOWN);
                        alive = false;
                        break;
                    }
                    mx_fence_after();
                    if (slot >= 0) {
                        const int mat = up ? (gu - item * upi) / KU : 0;
                        const uint32_t dcol = tmem + (db * kMxIssuers + w) * acc_cols + mat * w3off;
                        const uint32_t sa = ring_base + static_cast<uint32_t>(s) * SB;
                        mx_cp_atom(t_sfa, sa + kUnitCodeBytes);
                        mx_cp_atom(t_sfb, sa + off_sfb);
                        const bool started = mat ? started1 : started0;
                        mx_mma(dcol, mx_desc(sa, 128, 512), mx_desc(sa + kMxOffB, 128, 512), idesc0, t_sfa, t_sfb,
                               started ? 1u : 0u);
                        mx_mma(dcol, mx_desc(sa + 256, 128, 512), mx_desc(sa + kMxOffB + 256, 128, 512), idesc1,
                               t_sfa | (2u << 30), t_sfb | (2u << 30), 1u);
                        if (mat) started1 = true; else started0 = true;
                    }
                    mx_commit(&empty[s]);   // the slot is free once these MMAs have read it
                }
                if (alive) mx_commit(&accf[db]);   // this issuer's share of the part is done
            }
            mx_commit(&fin[w]);              // every MMA of this issuer completes before TMEM is released
            volatile int fresh = 0;
            mbar_wait(&fin[w], 0, &fresh);
        }
        __syncwarp();
    }
    else if (warp < kMxEpiWarps) {
        // ------------------------------------------------------------ epilogue (128 threads, row = thread)
        const uint32_t lane_base = tmem_s + (static_cast<uint32_t>(32 * warp) << 16);
        const int row = 32 * warp + lane;
        for (int j = 0; j < n_parts; ++j) {
            bool up;
            int item, ua, ub;
            part_of(j, up, item, ua, ub);
            const int gs = up ? item / RT : item / NT, tile = up ? item - gs * RT : item - gs * NT;
            const int ng = gs_n[gs], p0 = gs_p0[gs], slot = act_slot[gs_a[gs]];
            const int db = j & 1;
            // A wait that gives up does not leave the loop: the four warps take the
            // same named barriers whatever their own waits returned (a warp that
            // left would strand the others); the outputs of a launch that gave
            // up are not used, and later waits return at once.
            int ok = 1;
            if (lane == 0) ok = mbar_poll(&accf[db], (j >> 1) & 1, abort_flag, a.timeout_ns);
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok && lane == 0) latch_error(a.err, ERR_ETIMEOUT, j, up ? KID_UP : KID_DOWN);
            mx_fence_after();
            const int per = up ? upi : dpi, nall = up ? NU : ND;
            const int ibase = item * per;
            // units of w1 (or w2) and of w3 in this part, and the CTA-local index of the part's first unit
            const int m0a = ua, m0b = up ? min(ub, ibase + KU) : ub;
            const int m1a = up ? max(ua, ibase + KU) : ub, m1b = ub;
            const int i0 = up ? ua - u0 : nu + (ua - d0);
            float acc0[kMxGroup], acc1[kMxGroup];
#pragma unroll
            for (int e = 0; e < kMxGroup; ++e) {
                acc0[e] = 0.0f;
                acc1[e] = 0.0f;
            }
            for (int w = 0; w < kMxIssuers; ++w) {   // fixed order: results do not depend on timing
                // issuer w took unit gu iff (i0 + gu - ua) % kMxIssuers == w
                const int f0 = m0a + ((w - (i0 + m0a - ua)) % kMxIssuers + kMxIssuers) % kMxIssuers;
                const int f1 = m1a + ((w - (i0 + m1a - ua)) % kMxIssuers + kMxIssuers) % kMxIssuers;
                const bool t0 = f0 < m0b, t1 = f1 < m1b;
                const uint32_t dw = lane_base + (db * kMxIssuers + w) * acc_cols;
#pragma unroll
                for (int e = 0; e < kMxGroup; ++e) {
                    if (ok && slot >= 0 && e < ng) {
                        if (t0) acc0[e] += mx_ld8_sum(dw + 8 * e);
                        if (t1) acc1[e] += mx_ld8_sum(dw + 8 * GM + 8 * e);
                    }
                }
            }
            mx_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[db]);   // the MMAs may reuse this accumulator
            // the CTAs holding units of this item, in order
            const int bf = mx_cta_of(nall, G, ibase), bl = mx_cta_of(nall, G, ibase + per - 1);
            int nparts = 0;
            for (int bb = bf; bb <= bl; ++bb)
                nparts += mx_range_start(nall, G, bb) < mx_range_start(nall, G, bb + 1);
            if (nparts > 1) {   // split item: store this part, the last part to arrive adds them all
                const int side = (item == (up ? up_first : dn_first)) ? 0 : 1;
                float* pp = a.part + static_cast<size_t>(b) * kMxPartFloats +
                            (up ? side * kMxPartUp : 2 * kMxPartUp + side * kMxPartDown);
#pragma unroll
                for (int e = 0; e < kMxGroup; ++e) {
                    if (e < ng) {
                        pp[e * 128 + row] = acc0[e];
                        if (up) pp[kMxGroup * 128 + e * 128 + row] = acc1[e];
                    }
                }
                mx_named_barrier(1, kMxEpiWarps * 32);
                if (tid == 0) {
                    __threadfence();
                    const unsigned int c = mx_arrive(up ? up_cnt + item : dn_cnt + item);
                    last_s = c == static_cast<unsigned int>(nparts);
                }
                mx_named_barrier(1, kMxEpiWarps * 32);
                if (!last_s) continue;
                __threadfence();
#pragma unroll
                for (int e = 0; e < kMxGroup; ++e) {
                    acc0[e] = 0.0f;
                    acc1[e] = 0.0f;
                }
                for (int bb = bf; bb <= bl; ++bb) {
                    const int st = mx_range_start(nall, G, bb);
                    if (st == mx_range_start(nall, G, bb + 1)) continue;
                    const int sd = (item == st / per) ? 0 : 1;
                    const float* q = a.part + static_cast<size_t>(bb) * kMxPartFloats +
                                     (up ? sd * kMxPartUp : 2 * kMxPartUp + sd * kMxPartDown);
#pragma unroll
                    for (int e = 0; e < kMxGroup; ++e) {
                        if (e < ng) {
                            acc0[e] += __ldcg(q + e * 128 + row);
                            if (up) acc1[e] += __ldcg(q + kMxGroup * 128 + e * 128 + row);
                        }
                    }
                }
            }
            if (up) {
                // h = bf16(silu(a1) * a3) of rows 128 tile + row, then its digit planes (block = warp)
#pragma unroll
                for (int e = 0; e < kMxGroup; ++e) {
                    if (e < ng) {
                        const float a1 = acc0[e], a3 = acc1[e];
                        const float hv = (slot >= 0) ? a1 / (1.0f + expf(-a1)) * a3 : 0.0f;
                        const float hf = __uint_as_float(static_cast<uint32_t>(f32_to_bf16_rne(hv)) << 16);
                        const size_t tt = static_cast<size_t>(p0 + e) * KD + tile;
                        mx_split_block(hf, lane, a.hp + tt * kMxPlaneTile + warp * 128, a.hsf + tt * kMxPlaneScale + warp);
                    }
                }
                mx_named_barrier(1, kMxEpiWarps * 32);
                if (tid == 0) {
                    __threadfence();
                    mx_fence_proxy_global();
                    mx_st_release(a.ready + item, tag);
                    if (slot < 0) latch_error(a.err, ERR_ESLOT, act_e[gs_a[gs]], KID_UP);
                }
            } else {
#pragma unroll
                for (int e = 0; e < kMxGroup; ++e) {
                    if (e < ng) {
                        const int ent = entry_of(p0 + e);
                        if (ent >= 0)
                            a.obuf[static_cast<size_t>(ent) * H + tile * 128 + row] = (slot >= 0) ? acc0[e] : 0.0f;
                    }
                }
                if (slot < 0 && tid == 0) latch_error(a.err, ERR_ESLOT, act_e[gs_a[gs]], KID_DOWN);
                if (a.y != nullptr) {
                    // the CTA finishing the last item of this 128-row tile combines it for every token
                    mx_named_barrier(1, kMxEpiWarps * 32);
                    if (tid == 0) {
                        __threadfence();
                        last_s = mx_arrive(tile_cnt + tile) == static_cast<unsigned int>(n_gs);
                    }
                    mx_named_barrier(1, kMxEpiWarps * 32);
                    if (last_s) {
                        __threadfence();
                        const int n0 = tile * 128 + row;
                        for (int t = 0; t < a.T; ++t) {
                            float yv = 0.0f;
                            for (int jj = 0; jj < k; ++jj) {
                                const float wj = routed ? r_w[t * k + jj] : __ldg(a.weights + t * k + jj);
                                yv = fmaf(wj, __ldcg(a.obuf + static_cast<size_t>(t * k + jj) * H + n0), yv);
                            }
                            a.y[static_cast<size_t>(t) * H + n0] = yv;
                            if (a.x_out) {
                                const float xv = bf16_to_f32(a.x[static_cast<size_t>(t) * H + n0]);
                                a.x_out[static_cast<size_t>(t) * H + n0] = f32_to_bf16_rne(xv + yv);
                            }
                        }
                    }
                }
            }
        }
    }

    // ------------------------------------------------------------ exit
    mx_fence_before();
    __syncthreads();
    mx_fence_after();
    if (warp == kMxMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_s), "r"(kMxTmemCols));
    if (tid == 0) {   // the last CTA out advances the launch sequence number
        __threadfence();
        if (atomicAdd(a.seq + 1, 1u) == static_cast<unsigned int>(G - 1)) {
            *reinterpret_cast<volatile unsigned int*>(a.seq + 1) = 0u;
            __threadfence();
            atomicAdd(a.seq, 1u);
        }
    }
}

// ------------------------------------------------------------------ host side
// Plan of one launch; ok = 0 when the shape or the batch does not fit.
// Shared memory: barriers, routing tables, then the ring of S slots.
inline MxPlan make_mx_plan(const SlotLayout& L, int T, int k, int E, bool routed, int smem_limit) {
    MxPlan p{};
    const int n_ent = T * k;
    if (T < 1 || k < 1 || E < 1 || L.H % 128 || L.I % 128) return p;
    if (routed && (n_ent > kMxRouteMax || E > kMxRouteExperts)) return p;
    p.max_ent = n_ent;
    p.max_act = min(E, n_ent);
    p.max_gs = min(n_ent, p.max_act + n_ent / kMxGroup);   // groups of <= kMxGroup entries
    p.max_up_items = p.max_gs * L.RT;
    p.max_dn_items = p.max_gs * L.NT;
    p.gmax = T == 1 ? 1 : kMxGroup;
    p.slot_bytes = kUnitBytes + p.gmax * (kMxPlaneTile + kMxPlaneScale);
    const int tab_ints = 4 * p.max_act + 3 * p.max_gs + E + max(4 * kMxRouteMax, E + 1);
    p.off_tab = 1024;                                           // barriers first
    p.off_ring = (p.off_tab + 4 * tab_ints + 1023) / 1024 * 1024;
    // 1024: alignment of the dynamic base; 512: the last slot's B scale copy reads 512 bytes
    int slots = (smem_limit - 1024 - 512 - p.off_ring) / p.slot_bytes;
    slots = min(slots, kMxMaxSlots) / kMxSlotQuantum * kMxSlotQuantum;
    if (slots < kMxSlotQuantum) return p;
    p.slots = slots;
    p.smem_bytes = p.off_ring + slots * p.slot_bytes + 512 + 1024;
    p.ok = 1;
    return p;
}

// Workspace of the kernel for batches up to T tokens of top-k (bytes of each buffer).
struct MxSizes {
    size_t xp, xsf, hp, hsf, part, cnt, ready;
};
inline MxSizes mx_sizes(const SlotLayout& L, int T, int k, int E, int grid) {
    const MxPlan p = make_mx_plan(L, T, k, E, false, 1 << 30);
    MxSizes z;
    z.xp = static_cast<size_t>(T) * L.KU * kMxPlaneTile;
    z.xsf = static_cast<size_t>(T) * L.KU * kMxPlaneScale;
    z.hp = static_cast<size_t>(T) * k * L.KD * kMxPlaneTile;
    z.hsf = static_cast<size_t>(T) * k * L.KD * kMxPlaneScale;
    z.part = static_cast<size_t>(grid) * kMxPartFloats * sizeof(float);
    z.cnt = (1 + static_cast<size_t>(p.max_up_items) + p.max_dn_items + L.NT) * sizeof(unsigned int);   // one bank
    z.ready = static_cast<size_t>(p.max_up_items) * sizeof(unsigned int);
    return z;
}

}  // namespace moe
