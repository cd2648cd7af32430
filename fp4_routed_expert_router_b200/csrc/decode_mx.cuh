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
// plane's unit, so after 8 planes it is at most 2^(E0-16) < max|v| * 2^-16,
// and every element within 2^8 of the block maximum is represented exactly
// (bf16 has 8 significant bits).  The planes are the N columns of the MMA
// (8 per entry); the epilogue adds them in fp32.  Power-of-two rescalings of
// a row rescale its planes exactly (the digits depend on v / 2^E0 only).
//
// Work.  A unit is one 128-row x 128-K tile of one weight matrix (8,704
// bytes: codes and block scales, slot_layout.cuh) plus the B tile of its
// token group (<= 2 entries x 8 planes x 128 K, and their scale bytes; one
// entry per group for a single token).  An up item is (token group, 128 rows
// of w1 and w3) over all of H; a down item (group, 128 rows of w2) over all
// of I.  The up units of all items form one sequence split contiguously over
// the CTAs (one per SM); an up item cut by a range boundary is finished by
// whichever of its CTAs completes last, which adds the fp32 partials in CTA
// order (results do not depend on timing).  Down items are dealt out whole,
// so no down partial crosses CTAs.  Inside a CTA:
//   warps 10-15         producers, one lane per ring slot (S / 6 lanes each):
//                       bulk copies of unit i (A + scales from the arena, B +
//                       B scales from the plane buffers) into slot i % S.  A
//                       lane copies the weights as soon as its slot is free
//                       and the B tile once it exists, so weights stream
//                       ahead of the activations they meet;
//   warps 4-9, lane 0   MMA issuers: slot s belongs to issuer s % 6 --
//                       tcgen05.cp of both scale atoms into its own TMEM
//                       columns, two K = 64 MMAs into its own double-buffered
//                       accumulator, tcgen05.commit frees the slot.  One
//                       thread's tcgen05 stream stalls at every commit
//                       (measured on B200: one issuer 307 ns per unit, two
//                       154, four 77), so six issuers take turns and keep the
//                       pipe ahead of HBM;
//   warps 0-3           epilogue (TMEM lane quadrant = warp): planes and the
//                       issuers' accumulators summed (fixed order), then a
//                       partial, or the item's finish: SwiGLU, bf16 h and its
//                       digit planes (up), per-entry o and the combine of a
//                       128-row output tile by the CTA that completes its
//                       last item (down);
//   all warps           prologue: routing, and a share of the x planes; the
//                       mbarrier and TMEM set-up runs in warp 4 meanwhile.
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
constexpr int kMxProdWarp = kMxMmaWarp + kMxIssuers;   // warps 10 .. 15: S / 6 producer lanes each
constexpr int kMxProdWarps = kMxWarps - kMxProdWarp;
// Ring slots come in multiples of this: slot s is always filled by its own
// producer lane and drained by issuer s % 6, so each thread sees the uses of
// its slots in order and every mbarrier parity wait is unambiguous.
constexpr int kMxSlotQuantum = kMxIssuers;
static_assert(kMxProdWarps == kMxIssuers, "one producer lane per slot: S / 6 lanes in each of 6 warps");
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
constexpr int kMxPartUp = 2 * kMxGroup * 128;     // floats of one up side (w1 then w3)
constexpr int kMxPartDown = kMxGroup * 128;       // floats of one down side
constexpr int kMxPartFloats = 2 * kMxPartUp + 2 * kMxPartDown;  // split-item partials of one CTA: 2 up, 2 down sides
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

// 8 or 16 consecutive fp32 TMEM columns of this thread's lane into r[0 .. n), no wait.
__device__ __forceinline__ void mx_ld_issue16(uint32_t taddr, int n, uint32_t (&r)[16]) {
    if (n == 8) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
    }
}

// n (8, 16 or 32) consecutive fp32 TMEM columns of this thread's lane into r[0 .. n).
__device__ __forceinline__ void mx_ld_cols(uint32_t taddr, int n, uint32_t (&r)[32]) {
    if (n == 8) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                     : "r"(taddr));
    } else if (n == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(taddr));
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
              "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
              "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
              "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
            : "r"(taddr));
    }
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
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

// x * 2^e, exact whenever the result is representable (two multiplies by
// normal powers of two; -252 <= e <= 254).
__device__ __forceinline__ float mx_mul_pow2(float x, int e) {
    const int e1 = e / 2, e2 = e - e1;
    return (x * __uint_as_float(static_cast<uint32_t>(e1 + 127) << 23)) * __uint_as_float(static_cast<uint32_t>(e2 + 127) << 23);
}

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
    // this lane's digit of every plane, one nibble each (plane p in bits 4p .. 4p+3)
    float r = v;
    uint32_t x = 0u;
#pragma unroll
    for (int p = 0; p < kMxPlanes; ++p) {
        const int s = e0 - 2 * p;               // plane scale 2^s
        if (live && s >= -127) {
            const float d = rintf(2.0f * mx_mul_pow2(r, -s)) * 0.5f;   // nearest half: |d| <= 2
            const float ad = fabsf(d);
            x |= (static_cast<uint32_t>(2.0f * ad) | (d < 0.0f ? 8u : 0u)) << (4 * p);
            r -= mx_mul_pow2(d, s);             // exact: |r| shrinks below 2^(s-2)
        }
    }
    // Transpose the 8 x 8 nibbles of each group of 8 lanes (three butterfly
    // exchanges): lane 8j + p then holds plane p's digits of elements
    // 8j .. 8j+7, element 8j + i in nibble i -- one 32-bit word per lane, stored
    // by every lane at once.
#pragma unroll
    for (int bs = 4; bs >= 1; bs >>= 1) {
        const uint32_t m = bs == 4 ? 0x0000FFFFu : (bs == 2 ? 0x00FF00FFu : 0x0F0F0F0Fu);
        const uint32_t y = __shfl_xor_sync(0xFFFFFFFFu, x, bs);
        x = (lane & bs) ? (((y & ~m) >> (4 * bs)) | (x & ~m)) : ((x & m) | ((y & m) << (4 * bs)));
    }
    *reinterpret_cast<uint32_t*>(pc + 16 * (lane & 7) + 4 * (lane >> 3)) = x;
    if (lane < kMxPlanes) {
        const int s = e0 - 2 * lane;
        sf[16 * lane] = static_cast<uint8_t>((live && s >= -127) ? s + 127 : ((!live && lane == 0 && mb != 0u) ? 255 : 0));
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

    // Set-up runs beside the first loads: lane 0 of the TMEM warp reads the
    // launch sequence number and initialises the barriers, the warp allocates
    // TMEM, a producer warp reads the slot table row, and from the first
    // instruction the other warps route (below) and make x planes.
    if (warp == kMxMmaWarp) {
        if (lane == 0) {
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
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_s)),
                     "r"(kMxTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (warp == kMxProdWarp)   // this layer's slot table row
        for (int e = lane; e < E; e += 32) slot_s[e] = __ldg(a.slot_table + static_cast<size_t>(a.layer) * E + e);

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
    // x planes, routing and set-up done: count this CTA's planes on the launch's
    // x counter (the copies of x planes wait for every CTA), clear the counter
    // bank of the next launch
    auto after_first_sync = [&]() {
        if (tid == kMxThreads - 32) {   // not warp 0, which groups the entries next
            __threadfence();
            mx_fence_proxy_global();
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;"
                         ::"l"(a.cnt + static_cast<size_t>(tag_s & 1u) * a.cnt_cap) : "memory");
        }
        unsigned int* other = a.cnt + static_cast<size_t>((tag_s + 1u) & 1u) * a.cnt_cap;
        for (int i = b * kMxThreads + tid; i < a.cnt_cap; i += G * kMxThreads) other[i] = 0u;
    };
    if (routed) {
        for (int t = warp; t < a.T; t += kMxWarps)
            route_one<kMxRouteExperts / 32>(a.logits + static_cast<size_t>(t) * E, a.keep, E, k, t, lane,
                                           r_ids + t * k, r_w + t * k, a.err);
        __syncthreads();
        after_first_sync();
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
        after_first_sync();
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
    // Two segments: every up unit of the batch, split contiguously over all
    // CTAs, then every down item, dealt whole.  (Interleaving the two -- the
    // down part of some groups after the up part of later ones -- measured
    // 3.4x slower at batch 1 on B200: accumulators and the epilogue run in
    // order, so a down part waiting for another CTA's h holds up every part
    // queued behind it.)
    const int n_gs = n_gs_s;
    const unsigned int tag = tag_s;
    const int upi = 2 * KU, dpi = KD;                       // units per up / down item
    const int n_seg = 2;
    unsigned int* x_cnt = a.cnt + static_cast<size_t>(tag & 1u) * a.cnt_cap;   // this launch's bank
    unsigned int* up_cnt = x_cnt + 1;
    unsigned int* dn_cnt = up_cnt + p.max_up_items;
    unsigned int* tile_cnt = dn_cnt + p.max_dn_items;
    // grouped position -> entry t*k+j; -1 for an entry outside [0, T*k)
    auto entry_of = [&](int pos) -> int {
        const int ent = routed ? r_perm[pos] : __ldg(a.perm + pos);
        return (ent >= 0 && ent < n_ent) ? ent : -1;
    };
    // segment sg (0: up, 1: down): its unit space [base, base + n) and this
    // CTA's range [ua, ub) in it (global unit indices)
    auto segment = [&](int sg, bool& up, int& c, int& base, int& n, int& ua, int& ub) {
        up = sg == 0;
        c = 0;
        base = 0;
        n = n_gs * (up ? RT * upi : NT * dpi);
        if (up) {   // up units split evenly: an item may be cut between CTAs
            ua = base + mx_range_start(n, G, b);
            ub = base + mx_range_start(n, G, b + 1);
        } else {    // whole down items: no partial sums; their weights stream while h is made
            const int items = n / dpi;
            ua = base + mx_range_start(items, G, b) * dpi;
            ub = base + mx_range_start(items, G, b + 1) * dpi;
        }
    };
    const uint32_t ring_base = smem_u32(ring);

    if (warp >= kMxProdWarp) {
        // ------------------------------------------------------------ producers
        // Producer p (lane p % (S/6) of warp 10 + p / (S/6)) owns ring slot p and
        // the CTA's units p, p + S, ... (unit i goes to slot i % S).  It never
        // blocks on one unit (lanes of a warp run independent producers): the weights of its units are copied as far ahead
        // as its slots allow (they depend on the routing only), and the B
        // operand of its oldest unit without one as soon as it is ready -- the
        // x planes once every CTA has stored its share, the h planes once their
        // up item is done -- so during the hand-off from the up to the down
        // GEMM the ring fills with down weights.  expect_tx without an arrive
        // keeps a unit's phase open until its B copies are issued too.
        const int lanes = S / kMxProdWarps;   // producer lanes per warp: one producer per slot
        if (lane < lanes) {
            const int pw = (warp - kMxProdWarp) * lanes + lane;   // this producer's slot
            const int kMxProducers = S;
            const uint64_t pol = policy_evict_first();
            // the CTA's units as segments: local index i -> global unit gu
            int seg_first[3], seg_ua[2];
            bool seg_up[2];
            int n_units = 0;
            for (int sg = 0; sg < n_seg; ++sg) {
                int c, base, n, ua, ub;
                bool up;
                segment(sg, up, c, base, n, ua, ub);
                seg_first[sg] = n_units;
                seg_ua[sg] = ua;
                seg_up[sg] = up;
                n_units += ub - ua;
            }
            seg_first[n_seg] = n_units;
            auto unit = [&](int i, bool& up, int& gs, int& tile, int& mat, int& ku) {
                int sg = 0;
                while (i >= seg_first[sg + 1]) ++sg;
                up = seg_up[sg];
                const int gu = seg_ua[sg] + (i - seg_first[sg]);
                const int item = up ? gu / upi : gu / dpi, v = up ? gu - item * upi : gu - item * dpi;
                gs = up ? item / RT : item / NT;
                tile = up ? item - gs * RT : item - gs * NT;
                mat = up ? v / KU : 0;
                ku = up ? v - mat * KU : v;
            };
            const int nm = n_units > pw ? (n_units - pw + kMxProducers - 1) / kMxProducers : 0;   // my units
            const int ahead = S / kMxProducers;                                                // my slots
            int mA = 0, mB = 0;            // my next unit for the weights / for the B operand
            bool x_ok = false;
            int ready_item = -1;
            uint64_t t_idle = global_timer_ns();
            while (mB < nm) {
                bool progress = false;
                while (mA < nm && mA < mB + ahead) {   // weights, as far ahead as my slots allow
                    const int i = pw + mA * kMxProducers, s = i % S;
                    if (i >= S && !mbar_test(&empty[s], ((i / S) - 1) & 1)) break;
                    bool up;
                    int gs, tile, mat, ku;
                    unit(i, up, gs, tile, mat, ku);
                    const int slot = act_slot[gs_a[gs]];
                    if (slot >= 0) {   // (an expert that is not resident gets no copies; the epilogue writes zeros)
                        const size_t uoff = up ? up_unit_offset(L, mat, tile, ku) : down_unit_offset(L, tile, ku);
                        mbar_expect_tx(&full[s], static_cast<uint32_t>(kUnitBytes));
                        bulk_g2s(ring + static_cast<size_t>(s) * SB, a.arena + static_cast<size_t>(slot) * a.slot_bytes + uoff,
                                 kUnitBytes, &full[s], pol);
                        reinterpret_cast<volatile int*>(last_issue)[s] = i;
                    }
                    ++mA;
                    progress = true;
                }
                if (mB < mA) {                         // the B operand of my oldest unit without one
                    const int i = pw + mB * kMxProducers, s = i % S;
                    bool up;
                    int gs, tile, mat, ku;
                    unit(i, up, gs, tile, mat, ku);
                    const int slot = act_slot[gs_a[gs]];
                    bool ready = slot < 0;
                    if (!ready && up) {
                        if (!x_ok) x_ok = mx_ld_acquire(x_cnt) >= static_cast<unsigned int>(G);
                        ready = x_ok;
                    } else if (!ready) {
                        if (ready_item != gs * RT + ku && mx_ld_acquire(a.ready + gs * RT + ku) == tag)
                            ready_item = gs * RT + ku;
                        ready = ready_item == gs * RT + ku;
                    }
                    if (ready) {
                        if (slot < 0) {
                            mbar_arrive(&full[s]);
                        } else {
                            const int ng = gs_n[gs], p0 = gs_p0[gs];
                            uint8_t* dst = ring + static_cast<size_t>(s) * SB;
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
                        ++mB;
                        progress = true;
                    }
                }
                if (progress) {
                    t_idle = global_timer_ns();
                } else {
                    if (*abort_flag) break;
                    if (global_timer_ns() - t_idle > a.timeout_ns) {
                        latch_error(a.err, ERR_ETIMEOUT, 200 + pw, KID_UP);
                        *abort_flag = 1;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            if (mB < nm) {   // gave up: the units whose B was never issued complete once their weights land
                for (int m = mB; m < mA; ++m) mbar_arrive(&full[(pw + m * kMxProducers) % S]);
                volatile int fresh = 0;   // then every copy of this warp in flight lands before the CTA may exit
                for (int m = 0; m < mA; ++m) {
                    const int i = pw + m * kMxProducers;
                    // a later unit in the same slot was only copied after unit i had been consumed
                    if (reinterpret_cast<volatile int*>(last_issue)[i % S] != i) continue;
                    fresh = 0;
                    mbar_wait(&full[i % S], (i / S) & 1, &fresh);
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
            int j = 0;   // part index
            bool alive = true;
            for (int sg = 0; sg < n_seg && alive; ++sg) {
                bool up;
                int c, base, n, ua, ub;
                segment(sg, up, c, base, n, ua, ub);
                if (ua == ub) continue;
                const int per = up ? upi : dpi;
                for (int item = ua / per; item <= (ub - 1) / per && alive; ++item, ++j) {
                    const int pa = max(ua, item * per), pb = min(ub, (item + 1) * per);
                    const int gs = up ? item / RT : item / NT;
                    const int slot = act_slot[gs_a[gs]];
                    const uint32_t idesc0 = mx_idesc(8 * gs_n[gs], 0), idesc1 = mx_idesc(8 * gs_n[gs], 2);
                    const int db = j & 1;
                    if (j >= 2 && !mbar_poll(&acce[db], ((j >> 1) - 1) & 1, abort_flag, a.timeout_ns)) {
                        latch_error(a.err, ERR_ETIMEOUT, j, up ? KID_UP : KID_DOWN);
                        alive = false;
                        break;
                    }
                    mx_fence_after();
                    bool started0 = false, started1 = false;
                    for (int gu = pa; gu < pb; ++gu, ++i) {
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
        int i = 0;   // CTA-local index of the part's first unit
        int j = 0;   // part index
        for (int sg = 0; sg < n_seg; ++sg) {
            bool up;
            int c, base, n, ua, ub;
            segment(sg, up, c, base, n, ua, ub);
            if (ua == ub) continue;
            const int per = up ? upi : dpi;
            const int first_item = ua / per;
            for (int item = first_item; item <= (ub - 1) / per; ++item, ++j) {
                const int pa = max(ua, item * per), pb = min(ub, (item + 1) * per);
                const int i0 = i;
                i += pb - pa;
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
                const int ibase = item * per;
                // units of w1 (or w2) and of w3 in this part
                const int m0a = pa, m0b = up ? min(pb, ibase + KU) : pb;
                const int m1a = up ? max(pa, ibase + KU) : pb, m1b = pb;
                float acc0[kMxGroup], acc1[kMxGroup];
#pragma unroll
                for (int e = 0; e < kMxGroup; ++e) {
                    acc0[e] = 0.0f;
                    acc1[e] = 0.0f;
                }
                const int ncols = up ? 16 * GM : 8 * GM;   // this part's columns of one issuer
                // issuer w took unit gu iff (i0 + gu - pa) % kMxIssuers == w; did it reach w1 (w2) / w3 units?
                auto touched = [&](int w, bool& t0, bool& t1) {
                    const int f0 = m0a + ((w - (i0 + m0a - pa)) % kMxIssuers + kMxIssuers) % kMxIssuers;
                    const int f1 = m1a + ((w - (i0 + m1a - pa)) % kMxIssuers + kMxIssuers) % kMxIssuers;
                    t0 = f0 < m0b;
                    t1 = f1 < m1b;
                };
                // sums of one issuer's columns: w1 (w2) planes at 8 e, w3 planes at 8 GM + 8 e
                auto add = [&](const uint32_t* r, bool t0, bool t1) {
#pragma unroll
                    for (int e = 0; e < kMxGroup; ++e) {
                        if (e < ng) {
                            float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                s0 += __uint_as_float(r[8 * e + q]);
                                s1 += __uint_as_float(GM == 1 ? r[(8 + 8 * e + q) & 31] : r[(16 + 8 * e + q) & 31]);
                            }
                            if (t0) acc0[e] += s0;
                            if (t1) acc1[e] += s1;
                        }
                    }
                };
                if (ok && slot >= 0) {
                    if (ncols <= 16) {   // two issuers per TMEM round trip, fixed order
                        for (int w = 0; w < kMxIssuers; w += 2) {
                            bool ta0, ta1, tb0, tb1;
                            touched(w, ta0, ta1);
                            touched(w + 1, tb0, tb1);
                            uint32_t ra[16], rb[16];
                            if (ta0 || ta1) mx_ld_issue16(lane_base + (db * kMxIssuers + w) * acc_cols, ncols, ra);
                            if (tb0 || tb1) mx_ld_issue16(lane_base + (db * kMxIssuers + w + 1) * acc_cols, ncols, rb);
                            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                            if (ta0 || ta1) add(ra, ta0, ta1);
                            if (tb0 || tb1) add(rb, tb0, tb1);
                        }
                    } else {
                        for (int w = 0; w < kMxIssuers; ++w) {
                            bool t0, t1;
                            touched(w, t0, t1);
                            if (!(t0 || t1)) continue;
                            uint32_t r[32];
                            mx_ld_cols(lane_base + (db * kMxIssuers + w) * acc_cols, ncols, r);
                            add(r, t0, t1);
                        }
                    }
                }
                mx_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[db]);   // the MMAs may reuse this accumulator
                // the CTAs holding units of this up item (relative to the chunk's unit space), in order;
                // a down item is never cut
                const int bf = up ? mx_cta_of(n, G, ibase - base) : b;
                const int bl = up ? mx_cta_of(n, G, ibase - base + per - 1) : b;
                int nparts = up ? 0 : 1;
                for (int bb = bf; up && bb <= bl; ++bb) nparts += mx_range_start(n, G, bb) < mx_range_start(n, G, bb + 1);
                if (nparts > 1) {   // split item: store this part, the last part to arrive adds them all
                    const int side = (item == first_item) ? 0 : 1;
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
                    if (tid == 0) {   // the acquire-release add orders the CTA's stores (named barrier) before it
                        const unsigned int cnt = mx_arrive(up ? up_cnt + item : dn_cnt + item);
                        last_s = cnt == static_cast<unsigned int>(nparts);
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
                        const int st = mx_range_start(n, G, bb);
                        if (st == mx_range_start(n, G, bb + 1)) continue;
                        const int sd = (item == (base + st) / per) ? 0 : 1;
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
                            mx_split_block(hf, lane, a.hp + tt * kMxPlaneTile + warp * 128,
                                           a.hsf + tt * kMxPlaneScale + warp);
                        }
                    }
                    mx_named_barrier(1, kMxEpiWarps * 32);
                    if (tid == 0) {   // the release store orders the CTA's stores (named barrier) before it
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
                        if (tid == 0)
                            last_s = mx_arrive(tile_cnt + tile) == static_cast<unsigned int>(n_gs);
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
