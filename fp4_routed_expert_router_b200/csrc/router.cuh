// router.cuh -- top-k routing and token->expert grouping in one launch.
//
// Router: 6 of 384 routed experts per token per layer (10100.com article
// 151357339, section "moe专家的容量瓶颈"); the function itself is not given
// on the pages.  It is read as softmax over fp32 logits, top-k under the
// total order (larger logit first, lower expert index on ties, -0 == +0),
// renormalised over the k chosen: w_j = exp(l_j - l_max) / sum_i exp(l_i - l_max).
// Experts outside the layer's keep mask are never chosen (section "方案二").
//
// Grouping: in prefill one read of an expert's weights serves every token
// routed to it (ai-shiz.ru "DeepSeek-V4.1-Flash дома", trick 4).  The
// entries t*k+j are grouped by expert with a stable counting sort: per-warp
// histograms with warp-aggregated updates (match_any), an exclusive scan,
// and a second, ordered pass that places each entry.
//
// Launch: one kernel whatever T is.  Up to 32 entries, one warp routes and
// sorts (route_small_kernel).  Beyond that a grid of co-resident CTAs
// (cooperative launch, at most one per SM) routes contiguous token ranges and
// groups all T*k entries together in three phases split by two bounded grid
// barriers (route_grid_kernel); no CTA ever walks all entries alone.
#pragma once
#include "common.cuh"
#include "tma.cuh"

namespace moe {

constexpr int kRouteWarps = 8;

// Order-preserving map of a float (after -0 -> +0) to uint32; 0 is below
// every real value and marks "not selectable".
__device__ __forceinline__ uint32_t orderable(float v) {
    uint32_t b = __float_as_uint(v + 0.0f);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_orderable(uint32_t u) {
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

struct RouteArgs {
    const float* logits;
    const uint8_t* keep;
    int T, E, k;
    int32_t* ids;
    float* weights;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm;
    unsigned int* ticket;   // [4 + grid * E]: two grid barriers, an exit count and a failure flag (zero
                            // between launches), then the per-CTA expert counts of route_grid_kernel
    int* err;
    unsigned long long timeout_ns;   // limit of each grid-barrier wait (route_grid_kernel)
};

// Top-k of one token's logits by one warp: writes the k chosen experts (in
// the total order) to ids_out[0..k) and their renormalised weights to
// w_out[0..k).  NaN logits, or fewer than k selectable experts, latch EINVAL.
template <int NI>   // logits held per lane: E <= 32 * NI
__device__ __forceinline__ void route_one(const float* l, const uint8_t* keep, int E, int k, int t, int lane,
                                          int32_t* ids_out, float* w_out, int* err) {
    uint32_t key[NI];
    bool nan = false;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        int e = lane + 32 * i;
        key[i] = 0;
        if (e < E) {
            float v = __ldg(l + e);
            nan |= (v != v);
            bool ok = (keep == nullptr) || (__ldg(keep + e) != 0);
            key[i] = ok ? orderable(v) : 0u;
        }
    }
    if (__any_sync(0xFFFFFFFFu, nan)) {
        if (lane == 0) latch_error(err, ERR_EINVAL, t, KID_ROUTE);
    }
    uint32_t removed = 0;
    int my_id = 0;
    float my_val = 0.f;
    bool short_of_experts = false;
    for (int r = 0; r < k; ++r) {
        uint32_t best = 0;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            uint32_t kk = (removed >> i) & 1u ? 0u : key[i];
            if (kk > best) { best = kk; bi = i; }
        }
        uint32_t wmax = __reduce_max_sync(0xFFFFFFFFu, best);
        uint32_t cand = (best == wmax) ? static_cast<uint32_t>(lane + 32 * bi) : 0xFFFFFFFFu;
        uint32_t win = __reduce_min_sync(0xFFFFFFFFu, cand);
        if (wmax == 0u) { short_of_experts = true; win = 0; }
        if ((win & 31u) == static_cast<uint32_t>(lane)) removed |= 1u << (win >> 5);
        if (lane == r) { my_id = static_cast<int>(win); my_val = from_orderable(wmax); }
    }
    if (short_of_experts) {
        if (lane == 0) latch_error(err, ERR_EINVAL, t, KID_ROUTE);
    }
    float lmax = __shfl_sync(0xFFFFFFFFu, my_val, 0);
    float p = (lane < k) ? expf(my_val - lmax) : 0.0f;
    float s = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if (lane < k) {
        ids_out[lane] = my_id;
        w_out[lane] = p / s;
    }
}

template <int NI>
__device__ __forceinline__ void route_token(const RouteArgs& a, int t, int lane) {
    route_one<NI>(a.logits + static_cast<size_t>(t) * a.E, a.keep, a.E, a.k, t, lane,
                  a.ids + static_cast<size_t>(t) * a.k, a.weights + static_cast<size_t>(t) * a.k, a.err);
}

// Stable grouping of all T*k entries by one CTA of kRouteWarps warps.
// smem: int hist[kRouteWarps][E].
__device__ void group_entries(const RouteArgs& a, int* hist) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int NE = a.T * a.k, E = a.E;
    for (int i = threadIdx.x; i < kRouteWarps * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int seg = (NE + kRouteWarps - 1) / kRouteWarps;
    const int lo = min(NE, warp * seg), hi = min(NE, lo + seg);
    int* h = hist + warp * E;
    // pass 1: per-warp histogram, one update per distinct expert of a batch
    for (int b = lo; b < hi; b += 32) {
        int i = b + lane;
        int e = (i < hi) ? ld_cg(a.ids + i) : -1;
        // id -1 marks an empty entry (left out silently); any other id outside [0, E) is an error
        if (e >= E || e < -1) { latch_error(a.err, ERR_EINVAL, i, KID_ROUTE); e = -1; }
        uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
        if (e >= 0 && lane == __ffs(peers) - 1) h[e] += __popc(peers);
    }
    __syncthreads();
    // exclusive scan of counts over experts (warp 0), then per-warp bases
    if (warp == 0) {
        const int per = (E + 31) / 32;
        int local = 0;
        for (int q = 0; q < per; ++q) {
            int e = lane * per + q;
            if (e < E) for (int w = 0; w < kRouteWarps; ++w) local += hist[w * E + e];
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int q = 0; q < per; ++q) {
            int e = lane * per + q;
            if (e < E) {
                int c = 0;
                a.offsets[e] = run;
                for (int w = 0; w < kRouteWarps; ++w) {
                    int v = hist[w * E + e];
                    hist[w * E + e] = run + c;
                    c += v;
                }
                a.counts[e] = c;
                run += c;
            }
        }
        if (lane == 31) a.offsets[E] = run;
    }
    __syncthreads();
    // pass 2: place entries in order
    for (int b = lo; b < hi; b += 32) {
        int i = b + lane;
        int e = (i < hi) ? ld_cg(a.ids + i) : -1;
        if (e >= E) e = -1;
        uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
        int base = (e >= 0) ? h[e] : 0;
        __syncwarp();
        if (e >= 0) {
            a.perm[base + __popc(peers & lanemask_lt())] = i;
            if (lane == __ffs(peers) - 1) h[e] = base + __popc(peers);
        }
        __syncwarp();
    }
}

// Grouping alone: the a.T given expert ids (a.k = 1) grouped by expert, as
// the route kernels group their selections (the expert-parallel owner side).
__global__ void __launch_bounds__(kRouteWarps * 32) group_kernel(RouteArgs a) {
    extern __shared__ int smem_hist[];
    pdl_wait();
    group_entries(a, smem_hist);
    pdl_trigger();
}

// Grid barrier over gridDim.x co-resident CTAs, called by all threads of the
// CTA: every thread's earlier global writes are published before thread 0
// arrives (release), and none of the CTA reads data of this phase before
// thread 0 has seen all arrivals (acquire).  Bounded: gives up after
// timeout_ns and returns false (the same answer in every thread).
__device__ __forceinline__ bool route_grid_sync(unsigned int* bar, unsigned long long timeout_ns, int* ok_s) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(bar) : "memory");
        const uint64_t t0 = global_timer_ns();
        int ok = 1;
        for (;;) {
            unsigned int v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
            if (v >= gridDim.x) break;
            if (global_timer_ns() - t0 > timeout_ns) { ok = 0; break; }
            __nanosleep(64);
        }
        *ok_s = ok;
    }
    __syncthreads();
    return *ok_s != 0;
}

// Route and group T*k entries on a grid of G co-resident CTAs (cooperative
// launch).  CTA c owns the tokens [c*tpc, (c+1)*tpc), so its entries are one
// contiguous range, and the phases are:
//   1. one warp per token routes; the CTA counts its entries per expert in
//      shared memory and publishes the row cnt[c][0..E);
//   2. one warp per expert: the exclusive prefix of cnt[.][e] over the CTAs in
//      CTA order (in place) and the expert's total, counts[e];
//   3. every CTA scans counts into offsets (CTA 0 stores them) and places its
//      own entries in order at offsets[e] + cnt[c][e] + (earlier entries of e
//      in the CTA).
// This is the stable order of group_entries: by expert, then by entry index.
// A barrier wait that gives up latches ETIMEOUT and ends the CTA's work.  The
// last CTA to leave clears the barrier words for the next launch and, if any
// CTA gave up, overwrites the grouping with an empty one (zero counts and
// offsets, perm = identity), so that the kernels after it find a valid
// routing with no work instead of whatever the outputs held before.
// smem: int [2E + 1] (the CTA's counts, then the offsets).
template <int NI>
__global__ void __launch_bounds__(kRouteWarps * 32) route_grid_kernel(RouteArgs a) {
    extern __shared__ int smem_route[];
    __shared__ int ok_s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = a.E, k = a.k, G = gridDim.x, c = blockIdx.x;
    unsigned int* bar = a.ticket;                    // [0], [1] barriers, [2] exits, [3] a CTA gave up
    int* cnt = reinterpret_cast<int*>(a.ticket + 4);  // [G][E]
    int* hist = smem_route;                           // [E]
    int* offs = smem_route + E;                       // [E + 1]
    const int tpc = (a.T + G - 1) / G;
    const int t0 = min(a.T, c * tpc), t1 = min(a.T, t0 + tpc);
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    pdl_wait();
    // phase 1
    for (int t = t0 + warp; t < t1; t += kRouteWarps) route_token<NI>(a, t, lane);
    __syncthreads();
    for (int i = t0 * k + threadIdx.x; i < t1 * k; i += blockDim.x) atomicAdd(&hist[a.ids[i]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[static_cast<size_t>(c) * E + e] = hist[e];
    bool ok = route_grid_sync(bar + 0, a.timeout_ns, &ok_s);
    // phase 2
    if (ok) {
        for (int e = c * kRouteWarps + warp; e < E; e += G * kRouteWarps) {
            int run = 0;
            for (int b = 0; b < G; b += 32) {
                const int cc = b + lane;
                const int v = (cc < G) ? __ldcg(cnt + static_cast<size_t>(cc) * E + e) : 0;
                int incl = v;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += u;
                }
                if (cc < G) cnt[static_cast<size_t>(cc) * E + e] = run + incl - v;
                run += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
            if (lane == 0) a.counts[e] = run;
        }
        ok = route_grid_sync(bar + 1, a.timeout_ns, &ok_s);
    }
    // phase 3
    if (ok) {
        if (warp == 0) {   // exclusive scan of counts over experts, per-lane runs of consecutive experts
            const int per = (E + 31) / 32;
            int local = 0;
            for (int q = 0; q < per; ++q) {
                const int e = lane * per + q;
                if (e < E) local += __ldcg(a.counts + e);
            }
            int incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += u;
            }
            int run = incl - local;
            for (int q = 0; q < per; ++q) {
                const int e = lane * per + q;
                if (e < E) {
                    offs[e] = run;
                    run += __ldcg(a.counts + e);
                }
            }
            if (lane == 31) offs[E] = run;
        }
        __syncthreads();
        if (c == 0)
            for (int e = threadIdx.x; e <= E; e += blockDim.x) a.offsets[e] = offs[e];
        for (int e = threadIdx.x; e < E; e += blockDim.x)
            if (hist[e] > 0) hist[e] = offs[e] + __ldcg(cnt + static_cast<size_t>(c) * E + e);
        __syncthreads();
        if (warp == 0) {
            for (int b = t0 * k; b < t1 * k; b += 32) {
                const int i = b + lane;
                const int e = (i < t1 * k) ? a.ids[i] : -1;
                const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
                const int base = (e >= 0) ? hist[e] : 0;
                __syncwarp();
                if (e >= 0) {
                    a.perm[base + __popc(peers & lanemask_lt())] = i;
                    if (lane == __ffs(peers) - 1) hist[e] = base + __popc(peers);
                }
                __syncwarp();
            }
        }
    } else if (threadIdx.x == 0) {
        latch_error(a.err, ERR_ETIMEOUT, c, KID_ROUTE);
        atomicOr(bar + 3, 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {   // the last CTA out clears the barrier words (no CTA waits on them any more)
        unsigned int prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(bar + 2) : "memory");
        ok_s = 0;
        if (prev == static_cast<unsigned int>(G) - 1) {
            ok_s = (atomicAdd(bar + 3, 0u) != 0u) ? 2 : 1;   // 2: some CTA gave up
            bar[0] = 0;
            bar[1] = 0;
            bar[2] = 0;
            bar[3] = 0;
        }
    }
    __syncthreads();
    if (ok_s == 2) {   // every other CTA has left: replace the grouping by an empty one
        for (int e = threadIdx.x; e <= E; e += blockDim.x) {
            a.offsets[e] = 0;
            if (e < E) a.counts[e] = 0;
        }
        for (int i = threadIdx.x; i < a.T * k; i += blockDim.x) a.perm[i] = i;
    }
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// Small batches (T*k <= 32): one warp routes the tokens, then groups the
// entries with a 32-lane bitonic sort on (expert, entry) keys; per-expert
// offsets come from binary searches in the sorted experts.  No grid-wide
// ticket, fence or CTA barrier on the critical path.
template <int NI>
__global__ void __launch_bounds__(32) route_small_kernel(RouteArgs a) {
    pdl_wait();
    const int lane = threadIdx.x;
    const int n = a.T * a.k;            // <= 32
    uint32_t key = 0xFFFFFFFFu;         // (expert << 5) | entry; empty lanes sort last
    for (int t = 0; t < a.T; ++t) {
        route_token<NI>(a, t, lane);
        // the chosen experts were just written by lanes 0..k-1 of this warp
        __syncwarp();
        const int q = lane - t * a.k;
        if (q >= 0 && q < a.k) {
            const int e = a.ids[static_cast<size_t>(t) * a.k + q];
            key = (static_cast<uint32_t>(e) << 5) | static_cast<uint32_t>(lane);
        }
    }
    // bitonic sort of 32 keys across the warp, ascending
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, key, stride);
            const bool ascending = ((lane & size) == 0);
            const bool lower = ((lane & stride) == 0);
            const uint32_t lo = min(key, other), hi = max(key, other);
            key = (lower == ascending) ? lo : hi;
        }
    }
    pdl_trigger();
    if (lane < n) a.perm[lane] = static_cast<int32_t>(key & 31u);
    const int sorted_e = (lane < n) ? static_cast<int>(key >> 5) : 0x7FFFFFFF;
    // lower_bound(e) = #entries with expert < e, by a branch-free binary search
    // over the sorted experts held one per lane (all lanes shuffle together)
    auto lower_bound = [&](int e) {
        int pos = 0;
#pragma unroll
        for (int step = 16; step > 0; step >>= 1) {
            const int v = __shfl_sync(0xFFFFFFFFu, sorted_e, pos + step - 1);
            if (v < e) pos += step;
        }
        const int v = __shfl_sync(0xFFFFFFFFu, sorted_e, pos & 31);
        return (pos < 32 && v < e) ? pos + 1 : pos;
    };
    for (int base = 0; base <= a.E; base += 32) {
        const int e = base + lane;
        const int lb0 = lower_bound(e), lb1 = lower_bound(e + 1);
        if (e < a.E) {
            a.offsets[e] = lb0;
            a.counts[e] = lb1 - lb0;
        } else if (e == a.E) {
            a.offsets[e] = n;
        }
    }
}

}  // namespace moe
