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
// Launch: one warp per token, 8 tokens per CTA.  The CTA that finishes last
// (a release/acquire ticket) runs the grouping over all T*k entries, so route
// is a single kernel whatever T is.
#pragma once
#include "common.cuh"

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
    unsigned int* ticket;   // zero between launches
    int* err;
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

template <int NI>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(RouteArgs a) {
    extern __shared__ int smem_hist[];
    __shared__ int is_last;
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kRouteWarps + warp;
    if (t < a.T) route_token<NI>(a, t, lane);
    if (gridDim.x == 1) {        // the only CTA: no ticket needed
        __syncthreads();
        group_entries(a, smem_hist);
        pdl_trigger();
        return;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned int prev;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(a.ticket) : "memory");
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    group_entries(a, smem_hist);
    pdl_trigger();
    if (threadIdx.x == 0) *a.ticket = 0;
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
