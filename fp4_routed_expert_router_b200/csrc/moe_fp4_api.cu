// moe_fp4_api.cu -- C ABI of libmoe_fp4 (declared in include/moe_fp4.h):
// context, HBM expert arena with its (layer, expert) -> slot table, slot
// loading, routing and the expert FFN forward.  All compute runs in the CUDA
// kernels of csrc/*.cuh; there is no host-side arithmetic on the data path and
// no CPU fallback.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moe_fp4.h"
#include "common.cuh"
#include "decode_common.cuh"
#include "decode_mx.cuh"
#include "router.cuh"
#include "slot_layout.cuh"
#include "residency.h"
#include "tc_prefill.cuh"

using namespace moe;

struct moe_fp4_ctx {
    moe_fp4_config cfg{};
    int device = 0;
    int sm_count = 0;
    size_t slot_bytes = 0;
    SlotLayout lay{};                  // arrangement of an expert inside its slot
    uint8_t* arena = nullptr;
    bool own_arena = false;
    int32_t* d_table = nullptr;        // [L][E]
    uint8_t* d_rowref = nullptr;       // [n_slots][2I + H] largest scale byte of each weight row
    uint8_t* d_staging = nullptr;      // one expert, checkpoint layout
    uint16_t* d_hh = nullptr;          // [max_tokens*k, I] f16 prescaled h rows (tcgen05 f16 path)
    float* d_o = nullptr;              // [max_tokens*k, H] fp32
    float* d_norm = nullptr;           // [max_tokens*k] fp32 (saliency)
    int32_t* d_grp = nullptr;          // expert_outputs grouping: counts [E], offsets [E+1], perm [max_tokens*k]
    // decode kernel (decode_mx.cuh) workspace, for up to mx_ent token-expert entries
    int mx_ent = 0;
    uint8_t* d_mx = nullptr;           // one allocation holding the buffers below
    MxArgs mx{};                       // its buffer pointers (xp, xsf, hp, hsf, part, seq, cnt, ready, zero)
    int* d_err = nullptr;              // error word [4]
    unsigned int* d_ticket = nullptr;  // route kernel barriers + per-CTA expert counts (ticket_words)
    unsigned long long timeout_ns = 1000000000ull;   // bounded device waits
    std::vector<int32_t> h_table;      // host mirror of d_table
    std::vector<int64_t> slot_owner;   // slot -> layer*E+expert or -1
    int path = MOE_FP4_PATH_AUTO;
    int smem_optin = 0;                // opt-in shared memory per block (bytes)
    bool profile = false;
    struct ProfRec { const char* name; cudaEvent_t a, b; };
    std::vector<ProfRec> prof;         // profiled launches not yet read
    std::vector<cudaEvent_t> ev_free;  // recycled events
    TcPlan tc{};                       // tcgen05 prefill workspace
    // expert streaming (moe_fp4_stream_experts): LRU clock per slot, two
    // staging buffers filled on a copy stream, statistics
    std::vector<uint64_t> slot_last;
    uint64_t lru_clock = 0;
    int64_t stream_stats[3] = {0, 0, 0};   // hits, misses, bytes copied
    uint8_t* d_stage2[2] = {nullptr, nullptr};
    cudaStream_t copy_stream = nullptr;
    cudaEvent_t st_ready[2] = {nullptr, nullptr}, st_free[2] = {nullptr, nullptr};
    unsigned ring = 0;
    std::string host_msg;
    moe_fp4_status host_status = MOE_FP4_OK;
};

namespace {

moe_fp4_status host_fail(moe_fp4_ctx* c, moe_fp4_status s, const char* fmt, ...) {
    if (c) {
        char buf[256];
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(buf, sizeof buf, fmt, ap);
        va_end(ap);
        c->host_msg = buf;
        c->host_status = s;
    }
    return s;
}

moe_fp4_status cuda_fail(moe_fp4_ctx* c, cudaError_t e, const char* what) {
    return host_fail(c, MOE_FP4_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool config_ok(const moe_fp4_config* c) {
    if (!c) return false;
    if (c->hidden <= 0 || c->inter <= 0 || c->hidden % 128 || c->inter % 128) return false;
    if (c->n_experts <= 0 || c->n_experts > 1024) return false;
    if (c->top_k < 1 || c->top_k > 32 || c->top_k > c->n_experts) return false;
    if (c->n_layers <= 0 || c->n_slots <= 0 || c->max_tokens <= 0) return false;
    if (static_cast<long long>(c->max_tokens) * c->top_k > (1LL << 30)) return false;
    return true;
}

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaEvent_t take_event(moe_fp4_ctx* c) {
    if (!c->ev_free.empty()) {
        cudaEvent_t e = c->ev_free.back();
        c->ev_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Launch with programmatic dependent launch; bracket with events when the
// context profiles (at most 65536 pending records are kept).
template <typename Kern, typename... Args>
cudaError_t launch_k(moe_fp4_ctx* c, const char* name, Kern kern, dim3 grid, dim3 block, size_t smem,
                     cudaStream_t s, Args... args) {
    const bool prof = c->profile && c->prof.size() < 65536;
    cudaEvent_t ea = nullptr, eb = nullptr;
    if (prof) {
        ea = take_event(c);
        eb = take_event(c);
        cudaEventRecord(ea, s);
    }
    cudaError_t e = launch_pdl(kern, grid, block, smem, s, args...);
    if (prof) {
        cudaEventRecord(eb, s);
        c->prof.push_back({name, ea, eb});
    }
    return e;
}

// Words of the route kernel's grid scratch: two barriers, an exit count and a
// failure flag, then one row of expert counts per CTA (at most one CTA per SM).
size_t ticket_words(const moe_fp4_ctx* c) {
    return 4 + static_cast<size_t>(c->sm_count) * static_cast<size_t>(c->cfg.n_experts);
}

// The same with a cooperative launch (all CTAs co-resident; no PDL attribute,
// so the kernel starts once its predecessor has completed).
template <typename Kern, typename... Args>
cudaError_t launch_coop_k(moe_fp4_ctx* c, const char* name, Kern kern, dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, Args... args) {
    const bool prof = c->profile && c->prof.size() < 65536;
    cudaEvent_t ea = nullptr, eb = nullptr;
    if (prof) {
        ea = take_event(c);
        eb = take_event(c);
        cudaEventRecord(ea, s);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (prof) {
        cudaEventRecord(eb, s);
        c->prof.push_back({name, ea, eb});
    }
    return e;
}

// Re-lay one expert from the staging buffer (checkpoint layout: w1, w3, w2
// codes, then s1, s3, s2 scales, row-major) into its slot (slot_layout.cuh):
// one thread per 16-byte chunk of codes (32 codes of one row and one scale
// block, contiguous in both layouts), one per scale byte (checked against the
// supported range [2, 252]), and one per weight row for the row's largest
// scale byte (rowref, used by the f16 tcgen05 path).  Thread 0 maps (layer,
// expert) -> slot.
__global__ void load_slot_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, SlotLayout L,
                                 uint8_t* __restrict__ rowref, int32_t* table, int map_index, int slot, int* err) {
    const size_t H = L.H, I = L.I;
    const size_t n13 = I * H / 32, n2 = H * I / 32;        // 16-byte code chunks of w1 (w3), w2
    const size_t s13 = I * H / 32, s2 = H * I / 32;        // scale bytes of s1 (s3), s2
    const size_t sbase = 3 * I * H / 2;                      // scales start after the codes
    const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
    if (i == 0 && map_index >= 0) table[map_index] = slot;
    if (i < 2 * n13 + n2) {
        size_t so, dofs;
        slot_code_chunk(L, i, &so, &dofs);
        uint4 w;   // the staging buffer is only 4-byte aligned
        w.x = *reinterpret_cast<const uint32_t*>(src + so + 0);
        w.y = *reinterpret_cast<const uint32_t*>(src + so + 4);
        w.z = *reinterpret_cast<const uint32_t*>(src + so + 8);
        w.w = *reinterpret_cast<const uint32_t*>(src + so + 12);
        *reinterpret_cast<uint4*>(dst + dofs) = w;
        return;
    }
    const size_t b = i - (2 * n13 + n2);
    if (b < 2 * s13 + s2) {
        const uint8_t v = src[sbase + b];
        dst[slot_scale_byte(L, b)] = v;
        if (v < 2 || v > 252) latch_error(err, ERR_EINVAL, static_cast<int>(b), KID_LOAD);
        return;
    }
    const size_t r = b - (2 * s13 + s2);                     // weight row: w1 rows, w3 rows, w2 rows
    if (r >= 2 * I + H || rowref == nullptr) return;
    const size_t n = r < 2 * I ? H / 32 : I / 32;
    const uint8_t* sp = src + sbase + (r < 2 * I ? r * (H / 32) : 2 * s13 + (r - 2 * I) * (I / 32));
    uint8_t mx = 0;
    for (size_t j = 0; j < n; ++j) mx = sp[j] > mx ? sp[j] : mx;
    rowref[static_cast<size_t>(slot) * (2 * I + H) + r] = mx;
}

inline size_t load_threads(const SlotLayout& L) {
    const size_t H = L.H, I = L.I;
    return 3 * I * H / 32 + 3 * I * H / 32 + 2 * I + H;   // code chunks + scale bytes + rows
}

const char* kernel_name(int kid) {
    switch (kid) {
        case KID_ROUTE: return "route";
        case KID_LOAD: return "load_expert_slot";
        case KID_UP: return "decode_layer (w1/w3)";
        case KID_DOWN: return "decode_layer (w2)";
        case KID_COMBINE: return "combine";
        case KID_TC_UP: return "tc_up";
        case KID_TC_DOWN: return "tc_down";
        case KID_GATHER: return "gather";
        default: return "?";
    }
}

// ---- decode path: the persistent layer kernel (decode_mx.cuh), one CTA per
// SM, all co-resident (cooperative launch): CTAs wait on one another's flags.
cudaError_t launch_mx(const MxArgs& a, const SlotLayout& L, const MxPlan& p, int grid, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kMxThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(p.smem_bytes);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, moe_fp4_decode_mx, a, L, p);
}

cudaError_t allow_mx_smem(int bytes) {
    return cudaFuncSetAttribute(reinterpret_cast<const void*>(moe_fp4_decode_mx),
                                cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// Byte offsets of the decode workspace buffers inside one allocation (each
// 256-byte aligned): first the part that persists across launches at fixed
// offsets -- the launch sequence number, 1 KB of zeros, the up-item flags and
// the tagged counters (all zero at creation) -- then the per-launch buffers.
struct MxOffsets {
    size_t seq, zero, ready, cnt, xp, xsf, hp, hsf, part, total;
};
inline MxOffsets mx_offsets(const MxSizes& z, size_t ready_bytes, size_t cnt_bytes) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    MxOffsets o;
    o.seq = 0;
    o.zero = 256;
    o.ready = 256 + 1024;
    o.cnt = up(o.ready + ready_bytes);
    o.xp = up(o.cnt + 2 * cnt_bytes);   // two counter banks
    o.xsf = up(o.xp + z.xp);
    o.hp = up(o.xsf + z.xsf);
    o.hsf = up(o.hp + z.hp);
    o.part = up(o.hsf + z.hsf);
    o.total = up(o.part + z.part);
    return o;
}
inline void mx_bind(MxArgs* a, uint8_t* base, const MxOffsets& o, size_t cnt_bytes) {
    a->seq = reinterpret_cast<unsigned int*>(base + o.seq);
    a->cnt = reinterpret_cast<unsigned int*>(base + o.cnt);
    a->cnt_cap = static_cast<int>(cnt_bytes / sizeof(unsigned int));
    a->ready = reinterpret_cast<unsigned int*>(base + o.ready);
    a->zero = base + o.zero;
    a->xp = base + o.xp;
    a->xsf = base + o.xsf;
    a->hp = base + o.hp;
    a->hsf = base + o.hsf;
    a->part = reinterpret_cast<float*>(base + o.part);
}

// Launch the decode kernel bracketed by profiling events when the context
// profiles (c may be NULL).
cudaError_t decode_run(moe_fp4_ctx* c, const MxArgs& a, const SlotLayout& L, const MxPlan& p, int grid,
                       cudaStream_t s) {
    const bool prof = c && c->profile && c->prof.size() < 65536;
    cudaEvent_t ea = nullptr, eb = nullptr;
    if (prof) {
        ea = take_event(c);
        eb = take_event(c);
        cudaEventRecord(ea, s);
    }
    cudaError_t e = launch_mx(a, L, p, grid, s);
    if (prof) {
        cudaEventRecord(eb, s);
        c->prof.push_back({"decode_layer", ea, eb});
    }
    return e;
}

// Plan of a decode launch over the context's workspace (ok = 0 if it does not fit).
MxPlan decode_plan(moe_fp4_ctx* c, int T, int k, bool routed) {
    if (T * k > c->mx_ent || T > c->mx_ent) return MxPlan{};
    return make_mx_plan(c->lay, T, k, c->cfg.n_experts, routed, c->smem_optin);
}

// Decode arguments over the context's workspace.
MxArgs decode_args(moe_fp4_ctx* c, int layer, int k, int T, const uint16_t* x) {
    MxArgs a = c->mx;
    a.arena = c->arena;
    a.slot_bytes = c->slot_bytes;
    a.slot_table = c->d_table;
    a.layer = layer;
    a.E = c->cfg.n_experts;
    a.k = k;
    a.H = c->cfg.hidden;
    a.I = c->cfg.inter;
    a.T = T;
    a.x = x;
    a.obuf = c->d_o;
    a.err = c->d_err;
    a.timeout_ns = c->timeout_ns;
    return a;
}

// tcgen05 path: gather x rows by expert (prescaled f16), up GEMM (bf16 h),
// h -> prescaled f16, down GEMM.
cudaError_t tc_forward(moe_fp4_ctx* c, const ExpertArgs& a, const SlotLayout& L, int T, cudaStream_t s) {
    const TcPlan& p = c->tc;
    if (!p.ready) return cudaErrorNotSupported;
    const int rows = T * a.k;
    cudaError_t e = launch_k(c, "gather", gather_rows_kernel, dim3(static_cast<unsigned>(rows)), dim3(256), 0, s,
                             a.x, a.perm, a.k, a.H, rows, p.xg, p.xcs);
    if (e != cudaSuccess) return e;
    const int nmax = tc_nmax_for(T);
    TcArgs tu = tc_args(p, a, L, T, true, c->d_rowref, nmax), td = tc_args(p, a, L, T, false, c->d_rowref, nmax);
    if (!tu.centries || !td.centries) return cudaErrorNotSupported;
    tu.timeout_ns = td.timeout_ns = c->timeout_ns;
    const dim3 grid(static_cast<unsigned>(p.sm_count)), block(kTcThreads);
    const bool narrow = nmax == kTcNmaxNarrow;
    e = launch_k(c, "tc_up", narrow ? tc_gemm_kernel<true, kTcNmaxNarrow> : tc_gemm_kernel<true, kTcNmaxWide>, grid,
                 block, tc_smem_bytes(tu), s, tu, p.map_x);
    if (e != cudaSuccess) return e;
    e = launch_k(c, "h_convert", h_convert_kernel, dim3(static_cast<unsigned>((rows * 32 + 255) / 256)), dim3(256), 0,
                 s, static_cast<const uint16_t*>(p.hb), a.I, rows, p.hh, p.hcs);
    if (e != cudaSuccess) return e;
    return launch_k(c, "tc_down", narrow ? tc_gemm_kernel<false, kTcNmaxNarrow> : tc_gemm_kernel<false, kTcNmaxWide>,
                    grid, block, tc_smem_bytes(td), s, td, p.map_h);
}

}  // namespace

extern "C" {

size_t moe_fp4_slot_bytes(const moe_fp4_config* cfg) {
    if (!config_ok(cfg)) return 0;
    const size_t H = cfg->hidden, I = cfg->inter;
    return 2 * (I * H / 2 + I * H / 32) + (H * I / 2 + H * I / 32);
}

moe_fp4_status moe_fp4_create(const moe_fp4_config* cfg, int device, void* arena,
                              size_t arena_bytes, moe_fp4_ctx** out) {
    if (!out) return MOE_FP4_EINVAL;
    *out = nullptr;
    if (!config_ok(cfg)) return MOE_FP4_EINVAL;
    moe_fp4_ctx* c = new moe_fp4_ctx();
    c->cfg = *cfg;
    c->device = device;
    const size_t H = cfg->hidden, I = cfg->inter, E = cfg->n_experts, L = cfg->n_layers;
    c->slot_bytes = moe_fp4_slot_bytes(cfg);
    c->lay = make_slot_layout(cfg->hidden, cfg->inter);
    const size_t need = c->slot_bytes * static_cast<size_t>(cfg->n_slots);
    auto bail = [&](moe_fp4_status s) {
        moe_fp4_destroy(c);
        return s;
    };
    if (arena && (arena_bytes < need || (reinterpret_cast<uintptr_t>(arena) & 255))) return bail(MOE_FP4_EINVAL);
    cudaError_t e = cudaSetDevice(device);
    if (e != cudaSuccess) return bail(MOE_FP4_ECUDA);
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
    cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, device);
    cudaDeviceGetAttribute(&c->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    if (major < 10) return bail(MOE_FP4_ECUDA);   // sm_100a code only
    if (arena) {
        c->arena = static_cast<uint8_t*>(arena);
    } else {
        if (cudaMalloc(&c->arena, need) != cudaSuccess) { cudaGetLastError(); return bail(MOE_FP4_ENOMEM); }
        c->own_arena = true;
    }
    const size_t ent = static_cast<size_t>(cfg->max_tokens) * cfg->top_k;
    const size_t rowref_bytes = static_cast<size_t>(cfg->n_slots) * (2 * I + H);
    if (cudaMalloc(&c->d_table, sizeof(int32_t) * L * E) != cudaSuccess ||
        cudaMalloc(&c->d_rowref, rowref_bytes) != cudaSuccess ||
        cudaMalloc(&c->d_staging, c->slot_bytes) != cudaSuccess ||
        cudaMalloc(&c->d_hh, sizeof(uint16_t) * ent * I) != cudaSuccess ||
        cudaMalloc(&c->d_o, sizeof(float) * ent * H) != cudaSuccess ||
        cudaMalloc(&c->d_norm, sizeof(float) * (ent > 0 ? ent : 1)) != cudaSuccess ||
        cudaMalloc(&c->d_grp, sizeof(int32_t) * (2 * static_cast<size_t>(cfg->n_experts) + 1 + ent)) != cudaSuccess ||
        cudaMalloc(&c->d_err, sizeof(int) * 4) != cudaSuccess ||
        cudaMalloc(&c->d_ticket, sizeof(unsigned int) * ticket_words(c)) != cudaSuccess) {
        cudaGetLastError();
        return bail(MOE_FP4_ENOMEM);
    }
    c->smem_optin -= 1024;   // room for the kernels' static shared memory
    // decode workspace: batches up to kMxMaxEntries token-expert entries
    c->mx_ent = static_cast<int>(ent < static_cast<size_t>(kMxMaxEntries) ? ent : kMxMaxEntries);
    const MxSizes mz = mx_sizes(c->lay, c->mx_ent, 1, cfg->n_experts, c->sm_count);
    const MxOffsets mo = mx_offsets(mz, mz.ready, mz.cnt);
    if (cudaMalloc(&c->d_mx, mo.total) != cudaSuccess) {
        cudaGetLastError();
        return bail(MOE_FP4_ENOMEM);
    }
    mx_bind(&c->mx, c->d_mx, mo, mz.cnt);
    if (allow_mx_smem(c->smem_optin) != cudaSuccess ||
        cudaMemset(c->d_mx, 0, mo.xp) != cudaSuccess) {   // sequence, counters, flags, zero block
        cudaGetLastError();
        return bail(MOE_FP4_ECUDA);
    }
    if (tc_plan_create(&c->tc, *cfg, c->d_hh, c->sm_count, c->smem_optin) != cudaSuccess) {
        cudaGetLastError();
        return bail(MOE_FP4_ENOMEM);
    }
    if (cudaMemset(c->d_table, 0xFF, sizeof(int32_t) * L * E) != cudaSuccess ||
        cudaMemset(c->d_rowref, 0, rowref_bytes) != cudaSuccess ||
        cudaMemset(c->d_err, 0, sizeof(int) * 4) != cudaSuccess ||
        cudaMemset(c->d_ticket, 0, sizeof(unsigned int) * ticket_words(c)) != cudaSuccess ||
        cudaDeviceSynchronize() != cudaSuccess)
        return bail(MOE_FP4_ECUDA);
    c->h_table.assign(L * E, -1);
    c->slot_owner.assign(cfg->n_slots, -1);
    *out = c;
    return MOE_FP4_OK;
}

void moe_fp4_destroy(moe_fp4_ctx* c) {
    if (!c) return;
    cudaSetDevice(c->device);
    cudaDeviceSynchronize();
    if (c->own_arena) cudaFree(c->arena);
    cudaFree(c->d_table);
    cudaFree(c->d_rowref);
    cudaFree(c->d_staging);
    cudaFree(c->d_hh);
    cudaFree(c->d_o);
    cudaFree(c->d_norm);
    cudaFree(c->d_grp);
    cudaFree(c->d_mx);
    for (int b = 0; b < 2; ++b) {
        if (c->d_stage2[b]) cudaFree(c->d_stage2[b]);
        if (c->st_ready[b]) cudaEventDestroy(c->st_ready[b]);
        if (c->st_free[b]) cudaEventDestroy(c->st_free[b]);
    }
    if (c->copy_stream) cudaStreamDestroy(c->copy_stream);
    cudaFree(c->d_err);
    cudaFree(c->d_ticket);
    tc_plan_destroy(&c->tc);
    for (auto& r : c->prof) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
    for (auto e : c->ev_free) cudaEventDestroy(e);
    delete c;
}

void* moe_fp4_arena(moe_fp4_ctx* c) { return c ? c->arena : nullptr; }

moe_fp4_status moe_fp4_set_option(moe_fp4_ctx* c, int option, int value) {
    if (!c) return MOE_FP4_EINVAL;
    if (option == MOE_FP4_OPT_PATH && value >= MOE_FP4_PATH_AUTO && value <= MOE_FP4_PATH_TC) {
        c->path = value;
        return MOE_FP4_OK;
    }
    if (option == MOE_FP4_OPT_PROFILE && (value == 0 || value == 1)) {
        c->profile = value != 0;
        return MOE_FP4_OK;
    }
    if (option == MOE_FP4_OPT_WAIT_LIMIT_US && value >= 0 && value <= 10000000) {
        c->timeout_ns = value == 0 ? 1000000000ull : static_cast<unsigned long long>(value) * 1000ull;
        return MOE_FP4_OK;
    }
    return host_fail(c, MOE_FP4_EINVAL, "set_option: unknown option %d / value %d", option, value);
}

moe_fp4_status moe_fp4_load_expert_slot(moe_fp4_ctx* c, int layer, int expert, int slot,
                                        const uint8_t* w1, const uint8_t* w1_scale,
                                        const uint8_t* w3, const uint8_t* w3_scale,
                                        const uint8_t* w2, const uint8_t* w2_scale, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (layer < 0 || layer >= g.n_layers || expert < 0 || expert >= g.n_experts || slot < -1 || slot >= g.n_slots)
        return host_fail(c, MOE_FP4_EINVAL, "load_expert_slot: layer %d expert %d slot %d out of range",
                         layer, expert, slot);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int idx = layer * g.n_experts + expert;
    cudaError_t e;
    // release what (layer, expert) and `slot` were bound to
    const int old_slot = c->h_table[idx];
    if (old_slot >= 0) c->slot_owner[old_slot] = -1;
    c->h_table[idx] = -1;
    if (slot == -1) {
        e = cudaMemsetAsync(c->d_table + idx, 0xFF, sizeof(int32_t), s);
        return e == cudaSuccess ? MOE_FP4_OK : cuda_fail(c, e, "load_expert_slot: unmap");
    }
    if (!w1 || !w1_scale || !w3 || !w3_scale || !w2 || !w2_scale)
        return host_fail(c, MOE_FP4_EINVAL, "load_expert_slot: NULL tensor");
    const int64_t prev = c->slot_owner[slot];
    if (prev >= 0) {
        c->h_table[prev] = -1;
        e = cudaMemsetAsync(c->d_table + prev, 0xFF, sizeof(int32_t), s);
        if (e != cudaSuccess) return cuda_fail(c, e, "load_expert_slot: evict");
    }
    const size_t H = g.hidden, I = g.inter;
    const size_t c13 = I * H / 2, sc0 = 3 * I * H / 2;     // checkpoint layout in the staging buffer
    const struct { const uint8_t* p; size_t off, n; } parts[6] = {
        {w1, 0, c13},           {w3, c13, c13},                 {w2, 2 * c13, H * I / 2},
        {w1_scale, sc0, I * H / 32}, {w3_scale, sc0 + I * H / 32, I * H / 32},
        {w2_scale, sc0 + 2 * I * H / 32, H * I / 32}};
    for (const auto& p : parts) {
        e = cudaMemcpyAsync(c->d_staging + p.off, p.p, p.n, cudaMemcpyDefault, s);
        if (e != cudaSuccess) return cuda_fail(c, e, "load_expert_slot: copy");
    }
    const size_t threads = load_threads(c->lay);
    load_slot_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(
        c->d_staging, c->arena + static_cast<size_t>(slot) * c->slot_bytes, c->lay, c->d_rowref, c->d_table, idx,
        slot, c->d_err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(c, e, "load_expert_slot: launch");
    c->h_table[idx] = slot;
    c->slot_owner[slot] = idx;
    return MOE_FP4_OK;
}

moe_fp4_status moe_fp4_stream_experts(moe_fp4_ctx* c, int layer, const int32_t* experts, int n,
                                      const uint8_t* const* objects, int32_t* slots_out, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (layer < 0 || layer >= g.n_layers || n < 0 || (n > 0 && !experts))
        return host_fail(c, MOE_FP4_EINVAL, "stream_experts: layer %d / n %d / experts", layer, n);
    if (n > g.n_slots)
        return host_fail(c, MOE_FP4_EINVAL, "stream_experts: %d experts exceed the %d slots", n, g.n_slots);
    std::vector<int64_t> keys(n);
    std::vector<uint8_t> seen(g.n_experts, 0);
    for (int i = 0; i < n; ++i) {
        const int e = experts[i];
        if (e < 0 || e >= g.n_experts || seen[e])
            return host_fail(c, MOE_FP4_EINVAL, "stream_experts: expert %d out of range or repeated", e);
        seen[e] = 1;
        keys[i] = static_cast<int64_t>(layer) * g.n_experts + e;
        if (c->h_table[keys[i]] < 0 && (!objects || !objects[i]))
            return host_fail(c, MOE_FP4_EINVAL, "stream_experts: expert %d is not resident and has no object", e);
    }
    if (n == 0) return MOE_FP4_OK;
    cudaSetDevice(c->device);
    cudaError_t e;
    if (!c->copy_stream) {   // first use: staging buffers, copy stream, events
        for (int b = 0; b < 2; ++b) {
            if ((e = cudaMalloc(&c->d_stage2[b], c->slot_bytes)) != cudaSuccess)
                return host_fail(c, MOE_FP4_ENOMEM, "stream_experts: staging allocation failed");
            if ((e = cudaEventCreateWithFlags(&c->st_ready[b], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&c->st_free[b], cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(c, e, "stream_experts: events");
        }
        if ((e = cudaStreamCreateWithFlags(&c->copy_stream, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(c, e, "stream_experts: copy stream");
    }
    if (c->slot_last.size() != static_cast<size_t>(g.n_slots)) c->slot_last.assign(g.n_slots, 0);
    std::vector<int32_t> slot(n);
    std::vector<uint8_t> hit(n);
    std::vector<int64_t> evicted(n);
    if (!lru_plan(c->slot_owner.data(), c->h_table.data(), c->slot_last.data(), g.n_slots, ++c->lru_clock,
                  keys.data(), n, slot.data(), hit.data(), evicted.data()))
        return host_fail(c, MOE_FP4_EINVAL, "stream_experts: no slot plan");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t threads = load_threads(c->lay);
    for (int i = 0; i < n; ++i) {
        if (hit[i]) {
            ++c->stream_stats[0];
            continue;
        }
        const unsigned b = c->ring++ & 1u;
        // the copy waits until the last relayout that read this staging buffer is done
        if ((e = cudaStreamWaitEvent(c->copy_stream, c->st_free[b], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(c->d_stage2[b], objects[i], c->slot_bytes, cudaMemcpyDefault, c->copy_stream)) !=
                cudaSuccess ||
            (e = cudaEventRecord(c->st_ready[b], c->copy_stream)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(s, c->st_ready[b], 0)) != cudaSuccess)
            return cuda_fail(c, e, "stream_experts: copy");
        if (evicted[i] >= 0 &&
            (e = cudaMemsetAsync(c->d_table + evicted[i], 0xFF, sizeof(int32_t), s)) != cudaSuccess)
            return cuda_fail(c, e, "stream_experts: evict");
        load_slot_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, s>>>(
            c->d_stage2[b], c->arena + static_cast<size_t>(slot[i]) * c->slot_bytes, c->lay, c->d_rowref,
            c->d_table, static_cast<int>(keys[i]), slot[i], c->d_err);
        if ((e = cudaGetLastError()) != cudaSuccess || (e = cudaEventRecord(c->st_free[b], s)) != cudaSuccess)
            return cuda_fail(c, e, "stream_experts: relayout");
        ++c->stream_stats[1];
        c->stream_stats[2] += static_cast<int64_t>(c->slot_bytes);
    }
    if (slots_out)
        for (int i = 0; i < n; ++i) slots_out[i] = slot[i];
    return MOE_FP4_OK;
}

moe_fp4_status moe_fp4_residency_stats(moe_fp4_ctx* c, int64_t* stats) {
    if (!c || !stats) return MOE_FP4_EINVAL;
    for (int i = 0; i < 3; ++i) stats[i] = c->stream_stats[i];
    return MOE_FP4_OK;
}

moe_fp4_status moe_fp4_route(moe_fp4_ctx* c, int layer, const float* logits, const uint8_t* keep_mask,
                             int T, int32_t* ids, float* weights, int32_t* counts, int32_t* offsets,
                             int32_t* perm, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (layer < 0 || layer >= g.n_layers || T < 0 || T > g.max_tokens)
        return host_fail(c, MOE_FP4_EINVAL, "route: layer %d / T %d out of range", layer, T);
    if ((T > 0 && (!logits || !ids || !weights || !perm)) || !counts || !offsets)
        return host_fail(c, MOE_FP4_EINVAL, "route: NULL output");
    RouteArgs a{logits, keep_mask, T, g.n_experts, g.top_k, ids, weights, counts, offsets, perm,
                c->d_ticket, c->d_err, c->timeout_ns};
    int want = T > 0 ? (T + kRouteWarps - 1) / kRouteWarps : 1;   // a warp per token, up to one CTA per SM
    const unsigned grid = static_cast<unsigned>(want < c->sm_count ? want : c->sm_count);
    const size_t smem = sizeof(int) * (2 * static_cast<size_t>(g.n_experts) + 1);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (T * g.top_k <= 32) {   // one warp: route + bitonic grouping
        if (g.n_experts <= 128)
            e = launch_k(c, "route", route_small_kernel<4>, dim3(1), dim3(32), 0, s, a);
        else if (g.n_experts <= 384)
            e = launch_k(c, "route", route_small_kernel<12>, dim3(1), dim3(32), 0, s, a);
        else
            e = launch_k(c, "route", route_small_kernel<32>, dim3(1), dim3(32), 0, s, a);
    } else if (g.n_experts <= 128)
        e = launch_coop_k(c, "route", route_grid_kernel<4>, dim3(grid), dim3(kRouteWarps * 32), smem, s, a);
    else if (g.n_experts <= 384)
        e = launch_coop_k(c, "route", route_grid_kernel<12>, dim3(grid), dim3(kRouteWarps * 32), smem, s, a);
    else
        e = launch_coop_k(c, "route", route_grid_kernel<32>, dim3(grid), dim3(kRouteWarps * 32), smem, s, a);
    return e == cudaSuccess ? MOE_FP4_OK : cuda_fail(c, e, "route: launch");
}

moe_fp4_status moe_fp4_forward(moe_fp4_ctx* c, int layer, const uint16_t* x, int T, const int32_t* ids,
                               const float* weights, const int32_t* counts, const int32_t* offsets,
                               const int32_t* perm, float* y, uint16_t* x_out, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (layer < 0 || layer >= g.n_layers || T < 0 || T > g.max_tokens)
        return host_fail(c, MOE_FP4_EINVAL, "forward: layer %d / T %d out of range", layer, T);
    if (T == 0) return MOE_FP4_OK;
    if (!x || !ids || !weights || !counts || !offsets || !perm || !y)
        return host_fail(c, MOE_FP4_EINVAL, "forward: NULL argument");
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15) ||
        (reinterpret_cast<uintptr_t>(x_out) & 7) || (reinterpret_cast<uintptr_t>(weights) & 3))
        return host_fail(c, MOE_FP4_EINVAL, "forward: x and y must be 16-byte aligned, x_out 8-byte");
    (void)ids;
    (void)counts;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int H = g.hidden, I = g.inter, E = g.n_experts, k = g.top_k;
    const bool want_tc = (c->path == MOE_FP4_PATH_TC) || (c->path == MOE_FP4_PATH_AUTO && tc_prefers(T, g));
    if (!want_tc) {   // decode path: one persistent kernel (+ the combine for batches above 16 tokens)
        const MxPlan p = decode_plan(c, T, k, false);
        if (p.ok) {
            MxArgs a = decode_args(c, layer, k, T, x);
            a.weights = const_cast<float*>(weights);
            a.offsets = const_cast<int32_t*>(offsets);
            a.perm = const_cast<int32_t*>(perm);
            const bool fuse = T <= kMxCombineMax;
            a.y = fuse ? y : nullptr;
            a.x_out = fuse ? x_out : nullptr;
            cudaError_t e = decode_run(c, a, c->lay, p, c->sm_count, s);
            if (e != cudaSuccess) return cuda_fail(c, e, "forward: decode launch");
            if (fuse) return MOE_FP4_OK;
            const int n4 = T * (H / 4);
            e = launch_k(c, "combine", combine_kernel, dim3((n4 + 255) / 256), dim3(256), 0, s,
                         static_cast<const float*>(c->d_o), weights, x, T, H, k, y, x_out);
            return e == cudaSuccess ? MOE_FP4_OK : cuda_fail(c, e, "forward: combine launch");
        }
        if (c->path == MOE_FP4_PATH_GEMV)
            return host_fail(c, MOE_FP4_EINVAL, "forward: T %d does not fit the decode kernel", T);
    }
    ExpertArgs a{c->arena, c->slot_bytes, c->d_table, layer, E, k, H, I, x, offsets, perm, c->d_o, c->d_err};
    cudaError_t e = tc_forward(c, a, c->lay, T, s);
    if (e != cudaSuccess) return cuda_fail(c, e, "forward: expert FFN launch");
    const int n4 = T * (H / 4);
    e = launch_k(c, "combine", combine_kernel, dim3((n4 + 255) / 256), dim3(256), 0, s,
                 static_cast<const float*>(c->d_o), weights, x, T, H, k, y, x_out);
    if (e != cudaSuccess) return cuda_fail(c, e, "forward: combine launch");
    return MOE_FP4_OK;
}

moe_fp4_status moe_fp4_route_forward(moe_fp4_ctx* c, int layer, const float* logits, const uint8_t* keep_mask,
                                     const uint16_t* x, int T, int32_t* ids, float* weights, int32_t* counts,
                                     int32_t* offsets, int32_t* perm, float* y, uint16_t* x_out, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (layer < 0 || layer >= g.n_layers || T < 0 || T > g.max_tokens)
        return host_fail(c, MOE_FP4_EINVAL, "route_forward: layer %d / T %d out of range", layer, T);
    if (!counts || !offsets) return host_fail(c, MOE_FP4_EINVAL, "route_forward: NULL output");
    if (T > 0 && (!logits || !x || !ids || !weights || !perm || !y))
        return host_fail(c, MOE_FP4_EINVAL, "route_forward: NULL argument");
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15) ||
        (reinterpret_cast<uintptr_t>(x_out) & 7) || (reinterpret_cast<uintptr_t>(weights) & 3))
        return host_fail(c, MOE_FP4_EINVAL, "route_forward: x and y must be 16-byte aligned, x_out 8-byte");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool want_tc = (c->path == MOE_FP4_PATH_TC) || (c->path == MOE_FP4_PATH_AUTO && tc_prefers(T, g));
    if (T > 0 && !want_tc) {
        const MxPlan p = decode_plan(c, T, g.top_k, true);
        if (p.ok) {   // routing inside the layer kernel: one launch for the whole layer
            MxArgs a = decode_args(c, layer, g.top_k, T, x);
            a.logits = logits;
            a.keep = keep_mask;
            a.ids = ids;
            a.weights = weights;
            a.counts = counts;
            a.offsets = offsets;
            a.perm = perm;
            a.y = y;
            a.x_out = x_out;
            cudaError_t e = decode_run(c, a, c->lay, p, c->sm_count, s);
            return e == cudaSuccess ? MOE_FP4_OK : cuda_fail(c, e, "route_forward: decode launch");
        }
    }
    moe_fp4_status st = moe_fp4_route(c, layer, logits, keep_mask, T, ids, weights, counts, offsets, perm, stream);
    if (st != MOE_FP4_OK || T == 0) return st;
    return moe_fp4_forward(c, layer, x, T, ids, weights, counts, offsets, perm, y, x_out, stream);
}

moe_fp4_status moe_fp4_expert_outputs(moe_fp4_ctx* c, int layer, const uint16_t* x, int n, const int32_t* experts,
                                      float* o, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (layer < 0 || layer >= g.n_layers || n < 0 || n > g.max_tokens * g.top_k)
        return host_fail(c, MOE_FP4_EINVAL, "expert_outputs: layer %d / n %d out of range", layer, n);
    if (n == 0) return MOE_FP4_OK;
    if (!x || !experts || !o) return host_fail(c, MOE_FP4_EINVAL, "expert_outputs: NULL argument");
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(o) & 15))
        return host_fail(c, MOE_FP4_EINVAL, "expert_outputs: x and o must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int H = g.hidden, I = g.inter, E = g.n_experts;
    int32_t* counts = c->d_grp;
    int32_t* offsets = counts + E;
    int32_t* perm = offsets + E + 1;
    // group the n entries by expert (one CTA; entries with an id outside [0, E) latch EINVAL)
    RouteArgs ra{nullptr, nullptr, n, E, 1, const_cast<int32_t*>(experts), nullptr, counts, offsets, perm,
                 c->d_ticket, c->d_err};
    cudaError_t e = launch_k(c, "group", group_kernel, dim3(1), dim3(kRouteWarps * 32),
                             sizeof(int) * kRouteWarps * E, s, ra);
    if (e != cudaSuccess) return cuda_fail(c, e, "expert_outputs: group launch");
    const bool want_tc = (c->path == MOE_FP4_PATH_TC) || (c->path == MOE_FP4_PATH_AUTO && 4LL * n >= 3LL * E);
    if (!want_tc) {
        const MxPlan p = decode_plan(c, n, 1, false);
        if (p.ok) {   // every row its own token (k = 1), per-entry outputs only
            MxArgs a = decode_args(c, layer, 1, n, x);
            a.offsets = offsets;
            a.perm = perm;
            a.obuf = o;
            e = decode_run(c, a, c->lay, p, c->sm_count, s);
            return e == cudaSuccess ? MOE_FP4_OK : cuda_fail(c, e, "expert_outputs: decode launch");
        }
        if (c->path == MOE_FP4_PATH_GEMV)
            return host_fail(c, MOE_FP4_EINVAL, "expert_outputs: n %d does not fit the decode kernel", n);
    }
    ExpertArgs a{c->arena, c->slot_bytes, c->d_table, layer, E, 1, H, I, x, offsets, perm, o, c->d_err};
    e = tc_forward(c, a, c->lay, n, s);
    if (e != cudaSuccess) return cuda_fail(c, e, "expert_outputs: expert FFN launch");
    return MOE_FP4_OK;
}

moe_fp4_status moe_fp4_combine(moe_fp4_ctx* c, int T, const float* o, const float* weights, const uint16_t* x,
                               float* y, uint16_t* x_out, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (T < 0 || T > g.max_tokens) return host_fail(c, MOE_FP4_EINVAL, "combine: T %d out of range", T);
    if (T == 0) return MOE_FP4_OK;
    if (!o || !weights || !y || (x_out && !x)) return host_fail(c, MOE_FP4_EINVAL, "combine: NULL argument");
    if ((reinterpret_cast<uintptr_t>(o) & 15) || (reinterpret_cast<uintptr_t>(y) & 15) ||
        (x_out && ((reinterpret_cast<uintptr_t>(x) & 7) || (reinterpret_cast<uintptr_t>(x_out) & 7))))
        return host_fail(c, MOE_FP4_EINVAL, "combine: o and y must be 16-byte aligned, x and x_out 8-byte");
    const int n4 = T * (g.hidden / 4);
    cudaError_t e = launch_k(c, "combine", combine_kernel, dim3((n4 + 255) / 256), dim3(256), 0,
                             static_cast<cudaStream_t>(stream), o, weights, x, T, g.hidden, g.top_k, y, x_out);
    if (e != cudaSuccess) return cuda_fail(c, e, "combine: launch");
    return MOE_FP4_OK;
}

moe_fp4_status moe_fp4_saliency(moe_fp4_ctx* c, int T, const float* weights, const int32_t* offsets,
                                const int32_t* perm, double* saliency, void* stream) {
    if (!c) return MOE_FP4_EINVAL;
    const moe_fp4_config& g = c->cfg;
    if (T < 0 || T > g.max_tokens) return host_fail(c, MOE_FP4_EINVAL, "saliency: T %d out of range", T);
    if (T == 0) return MOE_FP4_OK;
    if (!weights || !offsets || !perm || !saliency) return host_fail(c, MOE_FP4_EINVAL, "saliency: NULL argument");
    cudaSetDevice(c->device);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int n_ent = T * g.top_k;
    cudaError_t e = launch_k(c, "entry_norm", entry_norm_kernel, dim3((n_ent * 32 + 255) / 256), dim3(256), 0, s,
                             static_cast<const float*>(c->d_o), n_ent, g.hidden, c->d_norm);
    if (e != cudaSuccess) return cuda_fail(c, e, "saliency: norm launch");
    e = launch_k(c, "saliency", saliency_kernel, dim3((g.n_experts + 127) / 128), dim3(128), 0, s,
                 static_cast<const float*>(c->d_norm), weights, offsets, perm, g.n_experts, n_ent, saliency);
    if (e != cudaSuccess) return cuda_fail(c, e, "saliency: launch");
    return MOE_FP4_OK;
}

int moe_fp4_profile_read(moe_fp4_ctx* c, const char** names, float* ms, int max) {
    if (!c) return -1;
    cudaSetDevice(c->device);
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    int n = 0;
    for (const auto& r : c->prof) {
        if (n < max) {
            float t = 0.f;
            if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return -1;
            if (names) names[n] = r.name;
            if (ms) ms[n] = t;
            ++n;
        }
        c->ev_free.push_back(r.a);
        c->ev_free.push_back(r.b);
    }
    c->prof.clear();
    return n;
}

moe_fp4_status moe_fp4_last_error(moe_fp4_ctx* c, char* msg, size_t n) {
    if (!c) return MOE_FP4_EINVAL;
    cudaSetDevice(c->device);
    std::string text;
    moe_fp4_status st = MOE_FP4_OK;
    cudaError_t e = cudaDeviceSynchronize();
    int w[4] = {0, 0, 0, 0};
    if (e == cudaSuccess) e = cudaMemcpy(w, c->d_err, sizeof w, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(c->d_err, 0, sizeof w);
    if (e != cudaSuccess) {
        st = MOE_FP4_ECUDA;
        text = std::string("cuda: ") + cudaGetErrorString(e);
    } else if (w[0] != 0) {
        st = static_cast<moe_fp4_status>(w[0]);
        char buf[160];
        const char* what = w[0] == ERR_ESLOT ? "expert has no slot" : w[0] == ERR_ETIMEOUT ? "wait timed out"
                                                                                           : "invalid data";
        snprintf(buf, sizeof buf, "%s (kernel %s, detail %d)", what, kernel_name(w[2]), w[1]);
        text = buf;
    } else if (c->host_status != MOE_FP4_OK) {
        st = c->host_status;
        text = c->host_msg;
    }
    c->host_status = MOE_FP4_OK;
    c->host_msg.clear();
    if (msg && n) {
        snprintf(msg, n, "%s", text.c_str());
    }
    return st;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Forward without allocation (moe_fp4_forward_noalloc): the decode kernel
// with its scratch in a file-scope device array instead of a context
// workspace.  Host code must not use the array's name as a device address:
// its device address is looked up once per device with cudaGetSymbolAddress.
namespace {

constexpr size_t kNoallocScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr size_t kNoallocReady = 32768;                       // up-item flags at most
constexpr size_t kNoallocCnt = 65536;                         // counters per bank at most
// Zero-initialised: the decode kernel's launch sequence number, flags and
// counters at fixed offsets at the start, then the per-launch buffers.
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];
__device__ int g_noalloc_err_sink[4];                        // errors when err == NULL

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;

// Per-device set-up on the first call (that device current): the device
// addresses of the scratch array and the error sink, the SM count, the
// opt-in shared memory, and the kernel's shared-memory attribute.
struct NoallocDevice {
    void* scratch;
    int* sink;
    int sm_count;
    int smem_limit;
};
NoallocDevice g_noalloc_dev[kMaxDevices];

bool noalloc_setup(int dev, NoallocDevice* out) {
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoallocDevice& d = g_noalloc_dev[dev];
    if (!d.scratch) {
        void* p = nullptr;
        void* q = nullptr;
        int sms = 0, optin = 0;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return false;
        if (cudaGetSymbolAddress(&q, g_noalloc_err_sink) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
        optin -= 1024;
        if (allow_mx_smem(optin) != cudaSuccess) return false;
        d.sink = static_cast<int*>(q);
        d.sm_count = sms;
        d.smem_limit = optin;
        d.scratch = p;
    }
    *out = d;
    return true;
}


}  // namespace

extern "C" moe_fp4_status moe_fp4_forward_noalloc(const moe_fp4_config* cfg, const uint8_t* arena,
                                                  const int32_t* slot_table, int layer, const uint16_t* x,
                                                  int T, const float* weights, const int32_t* offsets,
                                                  const int32_t* perm, float* y, uint16_t* x_out,
                                                  int32_t* err, void* stream) {
    if (!config_ok(cfg) || !arena || !slot_table) return MOE_FP4_EINVAL;
    if (layer < 0 || layer >= cfg->n_layers || T < 0) return MOE_FP4_EINVAL;
    if (T == 0) return MOE_FP4_OK;
    if (!x || !weights || !offsets || !perm || !y) return MOE_FP4_EINVAL;
    if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(y) & 15) ||
        (reinterpret_cast<uintptr_t>(x_out) & 7) || (reinterpret_cast<uintptr_t>(weights) & 3) ||
        (reinterpret_cast<uintptr_t>(arena) & 255))
        return MOE_FP4_EINVAL;
    const size_t H = cfg->hidden, I = cfg->inter, k = cfg->top_k, E = cfg->n_experts;
    const size_t ent = static_cast<size_t>(T) * k;
    const SlotLayout L = make_slot_layout(cfg->hidden, cfg->inter);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_FP4_ECUDA;
    NoallocDevice d{};
    if (!noalloc_setup(dev, &d)) return MOE_FP4_ECUDA;
    // scratch: the persistent header, the decode workspace of this batch, per-entry outputs
    const MxSizes z = mx_sizes(L, T, static_cast<int>(k), static_cast<int>(E), d.sm_count);
    const MxOffsets o = mx_offsets(z, kNoallocReady * 4, kNoallocCnt * 4);
    const size_t o_o = o.total, need = o_o + ent * H * 4;
    if (need > kNoallocScratchBytes || z.ready > kNoallocReady * 4 || z.cnt > kNoallocCnt * 4) return MOE_FP4_EINVAL;
    const MxPlan p = make_mx_plan(L, T, static_cast<int>(k), static_cast<int>(E), false, d.smem_limit);
    if (!p.ok) return MOE_FP4_EINVAL;                         // shape or batch the decode kernel does not take
    uint8_t* sp = static_cast<uint8_t*>(d.scratch);
    MxArgs a{};
    mx_bind(&a, sp, o, kNoallocCnt * 4);
    a.arena = arena;
    a.slot_bytes = moe_fp4_slot_bytes(cfg);
    a.slot_table = slot_table;
    a.layer = layer;
    a.E = static_cast<int>(E);
    a.k = static_cast<int>(k);
    a.H = static_cast<int>(H);
    a.I = static_cast<int>(I);
    a.T = T;
    a.weights = const_cast<float*>(weights);
    a.offsets = const_cast<int32_t*>(offsets);
    a.perm = const_cast<int32_t*>(perm);
    a.x = x;
    a.obuf = reinterpret_cast<float*>(sp + o_o);
    const bool fuse = T <= kMxCombineMax;                     // else the combine kernel follows
    a.y = fuse ? y : nullptr;
    a.x_out = fuse ? x_out : nullptr;
    a.err = err ? reinterpret_cast<int*>(err) : d.sink;
    a.timeout_ns = 1000000000ull;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_mx(a, L, p, d.sm_count, s) != cudaSuccess) return MOE_FP4_ECUDA;
    if (!fuse) {
        const int n4 = T * static_cast<int>(H / 4);
        if (launch_pdl(combine_kernel, dim3((n4 + 255) / 256), dim3(256), 0, s, static_cast<const float*>(a.obuf),
                       weights, x, T, static_cast<int>(H), static_cast<int>(k), y, x_out) != cudaSuccess)
            return MOE_FP4_ECUDA;
    }
    return MOE_FP4_OK;
}
