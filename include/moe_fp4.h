/*
 * moe_fp4.h -- C ABI of the routed-expert FP4 FFN library (libmoe_fp4.so).
 *
 * One MoE layer of the DeepSeek-V4.1-Flash shape: hidden 5120, expert
 * intermediate 2304, 384 routed experts, top-6 per token (10100.com article
 * 151357339, section "moe专家的容量瓶颈").  Experts live in an HBM arena of
 * fixed-size slots addressed through a (layer, expert) -> slot table, the
 * "Expert Arena" of the same article (section "方案一：hot expert常驻内存").
 *
 * The layer computes, per token t:
 *   router   ids[t, 0..k) = top-k of the fp32 logits (larger first, lower
 *            expert index on ties), w[t, j] = softmax renormalised over them;
 *   permute  the (t, j) entries grouped by expert;
 *   expert   a1 = x W1^T, a3 = x W3^T, h = bf16(silu(a1) * a3), o = h W2^T
 *            with W = E2M1 code * 2^(UE8M0 - 127), one scale per 32 along K;
 *   combine  y[t] = sum_j w[t, j] * o[t, j].
 * The router function, the activation and the nibble order are not fixed by
 * the pages; this library reads them as above (softmax + renormalise,
 * SwiGLU with w1 = gate and w3 = up, low nibble = even K index).
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller unless a
 *    parameter says "host or device".  Layouts are row-major and dense.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls that launch work are asynchronous on that stream; their
 *    status reports argument checks and launch errors only.  Errors found by
 *    kernels (an expert with no slot, a NaN logit, a scale outside the
 *    supported range) are latched in a device error word and reported by
 *    moe_fp4_last_error.  No kernel traps; there is no CPU fallback.
 *  - A context is bound to one device; calls must be made with that device
 *    current.  A context is not thread-safe.
 *
 * Calls: slot_bytes, create, destroy, arena, set_option, profile_read (the
 * context); load_expert_slot, stream_experts, residency_stats (the arena);
 * route, forward, route_forward, last_error (the layer); expert_outputs,
 * combine (the two halves of forward, for expert-parallel use); saliency
 * (per-expert statistic of the last forward); forward_noalloc (forward
 * without any allocation, library-owned static scratch).
 */
#ifndef MOE_FP4_H
#define MOE_FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_fp4_ctx moe_fp4_ctx;

typedef enum {
    MOE_FP4_OK = 0,
    MOE_FP4_EINVAL = 1,   /* bad argument, shape, NaN logit or bad scale byte */
    MOE_FP4_ENOMEM = 2,   /* device allocation failed */
    MOE_FP4_ECUDA = 3,    /* a CUDA runtime call or launch failed */
    MOE_FP4_ESLOT = 4,    /* a routed (layer, expert) has no arena slot */
    MOE_FP4_ETIMEOUT = 5  /* a bounded device-side wait gave up */
} moe_fp4_status;

typedef struct {
    int32_t hidden;      /* H: model width (5120); multiple of 128 */
    int32_t inter;       /* I: expert intermediate width (2304); multiple of 128 */
    int32_t n_experts;   /* E: routed experts per layer (384); <= 1024 */
    int32_t top_k;       /* k: experts per token (6); 1 <= k <= min(E, 32) */
    int32_t n_layers;    /* L: layers addressed by the slot table */
    int32_t n_slots;     /* arena capacity in expert slots */
    int32_t max_tokens;  /* largest T accepted by route / forward */
} moe_fp4_config;

/* Execution-path override for moe_fp4_set_option(MOE_FP4_OPT_PATH, .). */
enum {
    MOE_FP4_PATH_AUTO = 0,  /* decode kernel while 4*T*k < 3*E, tcgen05 GEMM from there on */
    MOE_FP4_PATH_GEMV = 1,  /* always the decode kernel (one persistent block-scaled FP4 tcgen05 kernel; T*k <= 768) */
    MOE_FP4_PATH_TC = 2     /* always the tcgen05 grouped GEMM */
};
/* Options for moe_fp4_set_option. */
enum {
    MOE_FP4_OPT_PATH = 1,          /* value: MOE_FP4_PATH_* */
    MOE_FP4_OPT_PROFILE = 2,       /* value 1: time every kernel with CUDA events */
    MOE_FP4_OPT_WAIT_LIMIT_US = 3  /* value: limit of every bounded device-side wait of the
                                      layer kernels in microseconds (1 .. 10,000,000; 0 restores
                                      the default of 1 s).  A wait that runs out latches
                                      MOE_FP4_ETIMEOUT; the kernel then skips its remaining waits,
                                      lets its copies in flight land and returns (its outputs are
                                      not valid).  The context stays usable. */
};

/*
 * Bytes of one expert slot: 2*(I*H/2 + I*H/32) + (H*I/2 + H*I/32); for the
 * V4.1 shape 18,800,640 (10100.com article, section "moe专家的容量瓶颈").
 * Returns 0 for an invalid config.
 *
 * The checkpoint stores an expert as codes first, scales after (w1, w3, w2
 * codes, then s1, s3, s2; the article's section "SSD读取性能"); the loaders
 * take that layout.  Inside a slot the same bytes are regrouped into units,
 * each one 128-row x 128-K tile of one matrix, codes and scales together,
 * 8,704 contiguous bytes (16-byte aligned) that one bulk copy moves:
 *  up units    for mat in (w1, w3), row tile rt < I/128, K unit ku < H/128,
 *              at ((mat * I/128 + rt) * H/128 + ku) * 8704;
 *  down units  after them, for row tile nt < H/128, K unit ku < I/128,
 *              at up_bytes + (nt * I/128 + ku) * 8704, up_bytes =
 *              2 * (I/128) * (H/128) * 8704;
 *  in a unit   code of row r, K k (0..127): byte (r/8)*512 + (k/32)*128 +
 *              (r%8)*16 + (k%32)/2, nibble k & 1 (low = even K, as in the
 *              checkpoint) -- the tensor cores' K-major, no-swizzle operand
 *              layout for 4-bit types; scale of row r, 32-K block b:
 *              byte 8192 + (r%32)*16 + (r/32)*4 + b -- the tile one
 *              tcgen05.cp .32x128b.warpx4 puts in tensor memory.
 * H and I must be multiples of 128.  The total is unchanged (V4.1: 2,160
 * units).
 */
size_t moe_fp4_slot_bytes(const moe_fp4_config *cfg);

/*
 * Create a context on `device`.
 *  arena:       device pointer to at least n_slots * slot_bytes bytes, 256-byte
 *               aligned, owned by the caller and kept alive until destroy; or
 *               NULL, in which case the library allocates (and frees) it.
 *  arena_bytes: size of a caller arena (ignored when arena is NULL).
 * The library also allocates the slot table (int32 [L][E], every entry -1 =
 * unmapped), a table of each slot's largest scale byte per weight row
 * (n_slots * (2I + H) bytes), a staging buffer of one slot, a workspace sized
 * from max_tokens and a device error word.  On failure *out is NULL and
 * nothing is leaked.
 * Errors: EINVAL (bad config / pointers), ENOMEM, ECUDA.
 */
moe_fp4_status moe_fp4_create(const moe_fp4_config *cfg, int device, void *arena,
                              size_t arena_bytes, moe_fp4_ctx **out);

/* Destroy a context: synchronises the device, frees what the library
 * allocated.  NULL is ignored. */
void moe_fp4_destroy(moe_fp4_ctx *ctx);

/* Device pointer to the base of the arena (caller's or the library's). */
void *moe_fp4_arena(moe_fp4_ctx *ctx);

/* Set an option (MOE_FP4_OPT_PATH, MOE_FP4_OPT_PROFILE).  EINVAL on an
 * unknown option or value.  With profiling on, route and forward record a
 * CUDA event pair around each kernel they launch on the caller's stream (this
 * serialises kernels that would otherwise overlap through programmatic
 * dependent launch). */
moe_fp4_status moe_fp4_set_option(moe_fp4_ctx *ctx, int option, int value);

/*
 * Per-kernel device times of the profiled launches since the last read:
 * synchronises the device, writes up to `max` records (names[i] points at a
 * static string such as "decode_layer" or "tc_up", ms[i] its event-measured duration in
 * milliseconds) and returns the number of records (0 when profiling is off),
 * or -1 on a CUDA error.  Reading clears the record list.
 */
int moe_fp4_profile_read(moe_fp4_ctx *ctx, const char **names, float *ms, int max);

/*
 * Put expert `expert` of layer `layer` into arena slot `slot` and map
 * (layer, expert) -> slot.  The six tensors are in checkpoint layout
 * (10100.com article, section "moe专家的容量瓶颈"): w1/w3 codes uint8
 * [I, H/2] with the even K index in the low nibble, w1/w3 scales UE8M0
 * [I, H/32], w2 codes [H, I/2], w2 scales [H, I/32].  Each pointer may be
 * host or device memory (pageable host memory makes the call block until
 * the copy has been staged).  The copy and re-encode run on `stream`.
 * Whatever was mapped to `slot` before is unmapped; a previous slot of
 * (layer, expert) is released.  slot = -1 only unmaps (layer, expert) and the
 * pointers are ignored.  Supported scale bytes are 2..252 (every value whose
 * block multiplier 2^(s-127) is a normal fp32 number and whose E2M1 multiples
 * are normal bf16 numbers); others latch EINVAL in the error word.  Errors:
 * EINVAL (indices, NULL tensors), ECUDA.
 */
moe_fp4_status moe_fp4_load_expert_slot(moe_fp4_ctx *ctx, int layer, int expert, int slot,
                                        const uint8_t *w1, const uint8_t *w1_scale,
                                        const uint8_t *w3, const uint8_t *w3_scale,
                                        const uint8_t *w2, const uint8_t *w2_scale,
                                        void *stream);

/*
 * Stream experts into a smaller arena (the hot-expert arena of 10100.com
 * article 151357339, section "方案一": a fixed set of slots filled on demand,
 * the least recently used expert making room).  For the n distinct experts of
 * `layer` that one forward needs, experts already resident are hits; each
 * miss takes the lowest-numbered free slot, else the slot whose last request
 * is oldest among those this request does not use (lowest number on ties),
 * evicting its expert (csrc/residency.h).  A miss's object is copied on an
 * internal copy stream into one of two staging buffers, which overlaps with
 * the relayout of the previous miss on `stream`; the relayout (as
 * moe_fp4_load_expert_slot) and the slot-table update run on `stream`, so a
 * forward issued after this call on `stream` sees them.
 *  experts  int32 [n] host: distinct expert ids of `layer`, n <= n_slots.
 *  objects  host array [n] of pointers to contiguous expert objects in
 *           checkpoint layout (w1, w3, w2 codes, s1, s3, s2 scales; pinned
 *           host memory for the copy to be asynchronous, or device memory);
 *           objects[i] may be NULL only when experts[i] is resident.
 *  slots_out int32 [n] host or NULL: the slot of each expert after the call.
 * Work already queued on `stream` that reads an evicted slot is not affected
 * (the relayout runs after it); work on other streams must be ordered by the
 * caller.  Errors: EINVAL (before any change: bad layer, ids, repeated id,
 * n > n_slots, missing object), ENOMEM, ECUDA.
 */
moe_fp4_status moe_fp4_stream_experts(moe_fp4_ctx *ctx, int layer, const int32_t *experts, int n,
                                      const uint8_t *const *objects, int32_t *slots_out, void *stream);

/* Streaming counters since create: stats[0] hits, [1] misses, [2] bytes
 * copied by moe_fp4_stream_experts.  Errors: EINVAL (NULL). */
moe_fp4_status moe_fp4_residency_stats(moe_fp4_ctx *ctx, int64_t *stats);

/*
 * Route T tokens of one layer (one kernel launch).
 *  logits    fp32 [T, E], finite (a NaN latches EINVAL).
 *  keep_mask uint8 [E] or NULL: experts with 0 cannot be chosen (the pruned
 *            arena of 10100.com, section "方案二", where the router may pick
 *            only retained experts).  Fewer than k kept experts latches EINVAL.
 *  ids       int32 [T, k] out: chosen experts, larger logit first, lower index
 *            first on equal logits (-0.0 == +0.0).
 *  weights   fp32 [T, k] out: exp(l_j - l_max) / sum over the chosen k.
 *  counts    int32 [E] out: entries per expert.
 *  offsets   int32 [E+1] out: exclusive prefix sum of counts.
 *  perm      int32 [T*k] out: entry indices t*k+j grouped by expert, ascending
 *            (t, j) inside each expert (a stable counting sort).
 * `layer` is accepted for symmetry with forward and must be in [0, L).
 * T = 0 writes zero counts and offsets.  Above 32 entries (T*k) the launch is
 * cooperative: up to one CTA per SM, which route contiguous token ranges and
 * meet at two bounded grid barriers to group the entries (a barrier that
 * gives up latches ETIMEOUT).  Route calls of one context share those barrier
 * words, so they must not overlap on the GPU (one stream, or ordered streams).
 * Errors: EINVAL, ECUDA; latched EINVAL, ETIMEOUT.
 */
moe_fp4_status moe_fp4_route(moe_fp4_ctx *ctx, int layer, const float *logits,
                             const uint8_t *keep_mask, int T, int32_t *ids, float *weights,
                             int32_t *counts, int32_t *offsets, int32_t *perm, void *stream);

/*
 * Expert FFN and combine for T tokens of `layer`:
 *  x         bf16 [T, H] (uint16 bit patterns), 16-byte aligned.
 *  ids, weights, counts, offsets, perm: as produced by moe_fp4_route.
 *  y         fp32 [T, H] out, 16-byte aligned:
 *            sum_j weights[t, j] * expert_{ids[t,j]}(x[t]).
 *  x_out     bf16 [T, H] out or NULL, 8-byte aligned: bf16_rne(x + y), the
 *            residual update of a stacked layer; may alias x.
 * An entry routed to an expert with no slot contributes zero and latches
 * ESLOT.  Offsets outside [0, T*k] latch EINVAL and that expert contributes
 * nothing; perm entries outside [0, T*k) are skipped, so an invalid grouping
 * gives wrong outputs and an error, never an access outside the buffers.
 * Scratch (digit planes, prescaled x and h rows, per-entry fp32 outputs and
 * the decode kernel's counters) lives in the context's workspace, so calls
 * on one context must not overlap in time.
 * Path: while 4*T*k < 3*E one persistent kernel runs the whole layer on the
 * block-scaled FP4 tensor cores -- w1/w3 with SwiGLU, w2 and, for T <= 16,
 * the combine -- with one CTA per SM launched cooperatively; larger batches
 * run the tcgen05 grouped GEMMs.  MOE_FP4_OPT_PATH overrides the choice.
 * Errors: EINVAL, ECUDA; latched EINVAL, ESLOT, ETIMEOUT.
 */
moe_fp4_status moe_fp4_forward(moe_fp4_ctx *ctx, int layer, const uint16_t *x, int T,
                               const int32_t *ids, const float *weights,
                               const int32_t *counts, const int32_t *offsets,
                               const int32_t *perm, float *y, uint16_t *x_out, void *stream);

/*
 * Route and forward in one call: moe_fp4_route followed by moe_fp4_forward
 * with the same arguments (all outputs of both are written).  For decode
 * batches (T*k <= 64, T <= 16, E <= 384, on the decode path) the routing runs
 * inside the layer kernel -- every CTA routes the tokens itself and the first
 * writes ids, weights, counts, offsets and perm -- so the whole layer is one
 * kernel launch.  Results are identical to the two calls.
 * Errors: EINVAL, ECUDA (as route and forward).
 */
moe_fp4_status moe_fp4_route_forward(moe_fp4_ctx *ctx, int layer, const float *logits,
                                     const uint8_t *keep_mask, const uint16_t *x, int T,
                                     int32_t *ids, float *weights, int32_t *counts, int32_t *offsets,
                                     int32_t *perm, float *y, uint16_t *x_out, void *stream);

/*
 * The expert FFN for an arbitrary list of (row, expert) pairs of `layer`:
 *   o[i] = expert_{experts[i]}(x[i])   (fp32 [n, H], no router weight)
 * This is the work an expert-parallel rank does for the entries other ranks
 * dispatch to the experts it holds (moe_fp4_forward = route + this for every
 * (token, selected expert) pair + moe_fp4_combine).  The entries are grouped
 * by expert with the route kernels' stable grouping, then run on the decode
 * kernel, or on the tcgen05 path when 4n >= 3E (or as
 * MOE_FP4_OPT_PATH forces).
 * Entries are processed in the same per-expert order as moe_fp4_forward
 * processes (token, slot) entries, so listing a forward's entries in
 * (token, slot) order reproduces its per-entry outputs bit for bit.
 *  x        bf16 [n, H] device, 16-byte aligned (row i goes with experts[i]).
 *  experts  int32 [n] device; id -1 marks an empty entry (no work, its row
 *           of o is left unwritten: the expert-parallel exchange pads with
 *           it); any other id outside [0, E) latches EINVAL and its row of o
 *           is left unwritten.
 *  o        fp32 [n, H] device out, 16-byte aligned.
 * n <= max_tokens * top_k; uses the context's workspace like forward.
 * Errors: EINVAL, ECUDA; unmapped experts latch ESLOT (their rows are zero).
 */
moe_fp4_status moe_fp4_expert_outputs(moe_fp4_ctx *ctx, int layer, const uint16_t *x, int n,
                                      const int32_t *experts, float *o, void *stream);

/*
 * The combine step alone: y[t] = sum over j < k of weights[t, j] * o[t*k + j]
 * (fixed j order, fp32), and x_out = bf16_rne(x + y) when x_out is not NULL
 * (x_out may alias x).  o fp32 [T*k, H] and y fp32 [T, H] 16-byte aligned;
 * x, x_out bf16 [T, H] 8-byte aligned.  T <= max_tokens.  Errors: EINVAL,
 * ECUDA.
 */
moe_fp4_status moe_fp4_combine(moe_fp4_ctx *ctx, int T, const float *o, const float *weights,
                               const uint16_t *x, float *y, uint16_t *x_out, void *stream);

/*
 * Expert saliency of the last forward (10100.com article 151357339, section
 * "选哪些专家：频率 vs Saliency": router weight times the L2 norm of the
 * expert's output, summed over a corpus, used to rank experts for pruning):
 *   saliency[e] += sum over the entries p = t*k + j routed to e of
 *                  weights[p] * ||o_p||_2
 * where o_p is expert ids[p]'s fp32 output row for token t, as the last
 * moe_fp4_forward on this context left it in the workspace.  Call it on the
 * same stream after that forward (same T, weights, offsets, perm) and before
 * the next forward on the context.  Norms are fp32 sums in a fixed order;
 * each expert's entries are added in grouped (perm) order in fp64, and each
 * expert's total is added once to saliency[e], so the result does not depend
 * on the schedule.  Experts without entries are left unchanged.
 *  weights   fp32 [T, k], offsets int32 [E+1], perm int32 [T*k]: device.
 *  saliency  fp64 [E] device accumulator, owned by the caller (zero it to
 *            start a corpus).
 * T = 0 does nothing.  Errors: EINVAL (bad T or NULL pointer), ECUDA.
 */
moe_fp4_status moe_fp4_saliency(moe_fp4_ctx *ctx, int T, const float *weights,
                                const int32_t *offsets, const int32_t *perm,
                                double *saliency, void *stream);

/*
 * Synchronise the device, read and clear the device error word.  Returns the
 * first latched status (OK if none) and writes a one-line description into
 * msg (n bytes, may be NULL).  Host-side errors of the last failing call are
 * reported too.
 */
moe_fp4_status moe_fp4_last_error(moe_fp4_ctx *ctx, char *msg, size_t n);

/*
 * Forward without any allocation: the same decode kernel as moe_fp4_forward
 * (the whole layer in one launch: both expert GEMMs on the block-scaled FP4
 * tensor cores, SwiGLU, combine), for callers that cannot call cudaMalloc --
 * for example a plugin inside a host framework that owns all device memory
 * and forbids allocation on its execution path, or code that runs where the
 * CUDA allocator must not be entered.  This call has no counterpart on the
 * pages: it is a deployment variant of this library.
 *
 * Nothing is allocated and no context is used.  The caller passes every input
 * and output; the forward's scratch lives in one library-owned, file-scope
 * device array of 16 MiB (16,777,216 bytes) that every GPU which loads the
 * library holds until the process exits.  It starts with a fixed header of
 * 656,640 bytes (the kernel's launch sequence number, 1 KB of zeros, up to
 * 32,768 up-item flags and two banks of 65,536 counters, all zero at load and
 * kept consistent by every launch), followed by the per-call buffers: the digit
 * planes of x and h with their scales, split-item partial sums and fp32
 * per-entry outputs.  With KU = H/128, KD = I/128 and S the device's SM count
 * the scratch must hold
 *   656640 + T*KU*512 + T*KU*128 + T*k*KD*512 + T*k*KD*128 + S*6144 + T*k*H*4
 * bytes (each of the five middle parts rounded up to 256), and the batch's
 * work items must fit the header (max_gs*(I/128) flags and
 * 1 + max_gs*(I/128 + H/128) + H/128 counters per bank, max_gs = min(T*k, min(E, T*k)
 * + T*k/2)); a larger T, or a shape the decode kernel does not take, returns
 * EINVAL before any launch.  For the V4.1 shape (k = 6) on a 148-SM B200 that
 * allows T <= 69.  Up to 16 tokens the combine runs inside the kernel, above
 * that a second kernel.
 *
 * Every call, on every stream, shares that array and leaves the last call's
 * contents in it.  Calls whose executions overlap on the GPU race on it:
 * serialise them (one stream, or events).  The first call on a device looks
 * up the array's device address with cudaGetSymbolAddress (once per device,
 * that device current); make that first call before any stream capture.
 *
 *  cfg         the layer shape (as for moe_fp4_create; n_slots and max_tokens
 *              only bound the indices used).
 *  arena       device, n_slots slots of moe_fp4_slot_bytes(cfg) bytes in the
 *              library's slot layout (as filled by moe_fp4_load_expert_slot,
 *              e.g. the arena of a context created elsewhere), 256-byte aligned.
 *  slot_table  device int32 [n_layers][E]: slot of (layer, expert) or -1.
 *  x, weights, offsets, perm, y, x_out, T, layer: as for moe_fp4_forward
 *              (ids and counts are not needed); weights 4-byte aligned.
 *  err         device int32 [4] or NULL: first error latched by the kernel
 *              ([0] status, [1] detail), as moe_fp4_last_error reports them;
 *              the caller clears it.  With NULL, kernel-found errors are
 *              dropped.
 * Errors: EINVAL (arguments, T beyond the limits), ECUDA.
 */
moe_fp4_status moe_fp4_forward_noalloc(const moe_fp4_config *cfg, const uint8_t *arena,
                                       const int32_t *slot_table, int layer, const uint16_t *x,
                                       int T, const float *weights, const int32_t *offsets,
                                       const int32_t *perm, float *y, uint16_t *x_out,
                                       int32_t *err, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_FP4_H */
