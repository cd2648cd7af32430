/*
 * oracle.c -- plain, slow CPU reference of the routed-expert FP4 FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the tests, the package's smoke check and the bench's
 * CPU-baseline leg do.  It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes (every step in fp64 unless a rounding is stated):
 *
 *  - Expert storage (10100.com article 151357339, section
 *    "moe专家的容量瓶颈"): each routed expert holds w1, w2, w3; the checkpoint
 *    stores them as FP4 E2M1 codes, two per byte, plus UE8M0 scales:
 *    w1/w3 codes [2304,2560] + scales [2304,160], w2 codes [5120,1152] +
 *    scales [5120,72]; 18,800,640 bytes per expert.  The shapes fix one scale
 *    per 32 consecutive K values (5120/32 = 160, 2304/32 = 72) along each
 *    weight row, rows = output features.  The page only names the formats;
 *    E2M1 and UE8M0 follow the OCP Microscaling (MX) v1.0 definitions.
 *    Which nibble holds the even K index is not stated: the low nibble does.
 *  - Router (same section; 6 of 384 experts per token per layer): the page
 *    does not give the router function.  The reading used here is a softmax
 *    over fp32 logits, the top-k under the total order (larger logit first,
 *    lower expert index on ties), renormalised over the chosen k.  Experts
 *    outside a layer's keep mask cannot be chosen (section "方案二": the
 *    router may only pick the retained experts).
 *  - Token grouping by expert (ai-shiz.ru "DeepSeek-V4.1-Flash дома",
 *    trick 4: in prefill one read of an expert serves many tokens): counts
 *    per expert, exclusive offsets, and the (token, slot) entries listed per
 *    expert in ascending (token, slot) order.
 *  - Expert FFN: the page names w1/w2/w3 but not the activation; SwiGLU is
 *    the reading: a1 = x.W1^T, a3 = x.W3^T, h = bf16_rne(silu(a1) * a3),
 *    o = h.W2^T, silu(z) = z / (1 + exp(-z)).
 *  - Combine: y[t] = sum_j w[t,j] * o[t,j], j in selection order (the
 *    article's saliency, router weight x expert output, section
 *    "选哪些专家：频率 vs Saliency", implies the router-weighted sum).
 *  - Residual between stacked layers: x <- bf16_rne(x + y).
 *  - Expert saliency (10100.com article 151357339, section
 *    "选哪些专家：频率 vs Saliency": router weight times the L2 norm of the
 *    expert's output, summed over the tokens of a corpus):
 *    S[e] += sum over (t, j) with ids[t,j] = e of w[t,j] * ||o_{t,j}||_2,
 *    o_{t,j} the expert's output row for token t as in the FFN above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <fenv.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ formats */

/* E2M1 (OCP MX v1.0, FP4): bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa.  Exponent field 0 is subnormal: value = mantissa * 2^(1-1) * 0.5. */
double oracle_e2m1(unsigned code)
{
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

/* UE8M0 (OCP MX v1.0): unsigned 8-bit exponent, bias 127, no mantissa.
 * 0xFF encodes NaN; the generators never emit it. */
double oracle_ue8m0(unsigned e)
{
    if ((e & 0xFFu) == 0xFFu) return NAN;
    return ldexp(1.0, (int)(e & 0xFFu) - 127);
}

double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round an fp64 value to bfloat16, nearest with ties to even, in one step
 * (no intermediate fp32 rounding).  bfloat16: 8 significant bits, exponent
 * range of fp32, subnormals with quantum 2^-133. */
uint16_t oracle_bf16_rne(double v)
{
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                  /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 8;                 /* quantum of an 8-significant-bit value */
    if (q < -133) q = -133;        /* subnormal range */
    int old = fegetround();
    fesetround(FE_TONEAREST);
    double r = nearbyint(ldexp(a, -q));
    fesetround(old);
    double rv = ldexp(r, q);
    if (rv > 3.3895313892515355e38)  /* above the largest finite bf16 */
        return (uint16_t)(sign | 0x7F80);
    float f = (float)rv;           /* exact: rv has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

/* ------------------------------------------------------------- shape pins */

/* Bytes of one expert object for hidden size H and expert intermediate I:
 * codes hold two values per byte, scales one byte per 32 values along K. */
long long oracle_expert_bytes(int H, int I)
{
    long long w13 = 2LL * ((long long)I * (H / 2) + (long long)I * (H / 32));
    long long w2 = (long long)H * (I / 2) + (long long)H * (I / 32);
    return w13 + w2;
}

/* Weight element W[n][k] of a [rows, K] matrix stored as codes [rows, K/2]
 * and scales [rows, K/32]: E2M1 value of nibble (k & 1) of byte k/2 (low
 * nibble = even k) times 2^(scale - 127) of block k/32. */
static double weight_at(const uint8_t *codes, const uint8_t *scales, int K, int n, int k)
{
    uint8_t byte = codes[(size_t)n * (K / 2) + (k >> 1)];
    unsigned nib = (k & 1) ? (byte >> 4) : (byte & 0xF);
    return oracle_e2m1(nib) * oracle_ue8m0(scales[(size_t)n * (K / 32) + (k >> 5)]);
}

/* Dense fp64 copy of a whole matrix (used by tests on small shapes). */
void oracle_dequant(const uint8_t *codes, const uint8_t *scales, int rows, int K, double *out)
{
    for (int n = 0; n < rows; ++n)
        for (int k = 0; k < K; ++k)
            out[(size_t)n * K + k] = weight_at(codes, scales, K, n, k);
}

/* ------------------------------------------------------------------ router */

/* a ranks before b: larger logit, ties to the lower index (-0 == +0). */
static int ranks_before(float va, int ia, float vb, int ib)
{
    if (va > vb) return 1;
    if (va < vb) return 0;
    return ia < ib;
}

/*
 * Top-k routing of T tokens over E experts.  logits [T,E] fp32, keep [E]
 * (NULL = all experts routable).  Writes ids [T,k] in rank order and the
 * renormalised softmax weights w [T,k] in fp64:
 *   w_j = exp(l_j - l_max) / sum_{i chosen} exp(l_i - l_max).
 * Selection is a full insertion ranking of every routable expert, then the
 * first k.  Returns 0, or -1 if a logit is NaN or fewer than k experts are
 * routable.
 */
int oracle_route(const float *logits, const uint8_t *keep, int T, int E, int k,
                 int32_t *ids, double *w)
{
    int *order = (int *)malloc(sizeof(int) * (size_t)E);
    if (!order) return -2;
    int rc = 0;
    for (int t = 0; t < T && rc == 0; ++t) {
        const float *l = logits + (size_t)t * E;
        int n = 0;
        for (int e = 0; e < E; ++e) {
            if (isnan(l[e])) { rc = -1; break; }
            if (keep && !keep[e]) continue;
            /* insert e into the ranked list order[0..n) */
            int p = n;
            while (p > 0 && ranks_before(l[e], e, l[order[p - 1]], order[p - 1])) {
                order[p] = order[p - 1];
                --p;
            }
            order[p] = e;
            ++n;
        }
        if (rc) break;
        if (n < k) { rc = -1; break; }
        double lmax = (double)l[order[0]], den = 0.0;
        for (int j = 0; j < k; ++j) den += exp((double)l[order[j]] - lmax);
        for (int j = 0; j < k; ++j) {
            ids[(size_t)t * k + j] = order[j];
            w[(size_t)t * k + j] = exp((double)l[order[j]] - lmax) / den;
        }
    }
    free(order);
    return rc;
}

/* Group the T*k routing entries by expert.  counts[E], offsets[E+1]
 * (exclusive prefix sum), perm[T*k]: entries t*k+j listed expert by expert,
 * ascending (t, j) inside each expert. */
void oracle_permute(const int32_t *ids, int T, int k, int E,
                    int32_t *counts, int32_t *offsets, int32_t *perm)
{
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int i = 0; i < T * k; ++i) counts[ids[i]]++;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    for (int i = 0; i < T * k; ++i) perm[fill[ids[i]]++] = i;
    free(fill);
}

/* -------------------------------------------------------------- expert FFN */

typedef struct {
    const uint8_t *w1, *s1, *w3, *s3, *w2, *s2;
} expert_ptrs;

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One (token, expert) pair.  x [H] bf16 bits.  h_out [I] bf16 bits (may be
 * NULL), o [H] fp64. */
static void expert_ffn(const uint16_t *x, int H, int I, const expert_ptrs *ep,
                       uint16_t *h_out, double *o)
{
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *hd = (double *)malloc(sizeof(double) * (size_t)I);
    for (int k = 0; k < H; ++k) xd[k] = oracle_bf16_to_double(x[k]);
    for (int n = 0; n < I; ++n) {
        double a1 = 0.0, a3 = 0.0;
        for (int k = 0; k < H; ++k) {
            a1 += xd[k] * weight_at(ep->w1, ep->s1, H, n, k);
            a3 += xd[k] * weight_at(ep->w3, ep->s3, H, n, k);
        }
        uint16_t hb = oracle_bf16_rne(silu(a1) * a3);
        if (h_out) h_out[n] = hb;
        hd[n] = oracle_bf16_to_double(hb);
    }
    for (int n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += hd[i] * weight_at(ep->w2, ep->s2, I, n, i);
        o[n] = acc;
    }
    free(xd);
    free(hd);
}

void oracle_expert_ffn(const uint16_t *x, int H, int I,
                       const uint8_t *w1, const uint8_t *s1,
                       const uint8_t *w3, const uint8_t *s3,
                       const uint8_t *w2, const uint8_t *s2,
                       uint16_t *h_out, double *o)
{
    expert_ptrs ep = {w1, s1, w3, s3, w2, s2};
    expert_ffn(x, H, I, &ep, h_out, o);
}

/*
 * MoE layer output for T tokens.  x [T,H] bf16 bits; ids/w [T,k] from
 * oracle_route; objs[e] points at expert e's object in checkpoint layout
 * (w1, w3, w2 codes then s1, s3, s2 scales, contiguous), NULL if the expert
 * is not supplied (a token routed to a missing expert is an error, -1).
 * y [T,H] fp64 = sum_j w[t,j] * o(t, ids[t,j]).  The (t, j) pairs are
 * independent, so they run on n_threads OpenMP threads (<= 0: default).
 */
int oracle_moe_forward(const uint16_t *x, int T, int H, int I, int E, int k,
                       const int32_t *ids, const double *w,
                       const uint8_t *const *objs, int n_threads, double *y)
{
    size_t w13 = (size_t)I * (H / 2), w2b = (size_t)H * (I / 2);
    size_t s13 = (size_t)I * (H / 32);
    for (int i = 0; i < T * k; ++i)
        if (ids[i] < 0 || ids[i] >= E || !objs[ids[i]]) return -1;
    double *o = (double *)malloc(sizeof(double) * (size_t)T * k * H);
    if (!o) return -2;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int p = 0; p < T * k; ++p) {
        const uint8_t *b = objs[ids[p]];
        expert_ptrs ep = {b, b + 2 * w13 + w2b, b + w13, b + 2 * w13 + w2b + s13,
                          b + 2 * w13, b + 2 * w13 + w2b + 2 * s13};
        expert_ffn(x + (size_t)(p / k) * H, H, I, &ep, NULL, o + (size_t)p * H);
    }
    for (int t = 0; t < T; ++t)
        for (int n = 0; n < H; ++n) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += w[(size_t)t * k + j] * o[((size_t)t * k + j) * H + n];
            y[(size_t)t * H + n] = acc;
        }
    free(o);
    return 0;
}

/* Saliency accumulation: sal[e] += sum over entries p = t*k + j routed to e of
 * w[p] * ||o_p||_2, o_p = expert ids[p]'s output for token t (fp64 throughout).
 * Same expert layout and error codes as oracle_moe_forward. */
int oracle_moe_saliency(const uint16_t *x, int T, int H, int I, int E, int k,
                        const int32_t *ids, const double *w,
                        const uint8_t *const *objs, int n_threads, double *sal)
{
    size_t w13 = (size_t)I * (H / 2), w2b = (size_t)H * (I / 2);
    size_t s13 = (size_t)I * (H / 32);
    for (int i = 0; i < T * k; ++i)
        if (ids[i] < 0 || ids[i] >= E || !objs[ids[i]]) return -1;
    double *norm = (double *)malloc(sizeof(double) * (size_t)(T * k > 0 ? T * k : 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)(T * k > 0 ? T * k : 1) * H);
    if (!norm || !o) {
        free(norm);
        free(o);
        return -2;
    }
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int p = 0; p < T * k; ++p) {
        const uint8_t *b = objs[ids[p]];
        expert_ptrs ep = {b, b + 2 * w13 + w2b, b + w13, b + 2 * w13 + w2b + s13,
                          b + 2 * w13, b + 2 * w13 + w2b + 2 * s13};
        double *op = o + (size_t)p * H;
        expert_ffn(x + (size_t)(p / k) * H, H, I, &ep, NULL, op);
        double ss = 0.0;
        for (int n = 0; n < H; ++n) ss += op[n] * op[n];
        norm[p] = sqrt(ss);
    }
    for (int p = 0; p < T * k; ++p) sal[ids[p]] += w[p] * norm[p];
    free(norm);
    free(o);
    return 0;
}

/* Residual update between stacked layers: x <- bf16_rne(x + y). */
void oracle_residual(uint16_t *x, const double *y, size_t n)
{
    for (size_t i = 0; i < n; ++i) x[i] = oracle_bf16_rne(oracle_bf16_to_double(x[i]) + y[i]);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
