/*
 * logo_oracle.c -- plain, slow fp64 CPU oracle for the forward pass of
 * token-level dynamic local-global attention (LoGo / L2A).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may link,
 * load or call this file: it exists so that the tests, the smoke check and the
 * benchmark's CPU-baseline leg can compare the CUDA kernels against a
 * definition a reader can check by eye.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes (sources are the pages' titles and sections):
 *   - "LoGo: Token-Level Dynamic Local-Global Attention", Abstract: each
 *     layer pairs a windowed branch, run for every token, with a whole-prefix
 *     branch that a gate switches on per token; the share of switched-on
 *     tokens is held at a set fraction.
 *   - "Learning When to Attend", section "The Architecture of Conditional
 *     Attention": the windowed pass runs for all positions; the unrestricted
 *     pass is exact softmax attention, run only at the chosen positions.
 *   - "Local-global attention", Variants, "Alternating sliding-window and
 *     global layers (Gemma 2)": both kinds are causal; the windowed kind
 *     ignores keys that lie further back than the window.
 *   - "Local-global attention", Implementation sketch, notes, "Packed examples
 *     (LongT5)": packed examples must not attend to one another.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   window      key j is in the local window of query i iff 0 <= i - j < W
 *               (W keys including the query itself);
 *   budget      k = ceil(ratio * len) per sequence (with fp noise snapped, see
 *               oracle_num_selected), chosen as the k largest gate logits,
 *               ties to the lower index, -0 equal to +0, NaN below -inf;
 *               one selection per sequence, shared by every head;
 *   global      exact causal attention over positions 0..i of the sequence;
 *   merge       o_i = local_i + sigmoid(g_i) * global_i for selected i,
 *               o_i = local_i otherwise;
 *   scale       softmax scale 1/sqrt(d) unless the caller passes scale > 0;
 *   GQA         query head h reads key/value head h / (Hq / Hkv).
 *
 * Precision: inputs are bf16 (passed as raw uint16 bit patterns) and gate
 * logits fp32; both are widened exactly to double, and every sum, max,
 * exponential and division is done in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- scalar helpers --------------------------------------------------- */

/* bf16 -> double, exact: a bf16 value is the top half of an fp32 value. */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/*
 * Budget: the number of query tokens that take the global branch in a
 * sequence of `len` tokens at ratio `ratio` ("LoGo", Abstract: the share of
 * tokens on the global branch is held at a set value; "Learning When to
 * Attend", "The Architecture of Conditional Attention": about one token in
 * five).
 * Reading: k = ceil(ratio * len).  The product is formed in double; when it
 * lies within 1e-9 (relative, at least absolute 1e-9) of an integer it is
 * taken as that integer, so that 0.07 * 100 = 7.000000000000001 gives 7, not 8.
 * The result is clamped to [0, len].
 */
int64_t oracle_num_selected(double ratio, int64_t len)
{
    if (len <= 0 || !(ratio > 0.0)) return 0;
    double x = ratio * (double)len;
    double r = nearbyint(x);
    double tol = 1e-9 * (x > 1.0 ? x : 1.0);
    double kk = (fabs(x - r) <= tol) ? r : ceil(x);
    if (kk < 0.0) kk = 0.0;
    if (kk > (double)len) kk = (double)len;
    return (int64_t)kk;
}

/* ---- selection -------------------------------------------------------- */

typedef struct {
    float g;
    int32_t idx;
} gate_item;

/*
 * Order used by the budget rule: larger logit first; equal logits (and -0 vs
 * +0, which compare equal as floats) by lower index; NaN after every number,
 * NaNs among themselves by lower index.
 */
static int gate_order(const void *pa, const void *pb)
{
    const gate_item *a = (const gate_item *)pa;
    const gate_item *b = (const gate_item *)pb;
    int a_nan = isnan(a->g), b_nan = isnan(b->g);
    if (a_nan != b_nan) return a_nan ? 1 : -1;
    if (!a_nan) {
        if (a->g > b->g) return -1;
        if (a->g < b->g) return 1;
    }
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx ? 1 : 0);
}

static int ascending_i32(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * Select the k = oracle_num_selected(ratio, len) tokens of one sequence:
 * sort all positions by the order above, keep the first k, and return them
 * in ascending position order.  `out` holds at least k entries.  Returns k.
 */
int64_t oracle_select(const float *g, int64_t len, double ratio, int32_t *out)
{
    int64_t k = oracle_num_selected(ratio, len);
    if (k == 0) return 0;
    gate_item *items = (gate_item *)malloc(sizeof(gate_item) * (size_t)len);
    for (int64_t i = 0; i < len; ++i) {
        items[i].g = g[i];
        items[i].idx = (int32_t)i;
    }
    qsort(items, (size_t)len, sizeof(gate_item), gate_order);
    for (int64_t i = 0; i < k; ++i) out[i] = items[i].idx;
    free(items);
    qsort(out, (size_t)k, sizeof(int32_t), ascending_i32);
    return k;
}

/* ---- attention for one query row -------------------------------------- */

/*
 * Exact softmax attention of one query row over the keys j_lo..j_hi
 * (inclusive) of one key/value head:
 *   s_j = scale * <q, k_j>,  w_j = exp(s_j - max_j s_j),
 *   out = sum_j w_j v_j / sum_j w_j.
 * `q`, `kh`, `vh` point at the query row and at row 0 of the key and value
 * sequences; rows are d elements apart.  `s` is scratch for j_hi - j_lo + 1
 * doubles.
 */
static void attend_row(const uint16_t *q, const uint16_t *kh, const uint16_t *vh,
                       int64_t j_lo, int64_t j_hi, int d, double scale,
                       double *s, double *out)
{
    int64_t n = j_hi - j_lo + 1;
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t *kr = kh + (j_lo + t) * (int64_t)d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += bf16_bits_to_double(q[c]) * bf16_bits_to_double(kr[c]);
        s[t] = scale * dot;
        if (s[t] > m) m = s[t];
    }
    double den = 0.0;
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        double w = exp(s[t] - m);
        den += w;
        const uint16_t *vr = vh + (j_lo + t) * (int64_t)d;
        for (int c = 0; c < d; ++c) out[c] += w * bf16_bits_to_double(vr[c]);
    }
    for (int c = 0; c < d; ++c) out[c] /= den;
}

/* ---- problem geometry ------------------------------------------------- */

/*
 * Tensors are [B, H, L, d] (fixed length, cu_seqlens == NULL, nseq == B), or
 * packed [1, H, T, d] with sequence s at rows cu_seqlens[s] .. cu_seqlens[s+1]
 * of every head (varlen, B == 1, L == T).
 */
typedef struct {
    const uint16_t *q, *k, *v;
    const float *g;
    const int32_t *cu_seqlens;
    int nseq, Hq, Hkv, d;
    int64_t L; /* rows per head slab: L (fixed) or T (varlen) */
    int64_t W;
    double scale;
} problem;

static int64_t seq_start(const problem *p, int s)
{
    return p->cu_seqlens ? (int64_t)p->cu_seqlens[s] : 0;
}

static int64_t seq_len(const problem *p, int s)
{
    return p->cu_seqlens ? (int64_t)(p->cu_seqlens[s + 1] - p->cu_seqlens[s]) : p->L;
}

/* Pointer to row `row` (absolute within the slab) of head `h` of batch `b`. */
static const uint16_t *row_ptr(const uint16_t *base, int64_t b, int64_t H, int64_t h,
                               int64_t L, int64_t row, int d)
{
    return base + (((b * H + h) * L) + row) * (int64_t)d;
}

/*
 * One output row: sequence s, query head h, position i (relative to the
 * sequence start).  Writes the local row, and, if `want_global`, the global
 * row.  Either output pointer may be NULL.
 */
static void compute_row(const problem *p, int s, int h, int64_t i, int want_global,
                        double *scratch, double *loc, double *glo)
{
    int G = p->Hq / p->Hkv;
    int hk = h / G;
    int64_t b = p->cu_seqlens ? 0 : s;
    int64_t s0 = seq_start(p, s);
    const uint16_t *qr = row_ptr(p->q, b, p->Hq, h, p->L, s0 + i, p->d);
    const uint16_t *kh = row_ptr(p->k, b, p->Hkv, hk, p->L, s0, p->d);
    const uint16_t *vh = row_ptr(p->v, b, p->Hkv, hk, p->L, s0, p->d);
    if (loc) {
        int64_t j_lo = i - p->W + 1;
        if (j_lo < 0) j_lo = 0;
        attend_row(qr, kh, vh, j_lo, i, p->d, p->scale, scratch, loc);
    }
    if (want_global && glo) attend_row(qr, kh, vh, 0, i, p->d, p->scale, scratch, glo);
}

static double default_scale(double scale, int d) { return scale > 0.0 ? scale : 1.0 / sqrt((double)d); }

/* ---- public entry points ---------------------------------------------- */

/*
 * Full forward pass.
 *   out        [B, Hq, L, d] doubles: the merged output o.
 *   out_local  (may be NULL) [B, Hq, L, d]: the local branch for every row.
 *   out_global (may be NULL) [B, Hq, L, d]: the global branch on selected
 *              rows, 0 elsewhere.
 *   sel_idx    the selected positions, sequence after sequence, each
 *              sequence ascending; capacity sum_s k_s.
 *   cu_sel     [nseq + 1] offsets of each sequence's list in sel_idx.
 * Returns the total number of selected tokens.
 */
int64_t oracle_forward(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                       const int32_t *cu_seqlens, int nseq, int Hq, int Hkv, int64_t L, int d,
                       int64_t W, double ratio, double scale, double *out, double *out_local,
                       double *out_global, int32_t *sel_idx, int32_t *cu_sel)
{
    problem p = {q, k, v, g, cu_seqlens, nseq, Hq, Hkv, d, L, W, default_scale(scale, d)};
    int64_t B = cu_seqlens ? 1 : nseq;
    int64_t total_rows = B * (int64_t)Hq * L;

    /* Selection, one sequence at a time; the flag marks selected rows. */
    unsigned char *flag = (unsigned char *)calloc((size_t)(B * L), 1);
    int64_t off = 0;
    cu_sel[0] = 0;
    for (int s = 0; s < nseq; ++s) {
        int64_t b = cu_seqlens ? 0 : s;
        int64_t s0 = seq_start(&p, s), len = seq_len(&p, s);
        int64_t ks = oracle_select(g + b * L + s0, len, ratio, sel_idx + off);
        for (int64_t t = 0; t < ks; ++t) flag[b * L + s0 + sel_idx[off + t]] = 1;
        off += ks;
        cu_sel[s + 1] = (int32_t)off;
    }

    memset(out, 0, sizeof(double) * (size_t)(total_rows * d));
    if (out_local) memset(out_local, 0, sizeof(double) * (size_t)(total_rows * d));
    if (out_global) memset(out_global, 0, sizeof(double) * (size_t)(total_rows * d));

    /* Every (sequence, head, position) row is independent. */
    for (int s = 0; s < nseq; ++s) {
        int64_t b = cu_seqlens ? 0 : s;
        int64_t s0 = seq_start(&p, s), len = seq_len(&p, s);
#pragma omp parallel
        {
            double *scratch = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
            double *loc = (double *)malloc(sizeof(double) * (size_t)d);
            double *glo = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 16) collapse(2)
            for (int h = 0; h < Hq; ++h) {
                for (int64_t i = 0; i < len; ++i) {
                    int sel = flag[b * L + s0 + i];
                    compute_row(&p, s, h, i, sel, scratch, loc, glo);
                    double gs = sel ? sigmoid((double)g[b * L + s0 + i]) : 0.0;
                    int64_t r = ((b * Hq + h) * L + s0 + i) * (int64_t)d;
                    for (int c = 0; c < d; ++c) {
                        out[r + c] = loc[c] + (sel ? gs * glo[c] : 0.0);
                        if (out_local) out_local[r + c] = loc[c];
                        if (out_global && sel) out_global[r + c] = glo[c];
                    }
                }
            }
            free(scratch);
            free(loc);
            free(glo);
        }
    }
    free(flag);
    return off;
}

/*
 * A sample of rows, for problems too large to run whole.  Row t is
 * (seq[t], head[t], pos[t]) with pos relative to the sequence start;
 * selected[t] says whether that position is in the sequence's selection
 * (taken from oracle_select by the caller).  Writes d doubles per row into
 * each non-NULL output: the local branch, the global branch (0 when not
 * selected) and the merged output.
 */
void oracle_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                 const int32_t *cu_seqlens, int nseq, int Hq, int Hkv, int64_t L, int d, int64_t W,
                 double scale, int64_t n, const int32_t *seq, const int32_t *head,
                 const int64_t *pos, const unsigned char *selected, double *out_local,
                 double *out_global, double *out)
{
    problem p = {q, k, v, g, cu_seqlens, nseq, Hq, Hkv, d, L, W, default_scale(scale, d)};
    int64_t maxlen = 1;
    for (int s = 0; s < nseq; ++s)
        if (seq_len(&p, s) > maxlen) maxlen = seq_len(&p, s);
#pragma omp parallel
    {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)maxlen);
        double *loc = (double *)malloc(sizeof(double) * (size_t)d);
        double *glo = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n; ++t) {
            int s = seq[t];
            int64_t b = cu_seqlens ? 0 : s;
            int sel = selected[t] != 0;
            compute_row(&p, s, head[t], pos[t], sel, scratch, loc, glo);
            double gs = sel ? sigmoid((double)g[b * L + seq_start(&p, s) + pos[t]]) : 0.0;
            for (int c = 0; c < d; ++c) {
                if (out_local) out_local[t * d + c] = loc[c];
                if (out_global) out_global[t * d + c] = sel ? glo[c] : 0.0;
                if (out) out[t * d + c] = loc[c] + (sel ? gs * glo[c] : 0.0);
            }
        }
        free(scratch);
        free(loc);
        free(glo);
    }
}

/* ---- threshold form of the budget rule -------------------------------- */

/*
 * "LoGo: Token-Level Dynamic Local-Global Attention", Abstract: the budget is
 * kept by a controller that moves a threshold on the gate, rather than by a
 * fixed count.  Readings used here (the pages give no formula):
 *   selection   a token takes the global branch iff its logit is strictly
 *               greater than the threshold tau (NaN logits never do; a NaN
 *               tau selects nothing);
 *   target      for n logits (the whole batch) and ratio r, with
 *               k = oracle_num_selected(r, n), the target threshold is the
 *               (k+1)-th largest logit in the selection order (so that, without
 *               ties, exactly k logits lie above it); -inf when k = n; a NaN
 *               in that place also gives -inf;
 *   update      tau' = tau + beta * (q - tau), each operation rounded to fp32,
 *               and tau' = q when tau or q is not finite.
 */

/* Ascending positions i < len with g[i] > tau; returns their count. */
int64_t oracle_threshold_select(const float *g, int64_t len, float tau, int32_t *out)
{
    int64_t n = 0;
    for (int64_t i = 0; i < len; ++i)
        if (g[i] > tau) out[n++] = (int32_t)i; /* false for NaN on either side */
    return n;
}

/* The controller's target threshold for n logits at ratio r (see above). */
float oracle_threshold_target(const float *g, int64_t n, double ratio)
{
    int64_t k = oracle_num_selected(ratio, n);
    if (k >= n) return -INFINITY;
    gate_item *items = (gate_item *)malloc(sizeof(gate_item) * (size_t)n);
    for (int64_t i = 0; i < n; ++i) {
        items[i].g = g[i];
        items[i].idx = (int32_t)i;
    }
    qsort(items, (size_t)n, sizeof(gate_item), gate_order);
    float q = items[k].g; /* the (k+1)-th in the selection order */
    free(items);
    return isnan(q) ? -INFINITY : q;
}

/* One controller step, fp32 arithmetic with a rounding after each operation. */
float oracle_threshold_update(float tau, float q, float beta)
{
    if (!isfinite(tau) || !isfinite(q)) return q;
    volatile float diff = q - tau;
    volatile float step = beta * diff;
    volatile float out = tau + step;
    return out;
}

/* ---- decode: one new query per sequence against a key/value cache ------ */

/*
 * Decode step ("Learning When to Attend", "Empirical Validation and System
 * Optimization": the savings carry over to time-to-first-token and
 * generation; "LoGo", Abstract: the gate decides per token).  Readings: the
 * new token of sequence b sits at position t = cache_len[b] - 1 of the cache
 * (its key and value already written there); its local branch attends over
 * positions max(0, t - W + 1) .. t; it takes the global branch iff its gate
 * logit is strictly greater than the threshold tau (the threshold form of the
 * budget rule), and then attends over 0 .. t; o = local + sigmoid(g) * global.
 *   q        [B, Hq, d] bf16 bits;  k, v [B, Hkv, Lmax, d] bf16 bits.
 *   out      [B, Hq, d] doubles;  out_local / out_global may be NULL
 *            (out_global is 0 for tokens that do not take the global branch).
 *   selected [B] 0/1 (may be NULL).
 * Returns the number of tokens that took the global branch.
 */
int64_t oracle_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *cache_len,
                      const float *g, float tau, int B, int Hq, int Hkv, int64_t Lmax, int d, int64_t W,
                      double scale, double *out, double *out_local, double *out_global, int32_t *selected)
{
    scale = default_scale(scale, d);
    int G = Hq / Hkv;
    int64_t n_sel = 0;
    for (int b = 0; b < B; ++b) {
        int sel = (g[b] > tau) ? 1 : 0; /* false for NaN on either side */
        if (selected) selected[b] = sel;
        n_sel += sel;
    }
    /* every (sequence, head) row is independent */
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        double *loc = (double *)malloc(sizeof(double) * (size_t)d);
        double *glo = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
            int b = (int)(bh / Hq), h = (int)(bh % Hq);
            int64_t t = (int64_t)cache_len[b] - 1;
            int sel = (g[b] > tau) ? 1 : 0;
            double *o = out + bh * d;
            if (t < 0) { /* empty cache: nothing to attend to */
                for (int c = 0; c < d; ++c) {
                    o[c] = 0.0;
                    if (out_local) out_local[bh * d + c] = 0.0;
                    if (out_global) out_global[bh * d + c] = 0.0;
                }
                continue;
            }
            const uint16_t *qr = q + bh * d;
            const uint16_t *kh = k + (((int64_t)b * Hkv + h / G) * Lmax) * d;
            const uint16_t *vh = v + (((int64_t)b * Hkv + h / G) * Lmax) * d;
            int64_t j_lo = t - W + 1;
            if (j_lo < 0) j_lo = 0;
            attend_row(qr, kh, vh, j_lo, t, d, scale, s, loc);
            if (sel) attend_row(qr, kh, vh, 0, t, d, scale, s, glo);
            double gs = sel ? sigmoid((double)g[b]) : 0.0;
            for (int c = 0; c < d; ++c) {
                o[c] = loc[c] + (sel ? gs * glo[c] : 0.0);
                if (out_local) out_local[bh * d + c] = loc[c];
                if (out_global) out_global[bh * d + c] = sel ? glo[c] : 0.0;
            }
        }
        free(s);
        free(loc);
        free(glo);
    }
    return n_sel;
}

/* Number of threads the oracle runs on (for reporting). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the number of threads of the following calls (the benchmark's
 * single-thread baseline figure); n < 1 is ignored. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ---- backward pass ---------------------------------------------------- */

/*
 * Gradients of a scalar loss through the forward pass above, given the
 * loss's gradient with respect to the merged output ("dout").  The pages
 * print no backward formulas; they say the method is trained end to end and
 * that its kernels speed up training ("Learning When to Attend", "Empirical
 * Validation and System Optimization"; "LoGo", Abstract: a learned gate with
 * no auxiliary loss).  What follows is the chain rule through the forward
 * definition, with one reading:
 *   gate        o_i depends on g_i only through the factor sigmoid(g_i) on
 *               selected rows; the selection itself is a step function of the
 *               logits and passes no gradient.  So
 *               dL/dg_i = sigmoid(g_i) (1 - sigmoid(g_i)) sum_h <dout_hi, global_hi>
 *               for selected i, 0 otherwise.
 * For one softmax row with probabilities P_j over its keys, output
 * o = sum_j P_j v_j and upstream gradient e (dout for the local branch,
 * sigmoid(g_i) dout for the global branch):
 *   dv_j += P_j e;  dP_j = <e, v_j>;  D = <e, o>;  dS_j = P_j (dP_j - D);
 *   dq += scale sum_j dS_j k_j;  dk_j += scale dS_j q.
 * Key/value gradients sum over the query heads of a GQA group.
 */

/* The probabilities of one softmax row (keys j_lo..j_hi) into p[], its output into o[]. */
static void row_probs(const uint16_t *q, const uint16_t *kh, const uint16_t *vh, int64_t j_lo,
                      int64_t j_hi, int d, double scale, double *p, double *o)
{
    int64_t n = j_hi - j_lo + 1;
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t *kr = kh + (int64_t)d * (j_lo + t);
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += bf16_bits_to_double(q[c]) * bf16_bits_to_double(kr[c]);
        p[t] = scale * dot;
        if (p[t] > m) m = p[t];
    }
    double den = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        p[t] = exp(p[t] - m);
        den += p[t];
    }
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        p[t] /= den;
        const uint16_t *vr = vh + (int64_t)d * (j_lo + t);
        for (int c = 0; c < d; ++c) o[c] += p[t] * bf16_bits_to_double(vr[c]);
    }
}

/*
 * Backward of one softmax row with upstream gradient e = a * dout (a = 1 for
 * the local branch, sigmoid(g_i) for the global one).  p[] and o[] come from
 * row_probs.  Adds into dq (d doubles, may be NULL) and into the key/value
 * gradient rows dk[j], dv[j] (rows d apart, indexed from the sequence start;
 * may be NULL).  If only_key >= 0, only key j = only_key takes its dk/dv share.
 */
static void row_grad(const uint16_t *q, const uint16_t *kh, const uint16_t *vh, const uint16_t *dout,
                     double a, int64_t j_lo, int64_t j_hi, int d, double scale, const double *p,
                     const double *o, double *dq, double *dk, double *dv, int64_t only_key)
{
    double D = 0.0;
    for (int c = 0; c < d; ++c) D += a * bf16_bits_to_double(dout[c]) * o[c];
    for (int64_t j = j_lo; j <= j_hi; ++j) {
        if (!dq && only_key >= 0 && j != only_key) continue;
        const uint16_t *kr = kh + j * (int64_t)d;
        const uint16_t *vr = vh + j * (int64_t)d;
        double pj = p[j - j_lo];
        double dp = 0.0;
        for (int c = 0; c < d; ++c) dp += a * bf16_bits_to_double(dout[c]) * bf16_bits_to_double(vr[c]);
        double ds = pj * (dp - D);
        if (dq)
            for (int c = 0; c < d; ++c) dq[c] += scale * ds * bf16_bits_to_double(kr[c]);
        if (only_key >= 0 && j != only_key) continue;
        double *dkr = dk ? dk + (only_key >= 0 ? 0 : j * (int64_t)d) : NULL;
        double *dvr = dv ? dv + (only_key >= 0 ? 0 : j * (int64_t)d) : NULL;
        for (int c = 0; c < d; ++c) {
            if (dkr) dkr[c] += scale * ds * bf16_bits_to_double(q[c]);
            if (dvr) dvr[c] += pj * a * bf16_bits_to_double(dout[c]);
        }
    }
}

/*
 * Full backward pass.  Inputs as for oracle_forward, plus dout [B, Hq, L, d]
 * bf16 bits.  Outputs (doubles, overwritten): dq [B, Hq, L, d],
 * dk and dv [B, Hkv, L, d], dg [B, L] (0 on rows outside every sequence).
 * Returns the total number of selected tokens.
 */
int64_t oracle_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                        const uint16_t *dout, const int32_t *cu_seqlens, int nseq, int Hq, int Hkv, int64_t L,
                        int d, int64_t W, double ratio, double scale, double *dq, double *dk, double *dv,
                        double *dg)
{
    problem pr = {q, k, v, g, cu_seqlens, nseq, Hq, Hkv, d, L, W, default_scale(scale, d)};
    int64_t B = cu_seqlens ? 1 : nseq;
    int G = Hq / Hkv;
    memset(dq, 0, sizeof(double) * (size_t)(B * Hq * L * d));
    memset(dk, 0, sizeof(double) * (size_t)(B * Hkv * L * d));
    memset(dv, 0, sizeof(double) * (size_t)(B * Hkv * L * d));
    memset(dg, 0, sizeof(double) * (size_t)(B * L));
    int64_t total = 0;
    for (int s = 0; s < nseq; ++s) {
        int64_t b = cu_seqlens ? 0 : s;
        int64_t s0 = seq_start(&pr, s), len = seq_len(&pr, s);
        if (len <= 0) continue;
        unsigned char *flag = (unsigned char *)calloc((size_t)len, 1);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)len);
        int64_t ks = oracle_select(g + b * L + s0, len, ratio, sel);
        for (int64_t t = 0; t < ks; ++t) flag[sel[t]] = 1;
        total += ks;
        /* per row and head: <dout, global>, for the gate gradient */
        double *gdot = (double *)calloc((size_t)(len * Hq), sizeof(double));
        /* Key/value heads one after another.  Within a head, the (query head, row)
         * pairs of its group are independent except for the sums into dk and dv,
         * which each thread accumulates in a private copy; the copies are added
         * into dk, dv at the end (the same sums, in another fp64 order). */
        for (int hk = 0; hk < Hkv; ++hk) {
            const uint16_t *kh = row_ptr(k, b, Hkv, hk, L, s0, d);
            const uint16_t *vh = row_ptr(v, b, Hkv, hk, L, s0, d);
            double *dkh = dk + ((b * Hkv + hk) * L + s0) * (int64_t)d;
            double *dvh = dv + ((b * Hkv + hk) * L + s0) * (int64_t)d;
#pragma omp parallel
            {
                double *p = (double *)malloc(sizeof(double) * (size_t)len);
                double *o = (double *)malloc(sizeof(double) * (size_t)d);
                double *dkp = (double *)calloc((size_t)(len * d), sizeof(double));
                double *dvp = (double *)calloc((size_t)(len * d), sizeof(double));
#pragma omp for schedule(dynamic, 16) collapse(2)
                for (int h = hk * G; h < (hk + 1) * G; ++h) {
                    for (int64_t i = 0; i < len; ++i) {
                        const uint16_t *qr = row_ptr(q, b, Hq, h, L, s0 + i, d);
                        const uint16_t *er = row_ptr(dout, b, Hq, h, L, s0 + i, d);
                        double *dqr = dq + ((b * Hq + h) * L + s0 + i) * (int64_t)d;
                        int64_t j_lo = i - W + 1;
                        if (j_lo < 0) j_lo = 0;
                        row_probs(qr, kh, vh, j_lo, i, d, pr.scale, p, o);
                        row_grad(qr, kh, vh, er, 1.0, j_lo, i, d, pr.scale, p, o, dqr, dkp, dvp, -1);
                        if (flag[i]) {
                            double a = sigmoid((double)g[b * L + s0 + i]);
                            row_probs(qr, kh, vh, 0, i, d, pr.scale, p, o);
                            row_grad(qr, kh, vh, er, a, 0, i, d, pr.scale, p, o, dqr, dkp, dvp, -1);
                            double e = 0.0;
                            for (int c = 0; c < d; ++c) e += bf16_bits_to_double(er[c]) * o[c];
                            gdot[i * Hq + h] = e;
                        }
                    }
                }
#pragma omp critical
                {
                    for (int64_t x = 0; x < len * d; ++x) {
                        dkh[x] += dkp[x];
                        dvh[x] += dvp[x];
                    }
                }
                free(dvp);
                free(dkp);
                free(p);
                free(o);
            }
        }
        for (int64_t i = 0; i < len; ++i) {
            if (!flag[i]) continue;
            double sg = sigmoid((double)g[b * L + s0 + i]);
            double e = 0.0;
            for (int h = 0; h < Hq; ++h) e += gdot[i * Hq + h];
            dg[b * L + s0 + i] = sg * (1.0 - sg) * e;
        }
        free(gdot);
        free(sel);
        free(flag);
    }
    return total;
}

/*
 * Sampled gradient rows, for problems too large to run whole.  `flags` holds
 * one byte per row of the [B, L] gate (1 = selected; from oracle_select).
 *   Query rows t < nq: (qseq[t], qhead[t], qpos[t]) -> dq_out[t*d ..] and,
 *   summed over all heads at that position, dg_out[t].
 *   Key rows t < nk: (kseq[t], khead[t] = key/value head, kpos[t]) ->
 *   dk_out[t*d ..], dv_out[t*d ..]: the shares of every query row (local
 *   window and selected rows) of every query head of the group that reads it.
 * Positions are relative to the sequence start.
 */
void oracle_backward_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, const float *g,
                          const uint16_t *dout, const unsigned char *flags, const int32_t *cu_seqlens, int nseq,
                          int Hq, int Hkv, int64_t L, int d, int64_t W, double scale, int64_t nq,
                          const int32_t *qseq, const int32_t *qhead, const int64_t *qpos, double *dq_out,
                          double *dg_out, int64_t nk, const int32_t *kseq, const int32_t *khead,
                          const int64_t *kpos, double *dk_out, double *dv_out)
{
    problem pr = {q, k, v, g, cu_seqlens, nseq, Hq, Hkv, d, L, W, default_scale(scale, d)};
    int G = Hq / Hkv;
    int64_t maxlen = 1;
    for (int s = 0; s < nseq; ++s)
        if (seq_len(&pr, s) > maxlen) maxlen = seq_len(&pr, s);
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)maxlen);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < nq + nk; ++t) {
            int is_q = t < nq;
            int64_t u = is_q ? t : t - nq;
            int s = is_q ? qseq[u] : kseq[u];
            int64_t b = cu_seqlens ? 0 : s;
            int64_t s0 = seq_start(&pr, s), len = seq_len(&pr, s);
            if (is_q) {
                int h = qhead[u];
                int64_t i = qpos[u];
                const uint16_t *kh = row_ptr(k, b, Hkv, h / G, L, s0, d);
                const uint16_t *vh = row_ptr(v, b, Hkv, h / G, L, s0, d);
                double *dqr = dq_out + u * d;
                for (int c = 0; c < d; ++c) dqr[c] = 0.0;
                int64_t j_lo = i - W + 1;
                if (j_lo < 0) j_lo = 0;
                const uint16_t *qr = row_ptr(q, b, Hq, h, L, s0 + i, d);
                const uint16_t *er = row_ptr(dout, b, Hq, h, L, s0 + i, d);
                row_probs(qr, kh, vh, j_lo, i, d, pr.scale, p, o);
                row_grad(qr, kh, vh, er, 1.0, j_lo, i, d, pr.scale, p, o, dqr, NULL, NULL, -1);
                double e = 0.0;
                if (flags[b * L + s0 + i]) {
                    double sg = sigmoid((double)g[b * L + s0 + i]);
                    row_probs(qr, kh, vh, 0, i, d, pr.scale, p, o);
                    row_grad(qr, kh, vh, er, sg, 0, i, d, pr.scale, p, o, dqr, NULL, NULL, -1);
                    /* the gate: every head at this position */
                    for (int hh = 0; hh < Hq; ++hh) {
                        const uint16_t *q2 = row_ptr(q, b, Hq, hh, L, s0 + i, d);
                        const uint16_t *e2 = row_ptr(dout, b, Hq, hh, L, s0 + i, d);
                        const uint16_t *k2 = row_ptr(k, b, Hkv, hh / G, L, s0, d);
                        const uint16_t *v2 = row_ptr(v, b, Hkv, hh / G, L, s0, d);
                        row_probs(q2, k2, v2, 0, i, d, pr.scale, p, o);
                        for (int c = 0; c < d; ++c) e += bf16_bits_to_double(e2[c]) * o[c];
                    }
                    e *= sg * (1.0 - sg);
                }
                if (dg_out) dg_out[u] = e;
            } else {
                int hk = khead[u];
                int64_t j = kpos[u];
                const uint16_t *kh = row_ptr(k, b, Hkv, hk, L, s0, d);
                const uint16_t *vh = row_ptr(v, b, Hkv, hk, L, s0, d);
                double *dkr = dk_out + u * d, *dvr = dv_out + u * d;
                for (int c = 0; c < d; ++c) dkr[c] = dvr[c] = 0.0;
                for (int h = hk * G; h < (hk + 1) * G; ++h) {
                    for (int64_t i = j; i < len; ++i) {
                        int local = i - j < W;
                        int glob = flags[b * L + s0 + i] != 0;
                        if (!local && !glob) continue;
                        const uint16_t *qr = row_ptr(q, b, Hq, h, L, s0 + i, d);
                        const uint16_t *er = row_ptr(dout, b, Hq, h, L, s0 + i, d);
                        if (local) {
                            int64_t j_lo = i - W + 1;
                            if (j_lo < 0) j_lo = 0;
                            row_probs(qr, kh, vh, j_lo, i, d, pr.scale, p, o);
                            row_grad(qr, kh, vh, er, 1.0, j_lo, i, d, pr.scale, p, o, NULL, dkr, dvr, j);
                        }
                        if (glob) {
                            double sg = sigmoid((double)g[b * L + s0 + i]);
                            row_probs(qr, kh, vh, 0, i, d, pr.scale, p, o);
                            row_grad(qr, kh, vh, er, sg, 0, i, d, pr.scale, p, o, NULL, dkr, dvr, j);
                        }
                    }
                }
            }
        }
        free(p);
        free(o);
    }
}
