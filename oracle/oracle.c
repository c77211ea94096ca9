/*
 * Oracle for the DeepSeek-V4 CSA lightning-indexer distillation loss.
 *
 * TEST INFRASTRUCTURE ONLY. This is a plain, slow, fp64 CPU statement of what
 * the CUDA path computes. Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load it; the product never does. It shares
 * no code, header or table with the CUDA library.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "perf(deepseek-v4): fuse and enable the indexer distillation loss"
 *        (Primus pull request 992): commit messages, "Summary",
 *        "Why the target was wrong", "Test plan".
 *   [P2] "Docker Build for DeepSeek-v4 (Don't Merge)" (Primus pull request
 *        862): the gluon_v3 commit message, "Optimization Notes", "Forward".
 *   [P3] "Add Indexer Loss [Deepseek v4]" (MaxText pull request 5033):
 *        commit messages (causal block mask, packing), code review
 *        ("Teacher Distribution Semantic Mismatch", "Numerical & JAX
 *        Autodiff Stability Fixes").
 *
 * Every value is computed in double precision. bf16 inputs are widened
 * exactly. exp/log come from libm. No blocking, no reordering: each sum runs
 * in index order exactly as written below.
 *
 * Pins (tests under tests/): the window log-mass is pinned by closed forms
 * (one-key window, zero queries, document clipping) and by the full causal
 * log-sum-exp when the window covers the sequence; the target by the
 * joint softmax spelled out term by term, closed forms and invariants; the
 * KL by its zero at matching targets, a hand-computed two-slot value and
 * central finite differences. The normalisation of the loss by the number
 * of valid tokens is a reading of the pages (they do not state it): parity
 * unpinned for that constant only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the OpenMP loops below use (1 without OpenMP). */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

#define ORC_FLT_MIN 1.1754943508222875e-38 /* float32 tiny, 2^-126 */
#define ORC_OLD_FLOOR 1e-10                 /* the per-branch target's floor */
/* how distill_target forms lse_full[h] */
#define ORC_LSE_JOINT 0                     /* LSE(window, compressed, sink) */
#define ORC_LSE_PER_BRANCH 1                /* the compressed LSE alone */
#define ORC_LSE_GIVEN 2                     /* passed in by the caller */

static double bf16_val(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double dot_bf16(const uint16_t *a, const uint16_t *b, int64_t D)
{
    double s = 0.0;
    for (int64_t d = 0; d < D; ++d)
        s += bf16_val(a[d]) * bf16_val(b[d]);
    return s;
}

/* log(sum(exp(x[i]))) over n entries; -inf entries contribute nothing and an
 * all -inf (or empty) list gives -inf. */
static double lse_list(const double *x, int64_t n)
{
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (x[i] > mx)
            mx = x[i];
    if (mx == -INFINITY)
        return -INFINITY;
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i)
        if (x[i] != -INFINITY)
            s += exp(x[i] - mx);
    return mx + log(s);
}

/* Start of the document that holds token t: doc_start[b,t] clamped to [0, t]
 * (a document begins at or before its token); 0 when there is no table. */
static int64_t doc_begin(const int32_t *doc_start, int64_t g, int64_t t)
{
    if (!doc_start)
        return 0;
    int64_t d0 = doc_start[g];
    if (d0 < 0)
        d0 = 0;
    if (d0 > t)
        d0 = t;
    return d0;
}

/*
 * Sliding-window log-mass [P1, third commit message: the extra work of the
 * joint target is this per-head window mass; indexer_distill_window_lse]:
 *
 *   window_lse[b,t,h] = log sum_{s = max(d0, t-W+1)}^{t} exp(scale * <Q[b,t,h,:], Kw[b,s,:]>)
 *
 * The window holds W keys ending at the token itself, clipped at the start of
 * the token's document. Keys are single-latent (one Kw row per token, shared
 * by all heads). The per-head sink is not part of this sum.
 *
 * tokens: flat ids g = b*S + t to evaluate (NULL = all B*S, in order).
 * out: [n, H], row i for tokens[i].
 */
void orc_window_lse(const uint16_t *Q, const uint16_t *Kw, const int32_t *doc_start,
                    int64_t B, int64_t S, int64_t H, int64_t D, int64_t W, double scale,
                    const int64_t *tokens, int64_t n_tokens, double *out)
{
    int64_t n = tokens ? n_tokens : B * S;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t i = 0; i < n; ++i) {
        int64_t g = tokens ? tokens[i] : i;
        int64_t b = g / S, t = g % S;
        int64_t d0 = doc_begin(doc_start, g, t);
        int64_t lo = t - W + 1;
        if (lo < d0)
            lo = d0;
        int64_t nw = t - lo + 1;
        double *z = (double *)malloc(sizeof(double) * (size_t)nw);
        for (int64_t h = 0; h < H; ++h) {
            const uint16_t *q = Q + (g * H + h) * D;
            for (int64_t s = lo; s <= t; ++s)
                z[s - lo] = scale * dot_bf16(q, Kw + (b * S + s) * D, D);
            out[i * H + h] = lse_list(z, nw);
        }
        free(z);
    }
}

/*
 * Distillation target [P1, first and third commit messages, "Why the target
 * was wrong"]. Each head has a single softmax whose logits are the window
 * keys, the chosen pool rows and a sink logit; the target keeps the part of
 * that distribution that falls on the chosen pool rows, adds it up over heads
 * and L1-normalises the result, flooring the sum at FLT_MIN.
 *
 *   slot k of token (b,t) is selected iff 0 <= idx < P, the block lies wholly
 *   at or before the token, (idx+1)*cr - 1 <= t  [P3: causal block mask, with
 *   t=4, cr=4 block 0 allowed and block 1 masked], and the block starts inside
 *   the token's document, idx*cr >= d0 [P3: segment/packing mask];
 *   z[h,k]       = scale * <Q[b,t,h,:], pool[b, idx[k], :]>   (selected k)
 *   clse[h]      = log sum_k exp z[h,k]                       (-inf if none)
 *   lse_full[h]  = log( exp wl[h] + exp clse[h] + exp sink[h] )  (no sink term
 *                  when sink is NULL)  [head share exp(clse - lse_full)]
 *   u[k]         = sum_h exp(z[h,k] - lse_full[h])           [head sum]
 *   m            = sum_k u[k]
 *   p[k]         = u[k] / max(m, FLT_MIN)  (0 on masked slots) [the floor is the
 *                  smallest normal float32, no longer 1e-10]
 *
 * mode == ORC_LSE_PER_BRANCH selects the earlier per-branch target that the Primus page
 * keeps behind an A/B switch and the MaxText page prints [P1, second commit
 * message: PRIMUS_V4_DISTILL_NONCOMP_LSE=0 restores it; P3 commit messages]:
 * every head is normalised over the selected compressed entries alone,
 *   lse_full[h] = clse[h]   (window and sink ignored; wl and sink may be NULL)
 * and the floor is the old 1e-10: p[k] = u[k] / max(m, 1e-10).
 *
 * mode == ORC_LSE_GIVEN takes lse_full[h] from the wl rows as given: the
 * per-head log-normaliser of the whole attention row (window, selected
 * compressed entries and sink), which a CSA attention forward that returns
 * its LSE has already computed [P1, first commit message: the compressed
 * share of a head is exp(compressed_lse - full_lse); P2, gluon_v3
 * "Optimization Notes", "Forward": the CSA forward route returns its LSE].
 * The sink is not read and the floor is FLT_MIN, as for the joint target.
 *
 * wl: [n, H] rows aligned with the token list: the window log-mass, or
 * lse_full itself under ORC_LSE_GIVEN (unused under ORC_LSE_PER_BRANCH).
 * Returns the number of idx entries outside {-1} U [0, P) (data errors; those
 * slots are masked).
 */
int64_t orc_distill_target(const uint16_t *Q, const uint16_t *pool, const int32_t *idx,
                           const double *wl, const float *sink, const int32_t *doc_start,
                           int64_t B, int64_t S, int64_t H, int64_t D, int64_t K, int64_t cr,
                           double scale, const int64_t *tokens, int64_t n_tokens, int mode, double *p)
{
    int64_t n = tokens ? n_tokens : B * S;
    int64_t P = S / cr;
    int64_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (int64_t i = 0; i < n; ++i) {
        int64_t g = tokens ? tokens[i] : i;
        int64_t b = g / S, t = g % S;
        int64_t d0 = doc_begin(doc_start, g, t);
        const int32_t *row = idx + g * K;
        unsigned char *sel = (unsigned char *)calloc((size_t)K, 1);
        double *z = (double *)malloc(sizeof(double) * (size_t)(K * H)); /* [h][k] */
        double *lse_full = (double *)malloc(sizeof(double) * (size_t)H);
        for (int64_t k = 0; k < K; ++k) {
            int64_t j = row[k];
            if (!(j == -1 || (j >= 0 && j < P)))
                bad += 1;
            sel[k] = (j >= 0 && j < P && (j + 1) * cr - 1 <= t && j * cr >= d0) ? 1 : 0;
        }
        for (int64_t h = 0; h < H; ++h) {
            const uint16_t *q = Q + (g * H + h) * D;
            for (int64_t k = 0; k < K; ++k)
                z[h * K + k] = sel[k] ? scale * dot_bf16(q, pool + (b * P + row[k]) * D, D) : -INFINITY;
            double clse = lse_list(z + h * K, K);
            if (mode == ORC_LSE_PER_BRANCH) {
                lse_full[h] = clse;
                continue;
            }
            if (mode == ORC_LSE_GIVEN) {
                lse_full[h] = wl[i * H + h];
                continue;
            }
            double parts[3];
            int np = 0;
            parts[np++] = wl[i * H + h];
            parts[np++] = clse;
            if (sink)
                parts[np++] = (double)sink[h];
            lse_full[h] = lse_list(parts, np);
        }
        double m = 0.0;
        double *u = p + i * K;
        for (int64_t k = 0; k < K; ++k) {
            double acc = 0.0;
            if (sel[k])
                for (int64_t h = 0; h < H; ++h)
                    acc += exp(z[h * K + k] - lse_full[h]);
            u[k] = acc;
            m += acc;
        }
        const double floor_ = mode == ORC_LSE_PER_BRANCH ? ORC_OLD_FLOOR : ORC_FLT_MIN;
        double den = m > floor_ ? m : floor_;
        for (int64_t k = 0; k < K; ++k)
            u[k] = sel[k] ? u[k] / den : 0.0;
        free(sel);
        free(z);
        free(lse_full);
    }
    return bad;
}

/* Number of rows with at least one valid slot. */
int64_t orc_count_valid_rows(const uint8_t *valid, int64_t n_rows, int64_t K)
{
    int64_t N = 0;
    for (int64_t r = 0; r < n_rows; ++r) {
        int any = 0;
        for (int64_t k = 0; k < K; ++k)
            if (valid[r * K + k])
                any = 1;
        N += any;
    }
    return N;
}

/*
 * KL(attention || indexer) with its analytic gradient [P1, first commit
 * message: indexer_distill_kl computes the KL and its gradient in closed form
 * in one pass; P3 review: the gradient of a log-softmax KL is q - p, and rows
 * must be masked by the indexer's own mask so none is all -inf].
 *
 * Per row (token) over its valid slots:
 *   log q[k]  = s[k] - log sum_{valid k'} exp s[k']
 *   KL_row    = sum_{valid k, p[k] > 0} p[k] * (log p[k] - log q[k])   (0 log 0 = 0)
 *   loss      = coeff * sum_rows KL_row / max(N, 1)
 *   dscores[k]= coeff / max(N,1) * ( q[k] * sum_{valid} p - p[k] )  on valid slots
 * N is the number of rows with a valid slot (n_norm >= 0 overrides it, for
 * sampled rows of a larger batch). Rows without a valid slot give 0.
 * dscores and kl_rows may be NULL.
 */
void orc_distill_kl(const double *p, const float *scores, const uint8_t *valid,
                    int64_t n_rows, int64_t K, double coeff, int64_t n_norm,
                    double *loss, double *dscores, double *kl_rows)
{
    int64_t N = n_norm >= 0 ? n_norm : orc_count_valid_rows(valid, n_rows, K);
    double den = (double)(N > 1 ? N : 1);
    double total = 0.0;
    double *klr = (double *)malloc(sizeof(double) * (size_t)(n_rows > 0 ? n_rows : 1));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        const double *pr = p + r * K;
        const float *sr = scores + r * K;
        const uint8_t *vr = valid + r * K;
        double *x = (double *)malloc(sizeof(double) * (size_t)K);
        int any = 0;
        for (int64_t k = 0; k < K; ++k) {
            x[k] = vr[k] ? (double)sr[k] : -INFINITY;
            any |= vr[k] != 0;
        }
        double kl = 0.0;
        if (any) {
            double lz = lse_list(x, K);
            double psum = 0.0;
            for (int64_t k = 0; k < K; ++k)
                if (vr[k])
                    psum += pr[k];
            for (int64_t k = 0; k < K; ++k) {
                if (!vr[k]) {
                    if (dscores)
                        dscores[r * K + k] = 0.0;
                    continue;
                }
                double logq = (double)sr[k] - lz;
                if (pr[k] > 0.0)
                    kl += pr[k] * (log(pr[k]) - logq);
                if (dscores)
                    dscores[r * K + k] = coeff / den * (exp(logq) * psum - pr[k]);
            }
        } else if (dscores) {
            for (int64_t k = 0; k < K; ++k)
                dscores[r * K + k] = 0.0;
        }
        klr[r] = kl;
        free(x);
    }
    for (int64_t r = 0; r < n_rows; ++r) {
        total += klr[r];
        if (kl_rows)
            kl_rows[r] = klr[r];
    }
    free(klr);
    if (loss)
        *loss = coeff * total / den;
}

/*
 * Top-K selection of compressed blocks per token, from given indexer scores
 * [P3, the indexer's selection: top-k block indices, with -1 wherever the
 * selection is invalid, returned together with the index scores; P3 commit
 * messages: causal block mask and packing mask]. The score formula of the
 * indexer itself is not on the pages; its output is this function's input.
 *
 *   block j of token (b,t) is a candidate iff (j+1)*cr - 1 <= t, j*cr >= d0,
 *   and its score is neither NaN nor -inf (a masked or invalid entry);
 *   the K candidates with the largest scores are selected, an equal score
 *   going to the lower block index (+0 and -0 are equal);
 *   slot k holds the k-th selected block in ascending block order; the
 *   slots past the number selected hold -1.
 *
 * scores: [B*S, P] fp32 with P = S/cr. Outputs for the flat token ids in
 * tokens (all when NULL): idx [n, K]; sel [n, K] = the score of the block in
 * each slot (0 on -1 slots); valid [n, K] = 1 on selected slots.
 */
typedef struct {
    float s;
    int64_t j;
} orc_cand;

static int orc_cand_by_score(const void *pa, const void *pb)
{
    const orc_cand *a = (const orc_cand *)pa, *b = (const orc_cand *)pb;
    if (a->s > b->s)
        return -1;
    if (a->s < b->s)
        return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int orc_cand_by_block(const void *pa, const void *pb)
{
    const orc_cand *a = (const orc_cand *)pa, *b = (const orc_cand *)pb;
    return (a->j > b->j) - (a->j < b->j);
}

void orc_indexer_topk(const float *scores, const int32_t *doc_start, int64_t B, int64_t S, int64_t cr, int64_t K,
                      const int64_t *tokens, int64_t n_tokens, int32_t *idx, float *sel, uint8_t *valid)
{
    int64_t n = tokens ? n_tokens : B * S;
    int64_t P = S / cr;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i) {
        int64_t g = tokens ? tokens[i] : i;
        int64_t t = g % S;
        int64_t d0 = doc_begin(doc_start, g, t);
        const float *row = scores + g * P;
        orc_cand *c = (orc_cand *)malloc(sizeof(orc_cand) * (size_t)(P > 0 ? P : 1));
        int64_t m = 0;
        for (int64_t j = 0; j < P; ++j) {
            float s = row[j];
            if ((j + 1) * cr - 1 <= t && j * cr >= d0 && !isnan(s) && !(isinf(s) && s < 0)) {
                c[m].s = s;
                c[m].j = j;
                ++m;
            }
        }
        qsort(c, (size_t)m, sizeof(orc_cand), orc_cand_by_score);
        int64_t take = m < K ? m : K;
        qsort(c, (size_t)take, sizeof(orc_cand), orc_cand_by_block);
        for (int64_t k = 0; k < K; ++k) {
            const int inr = k < take;
            idx[i * K + k] = inr ? (int32_t)c[k].j : -1;
            if (sel)
                sel[i * K + k] = inr ? c[k].s : 0.0f;
            if (valid)
                valid[i * K + k] = (uint8_t)(inr ? 1 : 0);
        }
        free(c);
    }
}
