/*
 * Parallax decode oracle: plain fp64 CPU loops.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library
 * and its Python binding) may include, link or call this file. It is used by
 * the tests, by the bench's CPU-baseline leg and by the smoke check.
 *
 * What it computes (sources are the pages on Parallax, cited by title and
 * section):
 *   - "Parallax: Parameterized Local Linear Attention for Language Modeling"
 *     (bayesiansapien blog), opening diagram and "TL;DR": softmax attention
 *     is a local-constant (Nadaraya-Watson) estimate over the KV cache; Local
 *     Linear Attention upgrades it to a local-linear estimate, which needs a
 *     per-query solve.
 *   - same title (neuraltrendhub summary), "What the paper found" and
 *     "Original abstract": Parallax removes that solve and learns an extra
 *     query-like projector R that probes the KV covariance; the kernel
 *     streams the same K/V tiles as FlashAttention.
 *   - "Integrazioni AI personalizzate dopo l'attenzione Parallax" (encorp.ai),
 *     "Parallax conserva softmax ..." and FAQ: with the projection at zero the
 *     layer is exactly softmax attention.
 *   - parallax-kernel 0.1.0 README, "Decoding (CuTeDSL)": a decode call takes
 *     q, r (one probe row per query head, shaped like q), k, v and qk_scale.
 *
 * Written out, with w_i = softmax_i(scale * q.k_i) over the cached keys and
 * s_i = r.k_i (the probe score; qk_scale is not applied to it):
 *
 *   o = vbar + sum_i w_i (s_i - sbar)(v_i - vbar),  vbar = sum w_i v_i,
 *                                                  sbar = sum w_i s_i
 *     = vbar + Cov_w(v, k) r.
 *
 * This is the intercept of the weighted local-linear fit with the solver
 * output Sigma_w^{-1}(q - kbar) replaced by the learned probe r. Expanding the
 * covariance with un-normalised weights e_i = exp(t_i - m):
 *
 *   l = sum e_i, A = sum e_i v_i, b = sum e_i s_i, C = sum e_i s_i v_i,
 *   o = A/l + C/l - (b/l)(A/l).
 *
 * Three forms are given so that tests can check them against each other:
 *   oracle_parallax_covariance  - the definition (two passes, centred)
 *   oracle_parallax_expanded    - the (l, A, b, C) expansion
 *   oracle_parallax_streaming   - the same accumulators updated one key at a
 *                                 time with a running max, in chunks that are
 *                                 combined by the max-rescaling merge
 * plus oracle_softmax_decode, the R = 0 special case written as plain softmax
 * attention, and oracle_parallax_prefill, the training-shape forward (every
 * query row of a sequence, causal), which applies the definition form to the
 * keys each row sees.
 *
 * Readings where the pages are silent (all documented in the design notes):
 *   - layouts: q, r, out are [B][Hq][D]; k, v are [B][Hkv][Lmax][D];
 *   - query head h reads kv head h / (Hq / Hkv) (contiguous GQA groups);
 *   - keys 0 .. seqlens[b]-1 are attended, nothing else is read;
 *   - a sequence with no keys returns a zero output.
 *
 * All inputs are doubles (callers widen bf16 / fp32 values exactly).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EBADARG (-1)
#define ORACLE_ENOMEM (-2)

static double dot(const double* a, const double* b, int D) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

static int check_args(const double* q, const double* k, const double* v,
                      const int32_t* seqlens, int B, int Hq, int Hkv, int Lmax,
                      int D, const double* out) {
    if (!q || !k || !v || !seqlens || !out) return ORACLE_EBADARG;
    if (B < 0 || Hq < 1 || Hkv < 1 || D < 1 || Lmax < 0) return ORACLE_EBADARG;
    if (Hq % Hkv != 0) return ORACLE_EBADARG;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Lmax) return ORACLE_EBADARG;
    return ORACLE_OK;
}

/* Pointers to the rows used by query head h of batch b. */
typedef struct {
    const double* q;
    const double* r; /* NULL for the softmax form */
    const double* k; /* key 0 of kv head h / G */
    const double* v;
    double* o;
    int n;
} head_view;

static head_view view_of(const double* q, const double* r, const double* k,
                         const double* v, const int32_t* seqlens, double* out,
                         int b, int h, int Hq, int Hkv, int Lmax, int D) {
    head_view hv;
    int G = Hq / Hkv;
    int g = h / G;
    size_t qo = ((size_t)b * Hq + h) * (size_t)D;
    size_t ko = ((size_t)b * Hkv + g) * (size_t)Lmax * (size_t)D;
    hv.q = q + qo;
    hv.r = r ? r + qo : NULL;
    hv.k = k + ko;
    hv.v = v + ko;
    hv.o = out + qo;
    hv.n = seqlens[b];
    return hv;
}

/* Logits t_i = scale * q.k_i and probe scores s_i = r.k_i for i < n. */
static void scores(const head_view* hv, int D, double scale, double* t,
                   double* s) {
    for (int i = 0; i < hv->n; ++i) {
        const double* ki = hv->k + (size_t)i * D;
        t[i] = scale * dot(hv->q, ki, D);
        if (s) s[i] = hv->r ? dot(hv->r, ki, D) : 0.0;
    }
}

/* Normalised softmax weights w_i = exp(t_i - max t) / sum_j exp(t_j - max t). */
static void softmax_weights(const double* t, int n, double* w) {
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) m = t[i] > m ? t[i] : m;
    double z = 0.0;
    for (int i = 0; i < n; ++i) {
        w[i] = exp(t[i] - m);
        z += w[i];
    }
    for (int i = 0; i < n; ++i) w[i] /= z;
}

/* ---- covariance (definition) form ------------------------------------- */

static void head_covariance(const head_view* hv, int D, double scale,
                            double* t, double* s, double* w, double* vbar) {
    int n = hv->n;
    if (n == 0) {
        memset(hv->o, 0, sizeof(double) * (size_t)D);
        return;
    }
    scores(hv, D, scale, t, s);
    softmax_weights(t, n, w);
    /* weighted means of v and of the probe scores */
    for (int d = 0; d < D; ++d) vbar[d] = 0.0;
    double sbar = 0.0;
    for (int i = 0; i < n; ++i) {
        const double* vi = hv->v + (size_t)i * D;
        for (int d = 0; d < D; ++d) vbar[d] += w[i] * vi[d];
        sbar += w[i] * s[i];
    }
    /* o = vbar + sum_i w_i (s_i - sbar)(v_i - vbar) */
    for (int d = 0; d < D; ++d) hv->o[d] = vbar[d];
    for (int i = 0; i < n; ++i) {
        const double* vi = hv->v + (size_t)i * D;
        double ws = w[i] * (s[i] - sbar);
        for (int d = 0; d < D; ++d) hv->o[d] += ws * (vi[d] - vbar[d]);
    }
}

/* ---- expanded (l, A, b, C) form ---------------------------------------- */

static void head_expanded(const head_view* hv, int D, double scale, double* t,
                          double* s, double* A, double* C) {
    int n = hv->n;
    if (n == 0) {
        memset(hv->o, 0, sizeof(double) * (size_t)D);
        return;
    }
    scores(hv, D, scale, t, s);
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) m = t[i] > m ? t[i] : m;
    double l = 0.0, bb = 0.0;
    for (int d = 0; d < D; ++d) A[d] = C[d] = 0.0;
    for (int i = 0; i < n; ++i) {
        const double* vi = hv->v + (size_t)i * D;
        double e = exp(t[i] - m);
        l += e;
        bb += e * s[i];
        for (int d = 0; d < D; ++d) {
            A[d] += e * vi[d];
            C[d] += e * s[i] * vi[d];
        }
    }
    for (int d = 0; d < D; ++d) {
        double vbar = A[d] / l;
        hv->o[d] = vbar + C[d] / l - (bb / l) * vbar;
    }
}

/* ---- streaming form: online accumulators per chunk, then a merge ------- */

typedef struct {
    double m, l, b;
    double* A;
    double* C;
} accum;

static void accum_reset(accum* a, int D) {
    a->m = -INFINITY;
    a->l = 0.0;
    a->b = 0.0;
    for (int d = 0; d < D; ++d) a->A[d] = a->C[d] = 0.0;
}

/* One key: m' = max(m, t); alpha = e^{m - m'}; e = e^{t - m'};
 * l = alpha l + e; A = alpha A + e v; b = alpha b + e s; C = alpha C + e s v. */
static void accum_push(accum* a, double t, double s, const double* v, int D) {
    double m_new = t > a->m ? t : a->m;
    double alpha = exp(a->m - m_new); /* exp(-inf) = 0 on the first key */
    double e = exp(t - m_new);
    a->l = alpha * a->l + e;
    a->b = alpha * a->b + e * s;
    for (int d = 0; d < D; ++d) {
        a->A[d] = alpha * a->A[d] + e * v[d];
        a->C[d] = alpha * a->C[d] + e * s * v[d];
    }
    a->m = m_new;
}

/* Merge of chunk partials: M = max m_j, alpha_j = e^{m_j - M},
 * l = sum alpha_j l_j, and the same for A, b, C. */
static void accum_merge(accum* into, const accum* part, int D) {
    if (part->l == 0.0) return; /* an empty chunk contributes nothing */
    double M = part->m > into->m ? part->m : into->m;
    double ai = exp(into->m - M);
    double ap = exp(part->m - M);
    into->l = ai * into->l + ap * part->l;
    into->b = ai * into->b + ap * part->b;
    for (int d = 0; d < D; ++d) {
        into->A[d] = ai * into->A[d] + ap * part->A[d];
        into->C[d] = ai * into->C[d] + ap * part->C[d];
    }
    into->m = M;
}

static void head_streaming(const head_view* hv, int D, double scale, int chunk,
                           accum* total, accum* part) {
    int n = hv->n;
    accum_reset(total, D);
    for (int lo = 0; lo < n; lo += chunk) {
        int hi = lo + chunk < n ? lo + chunk : n;
        accum_reset(part, D);
        for (int i = lo; i < hi; ++i) {
            const double* ki = hv->k + (size_t)i * D;
            double t = scale * dot(hv->q, ki, D);
            double s = hv->r ? dot(hv->r, ki, D) : 0.0;
            accum_push(part, t, s, hv->v + (size_t)i * D, D);
        }
        accum_merge(total, part, D);
    }
    if (n == 0 || total->l == 0.0) {
        memset(hv->o, 0, sizeof(double) * (size_t)D);
        return;
    }
    for (int d = 0; d < D; ++d) {
        double vbar = total->A[d] / total->l;
        hv->o[d] = vbar + total->C[d] / total->l - (total->b / total->l) * vbar;
    }
}

/* ---- softmax attention (R = 0 reference) ------------------------------- */

static void head_softmax(const head_view* hv, int D, double scale, double* t,
                         double* w) {
    int n = hv->n;
    memset(hv->o, 0, sizeof(double) * (size_t)D);
    if (n == 0) return;
    scores(hv, D, scale, t, NULL);
    softmax_weights(t, n, w);
    for (int i = 0; i < n; ++i) {
        const double* vi = hv->v + (size_t)i * D;
        for (int d = 0; d < D; ++d) hv->o[d] += w[i] * vi[d];
    }
}

/* ---- exported entry points --------------------------------------------- */

enum { FORM_COV = 0, FORM_EXP = 1, FORM_STREAM = 2, FORM_SOFTMAX = 3 };

static int run(int form, const double* q, const double* r, const double* k,
               const double* v, const int32_t* seqlens, int B, int Hq, int Hkv,
               int Lmax, int D, double scale, int chunk, double* out) {
    int rc = check_args(q, k, v, seqlens, B, Hq, Hkv, Lmax, D, out);
    if (rc) return rc;
    if (form != FORM_SOFTMAX && !r) return ORACLE_EBADARG;
    if (form == FORM_STREAM && chunk < 1) return ORACLE_EBADARG;
    int nmax = 1;
    for (int b = 0; b < B; ++b) nmax = seqlens[b] > nmax ? seqlens[b] : nmax;
    int failed = 0;
    long long pairs = (long long)B * Hq;
#pragma omp parallel
    {
        /* per-thread scratch */
        double* t = malloc(sizeof(double) * (size_t)nmax);
        double* s = malloc(sizeof(double) * (size_t)nmax);
        double* w = malloc(sizeof(double) * (size_t)nmax);
        double* x0 = malloc(sizeof(double) * (size_t)D * 4);
        if (!t || !s || !w || !x0) {
#pragma omp atomic write
            failed = 1;
        }
        accum total = {0, 0, 0, x0, x0 + D};
        accum part = {0, 0, 0, x0 + 2 * D, x0 + 3 * D};
#pragma omp for schedule(dynamic, 1)
        for (long long p = 0; p < pairs; ++p) {
            if (!t || !s || !w || !x0) continue;
            int b = (int)(p / Hq), h = (int)(p % Hq);
            head_view hv = view_of(q, form == FORM_SOFTMAX ? NULL : r, k, v,
                                   seqlens, out, b, h, Hq, Hkv, Lmax, D);
            switch (form) {
                case FORM_COV: head_covariance(&hv, D, scale, t, s, w, x0); break;
                case FORM_EXP: head_expanded(&hv, D, scale, t, s, x0, x0 + D); break;
                case FORM_STREAM: head_streaming(&hv, D, scale, chunk, &total, &part); break;
                default: head_softmax(&hv, D, scale, t, w); break;
            }
        }
        free(t);
        free(s);
        free(w);
        free(x0);
    }
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

int oracle_parallax_covariance(const double* q, const double* r,
                               const double* k, const double* v,
                               const int32_t* seqlens, int B, int Hq, int Hkv,
                               int Lmax, int D, double scale, double* out) {
    return run(FORM_COV, q, r, k, v, seqlens, B, Hq, Hkv, Lmax, D, scale, 1, out);
}

int oracle_parallax_expanded(const double* q, const double* r, const double* k,
                             const double* v, const int32_t* seqlens, int B,
                             int Hq, int Hkv, int Lmax, int D, double scale,
                             double* out) {
    return run(FORM_EXP, q, r, k, v, seqlens, B, Hq, Hkv, Lmax, D, scale, 1, out);
}

int oracle_parallax_streaming(const double* q, const double* r,
                              const double* k, const double* v,
                              const int32_t* seqlens, int B, int Hq, int Hkv,
                              int Lmax, int D, double scale, int chunk,
                              double* out) {
    return run(FORM_STREAM, q, r, k, v, seqlens, B, Hq, Hkv, Lmax, D, scale,
               chunk, out);
}

int oracle_softmax_decode(const double* q, const double* k, const double* v,
                          const int32_t* seqlens, int B, int Hq, int Hkv,
                          int Lmax, int D, double scale, double* out) {
    return run(FORM_SOFTMAX, q, NULL, k, v, seqlens, B, Hq, Hkv, Lmax, D, scale,
               1, out);
}

/* ---- prefill (training-shape forward) -----------------------------------
 *
 * parallax-kernel 0.1.0 README, "Training (Triton)": parallax_func(q, r, k, v)
 * maps (B, H, L, D) tensors to (B, H, L, D), causal. Row i of head h is the
 * decode output above over keys 0..i of kv head h / (Hq/Hkv) (all L keys when
 * causal == 0). Layouts: q, r, out [B][Hq][L][D]; k, v [B][Hkv][L][D].
 */
int oracle_parallax_prefill(const double* q, const double* r, const double* k,
                            const double* v, int B, int Hq, int Hkv, int L, int D,
                            double scale, int causal, double* out) {
    if (!q || !r || !k || !v || !out) return ORACLE_EBADARG;
    if (B < 0 || Hq < 1 || Hkv < 1 || L < 0 || D < 1 || Hq % Hkv != 0) return ORACLE_EBADARG;
    int G = Hq / Hkv;
    long long rows = (long long)B * Hq * L;
    int failed = 0;
#pragma omp parallel
    {
        int nmax = L > 0 ? L : 1;
        double* t = malloc(sizeof(double) * (size_t)nmax);
        double* s = malloc(sizeof(double) * (size_t)nmax);
        double* w = malloc(sizeof(double) * (size_t)nmax);
        double* vb = malloc(sizeof(double) * (size_t)D);
        if (!t || !s || !w || !vb) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (long long x = 0; x < rows; ++x) {
            if (!t || !s || !w || !vb) continue;
            int b = (int)(x / ((long long)Hq * L));
            int h = (int)((x / L) % Hq);
            int i = (int)(x % L);
            size_t qo = (((size_t)b * Hq + h) * (size_t)L + (size_t)i) * (size_t)D;
            size_t ko = ((size_t)b * Hkv + (size_t)(h / G)) * (size_t)L * (size_t)D;
            head_view hv;
            hv.q = q + qo;
            hv.r = r + qo;
            hv.k = k + ko;
            hv.v = v + ko;
            hv.o = out + qo;
            hv.n = causal ? i + 1 : L;
            head_covariance(&hv, D, scale, t, s, w, vb);
        }
        free(t);
        free(s);
        free(w);
        free(vb);
    }
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
