/*
 * losa_oracle.c -- plain, slow CPU oracle for LoSA per-denoising-step
 * attention ("LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion
 * Language Models").
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Every function restates one step of the method as the pages describe it,
 * with loops in the obvious order and no blocking, fusion or reordering:
 *
 *   locality score   per-token MSE between the current and the previous
 *                    step's query (paper, "locality of representation
 *                    changes"; methodology: locality pruning)
 *   active set       the tokens with the largest change (methodology)
 *   page bound       QUEST's upper bound sum_i max(q_i*kmax_i, q_i*kmin_i)
 *                    over per-page key min/max (methodology: sparse
 *                    attention for active tokens, "a selector such as QUEST")
 *   page selection   top-k pages under a token budget, k = budget/page_size
 *   prefix attention softmax attention over the selected pages' tokens,
 *                    giving o_p and the log-normaliser L_p (methodology)
 *   reuse            stable tokens keep last step's o_p, L_p (methodology)
 *   suffix attention dense attention over the block's own keys (mechanism)
 *   merge            online-softmax merge of prefix and suffix (mechanism)
 *   cold start       the first step of a block is dense (limitations)
 *
 * Precision.  Attention sums (scores, exp weights, normaliser, weighted
 * values) are carried in double from fp32 (or bf16-valued fp32) inputs and
 * rounded to fp32 at the end: the exact softmax up to fp64 rounding.  The two
 * scores that decide integers -- the locality MSE and the page bound -- are
 * computed in fp32, one rounding per operation, summing channels in order
 * i = 0..d-1, because the CUDA path takes the same decisions in fp32.  The
 * cached prefix state and the outputs are fp32.
 *
 * Compile with -O2 -fno-fast-math -ffp-contract=off (no fused multiply-add,
 * no reassociation).
 *
 * Parity pins: every function here is checked by tests against brute force,
 * closed forms and invariants (see the tests directory); none is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int S;        /* sequences                                  */
    int Hq;       /* query heads                                */
    int Hkv;      /* key/value heads; Hq % Hkv == 0             */
    int d;        /* head dimension                             */
    int L;        /* prefix length (tokens)                     */
    int ps;       /* page size (tokens per page)                */
    int B;        /* block size (tokens denoised together)      */
    int A;        /* active tokens per query head, |A|          */
    int budget;   /* token budget per active query              */
    float scale;  /* softmax scale                              */
    int flags;    /* variant bits, ORACLE_ATTEND_UNION below     */
} oracle_shape;

/* Variant: every active row attends to all pages of its GQA group's union
 * (the pages that are loaded once per group, paper, methodology: sparse
 * computation for active tokens) instead of only its own top-k pages. */
#define ORACLE_ATTEND_UNION 1

/* ---- planted-mistake switch (tests only) -------------------------------
 * 0 = the method as written.  A non-zero value plants one deliberate bug so
 * that the pin tests can show they catch it.  Never set outside tests. */
static int g_mut = 0;
void oracle_set_mutation(int m) { g_mut = m; }
#define MUT(n) (g_mut == (n))

static int n_pages(const oracle_shape* sh) { return (sh->L + sh->ps - 1) / sh->ps; }
static int pages_per_row(const oracle_shape* sh) {
    int k = sh->budget / sh->ps;
    int P = n_pages(sh);
    return k < P ? k : P;
}
/* KV head serving query head h: contiguous groups of G = Hq/Hkv heads. */
static int kv_head_of(const oracle_shape* sh, int h) {
    int G = sh->Hq / sh->Hkv;
    return MUT(4) ? h % sh->Hkv : h / G;
}

/* ------------------------------------------------------------------------
 * Page metadata: per page and channel, min and max of the keys of the
 * page's valid tokens (the prerequisite of the QUEST bound).
 * K [S][Hkv][L][d] -> kmin, kmax [S][Hkv][P][d].
 * ---------------------------------------------------------------------- */
void oracle_build_meta(const oracle_shape* sh, const float* K, float* kmin, float* kmax) {
    int P = n_pages(sh), d = sh->d;
    for (int s = 0; s < sh->S; ++s)
        for (int g = 0; g < sh->Hkv; ++g) {
            const float* Kg = K + ((size_t)s * sh->Hkv + g) * (size_t)sh->L * d;
            for (int p = 0; p < P; ++p) {
                float* mn = kmin + (((size_t)s * sh->Hkv + g) * P + p) * d;
                float* mx = kmax + (((size_t)s * sh->Hkv + g) * P + p) * d;
                int j0 = p * sh->ps;
                int j1 = j0 + sh->ps;
                if (j1 > sh->L) j1 = sh->L;
                if (MUT(8)) j1 = j1 - 1;
                for (int i = 0; i < d; ++i) {
                    float lo = Kg[(size_t)j0 * d + i], hi = lo;
                    for (int j = j0 + 1; j < j1; ++j) {
                        float x = Kg[(size_t)j * d + i];
                        if (x < lo) lo = x;
                        if (x > hi) hi = x;
                    }
                    mn[i] = lo;
                    mx[i] = hi;
                }
            }
        }
}

/* ------------------------------------------------------------------------
 * Softmax attention of one query over n key/value rows (row-major [*][d]),
 * the rows named by tok[0..n-1]:
 *   s_j = scale * q.k_j,  m = max s_j,  l = sum exp(s_j - m),
 *   o = sum exp(s_j - m) v_j / l,  lse = m + log l.
 * All in double.  o_out gets fp64 results (callers round).
 * ---------------------------------------------------------------------- */
static void attend(int d, double scale, const float* q, const float* K, const float* V,
                   int n, const int* tok, double* o_out, double* lse_out) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        const float* k = K + (size_t)tok[j] * d;
        double acc = 0.0;
        for (int i = 0; i < d; ++i) acc += (double)q[i] * (double)k[i];
        s[j] = (MUT(6) ? 1.0 : scale) * acc;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int i = 0; i < d; ++i) o_out[i] = 0.0;
    for (int j = 0; j < n; ++j) {
        double w = exp(s[j] - m);
        l += w;
        const float* v = V + (size_t)tok[j] * d;
        for (int i = 0; i < d; ++i) o_out[i] += w * (double)v[i];
    }
    for (int i = 0; i < d; ++i) o_out[i] /= l;
    *lse_out = MUT(10) ? log(l) : m + log(l);
    free(s);
}

/* Test entry: attention of q over rows tok[] of K, V; fp64 results. */
void oracle_attend_tokens(int d, float scale, const float* q, const float* K, const float* V,
                          int n, const int* tok, double* o, double* lse) {
    attend(d, (double)scale, q, K, V, n, tok, o, lse);
}

/* ------------------------------------------------------------------------
 * Online-softmax merge of two partial attentions (o1, L1) and (o2, L2):
 *   m = max(L1, L2), a = exp(L1 - m), b = exp(L2 - m),
 *   o = (a o1 + b o2) / (a + b),  lse = m + log(a + b).
 * ---------------------------------------------------------------------- */
static void merge(int d, const double* o1, double l1, const double* o2, double l2,
                  double* o, double* lse) {
    double m = l1 > l2 ? l1 : l2;
    double a = exp(l1 - m);
    double b = MUT(3) ? exp(m - l2) : exp(l2 - m);
    for (int i = 0; i < d; ++i) o[i] = (a * o1[i] + b * o2[i]) / (a + b);
    *lse = m + log(a + b);
}

void oracle_merge(int d, const double* o1, double l1, const double* o2, double l2,
                  double* o, double* lse) {
    merge(d, o1, l1, o2, l2, o, lse);
}

/* ------------------------------------------------------------------------
 * Locality score: mse[s][h][t] = (1/d) sum_i (Qc_i - Qp_i)^2, fp32, one
 * rounding per operation, channels in order.
 * ---------------------------------------------------------------------- */
void oracle_locality(const oracle_shape* sh, const float* Qc, const float* Qp, float* mse) {
    int d = sh->d;
    size_t rows = (size_t)sh->S * sh->Hq * sh->B;
    for (size_t r = 0; r < rows; ++r) {
        float acc = 0.0f;
        for (int i = 0; i < d; ++i) {
            float delta = MUT(7) ? Qc[r * d + i] + Qp[r * d + i] : Qc[r * d + i] - Qp[r * d + i];
            float sq = delta * delta;
            acc = acc + sq;
        }
        mse[r] = acc / (float)d;
    }
}

/* Active set of one query head: the A tokens with the largest mse (ties go
 * to the lower token index), returned in ascending token order. */
static const float* g_keys;
static int cmp_desc_then_index(const void* a, const void* b) {
    int i = *(const int*)a, j = *(const int*)b;
    float x = g_keys[i], y = g_keys[j];
    if (x > y) return -1;
    if (x < y) return 1;
    if (MUT(5)) return (i > j) ? -1 : (i < j);
    return (i < j) ? -1 : (i > j);
}
static int cmp_int_asc(const void* a, const void* b) {
    int i = *(const int*)a, j = *(const int*)b;
    return (i < j) ? -1 : (i > j);
}
/* Top-n of keys[0..m-1] by (key desc, index asc); out[0..n-1] ascending. */
static void top_n_ascending(const float* keys, int m, int n, int* out) {
    int* idx = (int*)malloc(sizeof(int) * (size_t)(m > 0 ? m : 1));
    for (int i = 0; i < m; ++i) idx[i] = i;
    g_keys = keys;
    qsort(idx, (size_t)m, sizeof(int), cmp_desc_then_index);
    for (int i = 0; i < n; ++i) out[i] = idx[i];
    qsort(out, (size_t)n, sizeof(int), cmp_int_asc);
    free(idx);
}

/* active_idx [S][Hq][A] from mse [S][Hq][B]. */
void oracle_active(const oracle_shape* sh, const float* mse, int* active_idx) {
    for (int sh_ = 0; sh_ < sh->S * sh->Hq; ++sh_)
        top_n_ascending(mse + (size_t)sh_ * sh->B, sh->B, sh->A, active_idx + (size_t)sh_ * sh->A);
}

/* ------------------------------------------------------------------------
 * QUEST page bound for one query over P pages of one KV head:
 *   U[p] = sum_i max(q_i * kmax[p][i], q_i * kmin[p][i])   (fp32, in order)
 * ---------------------------------------------------------------------- */
void oracle_bound_scores(int d, int P, const float* q, const float* kmin, const float* kmax,
                         float* U) {
    for (int p = 0; p < P; ++p) {
        const float* mn = kmin + (size_t)p * d;
        const float* mx = kmax + (size_t)p * d;
        float acc = 0.0f;
        int n = MUT(1) ? d - 1 : d;
        for (int i = 0; i < n; ++i) {
            float a = q[i] * mx[i];
            float b = q[i] * mn[i];
            float t = MUT(2) ? fminf(a, b) : fmaxf(a, b);
            acc = acc + t;
        }
        U[p] = acc;
    }
}

/* Top-k pages by (U desc, page asc), ascending page ids. -0 == +0. */
void oracle_topk_pages(int P, int k, const float* U, int* pages) {
    top_n_ascending(U, P, k, pages);
}

/* Token ids of the given pages (tokens j < L only). Returns the count. */
static int tokens_of_pages(const oracle_shape* sh, const int* pages, int np, int* tok) {
    int n = 0;
    for (int a = 0; a < np; ++a)
        for (int j = pages[a] * sh->ps; j < (pages[a] + 1) * sh->ps && j < sh->L; ++j) tok[n++] = j;
    return n;
}

/* ------------------------------------------------------------------------
 * Suffix attention + merge for every row of every head, reading the cached
 * prefix state (o_p, l_p) as it is after this step's update.
 * ---------------------------------------------------------------------- */
static void suffix_and_merge(const oracle_shape* sh, const float* Q, const float* Kb,
                             const float* Vb, const float* o_p, const float* l_p, float* out,
                             float* out_lse) {
    int d = sh->d, B = sh->B;
    int* tok = (int*)malloc(sizeof(int) * (size_t)B);
    double* os = (double*)malloc(sizeof(double) * (size_t)d);
    double* op = (double*)malloc(sizeof(double) * (size_t)d);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    for (int j = 0; j < B; ++j) tok[j] = j;
    for (int s = 0; s < sh->S; ++s)
        for (int h = 0; h < sh->Hq; ++h) {
            int g = kv_head_of(sh, h);
            const float* Kg = Kb + ((size_t)s * sh->Hkv + g) * (size_t)B * d;
            const float* Vg = Vb + ((size_t)s * sh->Hkv + g) * (size_t)B * d;
            for (int t = 0; t < B; ++t) {
                size_t r = ((size_t)s * sh->Hq + h) * B + t;
                double ls, lse;
                attend(d, (double)sh->scale, Q + r * d, Kg, Vg, B, tok, os, &ls);
                for (int i = 0; i < d; ++i) op[i] = (double)o_p[r * d + i];
                merge(d, op, (double)l_p[r], os, ls, o, &lse);
                for (int i = 0; i < d; ++i) out[r * d + i] = (float)o[i];
                if (out_lse) out_lse[r] = (float)lse;
            }
        }
    free(tok); free(os); free(op); free(o);
}

/* ------------------------------------------------------------------------
 * Cold-start dense pass (first denoising step of a block): every row attends
 * to the whole prefix, filling the cache for all B tokens; then suffix and
 * merge give the step output.
 * ---------------------------------------------------------------------- */
void oracle_dense_prefix(const oracle_shape* sh, const float* Q, const float* K, const float* V,
                         const float* Kb, const float* Vb, float* o_p, float* l_p, float* out,
                         float* out_lse) {
    int d = sh->d, L = sh->L;
    int* tok = (int*)malloc(sizeof(int) * (size_t)L);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    for (int j = 0; j < L; ++j) tok[j] = j;
    for (int s = 0; s < sh->S; ++s)
        for (int h = 0; h < sh->Hq; ++h) {
            int g = kv_head_of(sh, h);
            const float* Kg = K + ((size_t)s * sh->Hkv + g) * (size_t)L * d;
            const float* Vg = V + ((size_t)s * sh->Hkv + g) * (size_t)L * d;
            for (int t = 0; t < sh->B; ++t) {
                size_t r = ((size_t)s * sh->Hq + h) * sh->B + t;
                double lse;
                attend(d, (double)sh->scale, Q + r * d, Kg, Vg, L, tok, o, &lse);
                for (int i = 0; i < d; ++i) o_p[r * d + i] = (float)o[i];
                l_p[r] = (float)lse;
            }
        }
    free(tok); free(o);
    suffix_and_merge(sh, Q, Kb, Vb, o_p, l_p, out, out_lse);
}

/* Dense prefix attention of selected rows only (rows[] index [S][Hq][B]
 * flattened: r = (s*Hq + h)*B + t); for spot checks at sizes where the full
 * pass is too slow.  The same cold-start pass as oracle_dense_prefix (paper,
 * limitations: the forced dense first iteration of a block), row by row. */
void oracle_dense_rows(const oracle_shape* sh, const float* Q, const float* K, const float* V,
                       int n_rows, const int* rows, float* o_p, float* l_p) {
    int d = sh->d, L = sh->L;
    int* tok = (int*)malloc(sizeof(int) * (size_t)L);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    for (int j = 0; j < L; ++j) tok[j] = j;
    for (int a = 0; a < n_rows; ++a) {
        int r = rows[a];
        int h = (r / sh->B) % (MUT(13) ? sh->Hkv : sh->Hq), s = r / (sh->B * sh->Hq);
        int g = kv_head_of(sh, h);
        const float* Kg = K + ((size_t)s * sh->Hkv + g) * (size_t)L * d;
        const float* Vg = V + ((size_t)s * sh->Hkv + g) * (size_t)L * d;
        double lse;
        attend(d, (double)sh->scale, Q + (size_t)r * d, Kg, Vg, L, tok, o, &lse);
        for (int i = 0; i < d; ++i) o_p[(size_t)a * d + i] = (float)o[i];
        l_p[a] = (float)lse;
    }
    free(tok); free(o);
}

/* ------------------------------------------------------------------------
 * One LoSA step with the active set and page lists given (shared tail of
 * oracle_step; also used directly by tests that fix the selection).
 *   active_idx [S][Hq][A] ascending, page_idx [S][Hq][A][k] ascending.
 * Updates o_p, l_p of active rows in place (stable rows untouched), then
 * writes out/out_lse for all rows, and union_count [S][Hkv] (may be NULL).
 * ---------------------------------------------------------------------- */
void oracle_step_forced(const oracle_shape* sh, const float* Qc, const float* K, const float* V,
                        const float* Kb, const float* Vb, const int* active_idx,
                        const int* page_idx, float* o_p, float* l_p, float* out, float* out_lse,
                        int* union_count) {
    int d = sh->d, B = sh->B, A = sh->A, k = pages_per_row(sh), P = n_pages(sh);
    int* tok = (int*)malloc(sizeof(int) * (size_t)(P * sh->ps + 1));
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    char* used = (char*)malloc((size_t)P);
    int* ul = (int*)malloc(sizeof(int) * (size_t)P);
    for (int s = 0; s < sh->S; ++s)
        for (int g = 0; g < sh->Hkv; ++g) {
            /* the group's union: every page some active row of the group selected */
            memset(used, 0, (size_t)P);
            int cnt = 0;
            for (int h = 0; h < sh->Hq; ++h) {
                if (kv_head_of(sh, h) != g) continue;
                for (int a = 0; a < A; ++a)
                    for (int c = 0; c < k; ++c) {
                        int p = page_idx[(((size_t)s * sh->Hq + h) * A + a) * k + c];
                        if (!used[p] || MUT(9)) { used[p] = 1; ++cnt; }
                    }
            }
            if (union_count) union_count[s * sh->Hkv + g] = cnt;
            int nu = 0;
            for (int p = 0; p < P; ++p)
                if (used[p]) ul[nu++] = p;
            const float* Kg = K + ((size_t)s * sh->Hkv + g) * (size_t)sh->L * d;
            const float* Vg = V + ((size_t)s * sh->Hkv + g) * (size_t)sh->L * d;
            for (int h = 0; h < sh->Hq; ++h) {
                if (kv_head_of(sh, h) != g) continue;
                for (int a = 0; a < A; ++a) {
                    int t = active_idx[((size_t)s * sh->Hq + h) * A + a];
                    size_t r = ((size_t)s * sh->Hq + h) * B + t;
                    const int* pg = page_idx + (((size_t)s * sh->Hq + h) * A + a) * k;
                    int n = ((sh->flags & ORACLE_ATTEND_UNION) && !MUT(12)) ? tokens_of_pages(sh, ul, nu, tok)
                                                              : tokens_of_pages(sh, pg, k, tok);
                    double lse;
                    attend(d, (double)sh->scale, Qc + r * d, Kg, Vg, n, tok, o, &lse);
                    for (int i = 0; i < d; ++i) o_p[r * d + i] = (float)o[i];
                    l_p[r] = (float)lse;
                }
            }
        }
    free(tok); free(o); free(used); free(ul);
    suffix_and_merge(sh, Qc, Kb, Vb, o_p, l_p, out, out_lse);
}

/* ------------------------------------------------------------------------
 * One LoSA denoising step (steps 2..T of a block):
 *   1. locality score of every token (mse of Qc vs Qp)
 *   2. active set: top-|A| per query head
 *   3. QUEST bound of every page for each active query; top-k pages
 *   4. sparse prefix attention for active rows -> new o_p, L_p (cache)
 *   5. stable rows keep the cached o_p, L_p
 *   6. suffix attention + merge for every row
 * kmin/kmax [S][Hkv][P][d] from oracle_build_meta.  Optional outputs (may be
 * NULL): mse [S][Hq][B]; bound [S][Hq][A][P] (every page's U per active row).
 * ---------------------------------------------------------------------- */
void oracle_step(const oracle_shape* sh, const float* Qc, const float* Qp, const float* K,
                 const float* V, const float* kmin, const float* kmax, const float* Kb,
                 const float* Vb, float* o_p, float* l_p, float* out, float* out_lse,
                 int* active_idx, int* page_idx, int* union_count, float* mse_out,
                 float* bound_out) {
    int d = sh->d, B = sh->B, A = sh->A, k = pages_per_row(sh), P = n_pages(sh);
    size_t rows = (size_t)sh->S * sh->Hq * B;
    float* mse = (float*)malloc(sizeof(float) * rows);
    float* U = (float*)malloc(sizeof(float) * (size_t)P);
    oracle_locality(sh, Qc, Qp, mse);
    oracle_active(sh, mse, active_idx);
    for (int s = 0; s < sh->S; ++s)
        for (int h = 0; h < sh->Hq; ++h) {
            int g = kv_head_of(sh, h);
            const float* mn = kmin + ((size_t)s * sh->Hkv + g) * (size_t)P * d;
            const float* mx = kmax + ((size_t)s * sh->Hkv + g) * (size_t)P * d;
            for (int a = 0; a < A; ++a) {
                int t = active_idx[((size_t)s * sh->Hq + h) * A + a];
                size_t r = ((size_t)s * sh->Hq + h) * B + t;
                oracle_bound_scores(d, P, Qc + r * d, mn, mx, U);
                oracle_topk_pages(P, k, U, page_idx + (((size_t)s * sh->Hq + h) * A + a) * k);
                if (bound_out)
                    memcpy(bound_out + (((size_t)s * sh->Hq + h) * A + a) * (size_t)P, U,
                           sizeof(float) * (size_t)P);
            }
        }
    if (mse_out) memcpy(mse_out, mse, sizeof(float) * rows);
    free(mse); free(U);
    oracle_step_forced(sh, Qc, K, V, Kb, Vb, active_idx, page_idx, o_p, l_p, out, out_lse,
                       union_count);
}

/* ------------------------------------------------------------------------
 * Drift-safe locality (a variant; the pages score locality between steps
 * t-1 and t, methodology: locality pruning).  A stable row keeps the prefix
 * state computed from the query it had when it was last recomputed, so the
 * variant scores each token against that reference query instead of the
 * previous step's.  oracle_step is run with q_ref in place of Qp; this then
 * moves the recomputed (active) rows' current queries into q_ref
 * [S][Hq][B][d]; the other rows keep their reference.
 * ---------------------------------------------------------------------- */
void oracle_refresh_ref(const oracle_shape* sh, const float* Qc, const int* active_idx,
                        float* q_ref) {
    int d = sh->d, B = sh->B, A = sh->A;
    for (int s = 0; s < sh->S; ++s)
        for (int h = 0; h < sh->Hq; ++h)
            for (int a = 0; a < A; ++a) {
                int t = active_idx[((size_t)s * sh->Hq + h) * A + a];
                size_t r = ((size_t)s * sh->Hq + h) * B + t;
                if (MUT(11)) r = ((size_t)s * sh->Hq + h) * B + (t + 1) % B;
                memcpy(q_ref + r * d, Qc + r * d, sizeof(float) * (size_t)d);
            }
}
