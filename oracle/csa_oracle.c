/*
 * Plain fp64 CPU oracle for the CSA / HCA hot path of DeepSeek-V4 hybrid attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this
 * file: only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Every function is the definition written out as directly as possible, one loop per
 * index of the formula, in double precision, single-threaded.  No blocking, fusion or
 * reordering beyond what the formula states.
 *
 * Sources (page title, then section / equation):
 *   [P1] "DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch"
 *   [P4] bhhxx.wiki "MHA -> ... -> CSA/HCA" (Chinese), section 6.2.2
 *
 * Parity pins (tests/test_oracle_pins.py): the six-token worked example of [P1] in
 * closed form, the printed softmax vectors, invariants of softmax pooling, brute force
 * against library routines on tiny inputs, and the KV-cache ledger of [P1] section 12.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------
 * Projection  out[i][j] = sum_k H[i][k] * W[k][j]
 * [P1] section 3 (C^a = H W^{aKV}, ...), section 6.1-6.3 (c^Q, q^I, w^I), section 8
 * (q = c^Q W^{UQ}), section 10 (C = H W^{KV}, Z = H W^Z).
 * H: [n, d] row-major; W: [d, c]; out: [n, c].
 * ---------------------------------------------------------------------------------- */
void oracle_project(const double* H, const double* W, int64_t n, int64_t d, int64_t c,
                    double* out)
{
    for (int64_t i = 0; i < n; ++i)
        for (int64_t j = 0; j < c; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < d; ++k) acc += H[i * d + k] * W[k * c + j];
            out[i * c + j] = acc;
        }
}

/* ------------------------------------------------------------------------------------
 * CSA overlapped compressor, [P1] section 4 (overlapping 2m-softmax) and the boxed
 * weighted sum of section 5; [P4] section 6.2.2 "compressor path" for the same sum.
 *
 * For compressed entry i and column j the 2m logits are
 *     Z^a[m*i + r][j] + B^a[r][j]          r = 0..m-1   (current block, stream a)
 *     Z^b[m*(i-1) + r][j] + B^b[r][j]      r = 0..m-1   (previous block, stream b)
 * normalised jointly by one softmax over all 2m rows of that column ([P1] section 4:
 * "for each of the c output columns independently, normalize across the 2m stacked
 * rows").  For i = 0 the b-rows do not exist: their logits are -infinity and their
 * values zero ([P1] section 4, padding rule), so they take weight exactly 0.
 * The entry is sum_r S^a_r * C^a[m*i + r][j] + sum_r S^b_r * C^b[m*(i-1) + r][j].
 *
 * Streams Ca, Cb, Za, Zb: [n, c] row-major (token rows).  Ba, Bb: [m, c] or NULL
 * (NULL means zero bias).  Entries i0 <= i < i1 are written to out[(i - i0) * c + j].
 * The caller guarantees m * i1 <= n.
 * ---------------------------------------------------------------------------------- */
void oracle_csa_compress(const double* Ca, const double* Cb, const double* Za,
                         const double* Zb, const double* Ba, const double* Bb, int64_t n,
                         int64_t c, int64_t m, int64_t i0, int64_t i1, double* out)
{
    (void)n;
    double* logit = (double*)malloc(sizeof(double) * 2 * m);
    double* value = (double*)malloc(sizeof(double) * 2 * m);
    int* present = (int*)malloc(sizeof(int) * 2 * m);
    for (int64_t i = i0; i < i1; ++i) {
        for (int64_t j = 0; j < c; ++j) {
            /* stack the 2m candidates: a-rows first, then b-rows */
            for (int64_t r = 0; r < m; ++r) {
                int64_t row = m * i + r;
                logit[r] = Za[row * c + j] + (Ba ? Ba[r * c + j] : 0.0);
                value[r] = Ca[row * c + j];
                present[r] = 1;
            }
            for (int64_t r = 0; r < m; ++r) {
                int64_t row = m * (i - 1) + r;
                if (i == 0) {            /* padded: logit -inf, value 0 */
                    logit[m + r] = -INFINITY;
                    value[m + r] = 0.0;
                    present[m + r] = 0;
                } else {
                    logit[m + r] = Zb[row * c + j] + (Bb ? Bb[r * c + j] : 0.0);
                    value[m + r] = Cb[row * c + j];
                    present[m + r] = 1;
                }
            }
            /* softmax over the 2m stacked rows (max-subtracted for range only) */
            double mx = -INFINITY;
            for (int64_t r = 0; r < 2 * m; ++r)
                if (present[r] && logit[r] > mx) mx = logit[r];
            double denom = 0.0;
            for (int64_t r = 0; r < 2 * m; ++r)
                if (present[r]) denom += exp(logit[r] - mx);
            double acc = 0.0;
            for (int64_t r = 0; r < 2 * m; ++r) {
                double s = present[r] ? exp(logit[r] - mx) / denom : 0.0;
                acc += s * value[r];
            }
            out[(i - i0) * c + j] = acc;
        }
    }
    free(logit);
    free(value);
    free(present);
}

/* ------------------------------------------------------------------------------------
 * HCA compressor, [P1] section 10 (boxed equations); [P4] section 6.1 compressor path.
 * Non-overlapping blocks of m' tokens, one stream, per-column softmax over the m' rows
 * of Z + B, weighted sum of the matching rows of C.
 * C, Z: [n, c]; Bias: [m', c] or NULL.  Entries i0 <= i < i1 -> out[(i - i0) * c + j].
 * ---------------------------------------------------------------------------------- */
void oracle_hca_compress(const double* C, const double* Z, const double* Bias, int64_t n,
                         int64_t c, int64_t mp, int64_t i0, int64_t i1, double* out)
{
    (void)n;
    for (int64_t i = i0; i < i1; ++i) {
        for (int64_t j = 0; j < c; ++j) {
            double mx = -INFINITY;
            for (int64_t r = 0; r < mp; ++r) {
                double l = Z[(mp * i + r) * c + j] + (Bias ? Bias[r * c + j] : 0.0);
                if (l > mx) mx = l;
            }
            double denom = 0.0;
            for (int64_t r = 0; r < mp; ++r) {
                double l = Z[(mp * i + r) * c + j] + (Bias ? Bias[r * c + j] : 0.0);
                denom += exp(l - mx);
            }
            double acc = 0.0;
            for (int64_t r = 0; r < mp; ++r) {
                double l = Z[(mp * i + r) * c + j] + (Bias ? Bias[r * c + j] : 0.0);
                acc += exp(l - mx) / denom * C[(mp * i + r) * c + j];
            }
            out[(i - i0) * c + j] = acc;
        }
    }
}

/* ------------------------------------------------------------------------------------
 * Causal visibility, [P1] section 7: query t sees compressed entries s < floor(t / m)
 * (for HCA, s < floor(t / m'), [P1] section 10).  Entries beyond the cache capacity
 * N_cap do not exist, so the count is capped there.
 * ---------------------------------------------------------------------------------- */
int64_t oracle_visible(int64_t t, int64_t m, int64_t N_cap)
{
    if (t < 0) return 0;
    int64_t v = t / m;
    return v < N_cap ? v : N_cap;
}

/* ------------------------------------------------------------------------------------
 * Lightning-indexer score, [P1] section 6.4 (boxed):
 *     I[t][s] = sum_h w^I[h] * ReLU(q^I[h] . K^I[s])
 * qI: [n_hI, cI], wI: [n_hI], KI: [nvis, cI]  ->  scores[s], s < nvis.
 * ---------------------------------------------------------------------------------- */
void oracle_index_scores(const double* qI, const double* wI, const double* KI, int64_t nvis,
                         int64_t n_hI, int64_t cI, double* scores)
{
    for (int64_t s = 0; s < nvis; ++s) {
        double total = 0.0;
        for (int64_t h = 0; h < n_hI; ++h) {
            double dot = 0.0;
            for (int64_t j = 0; j < cI; ++j) dot += qI[h * cI + j] * KI[s * cI + j];
            double relu = dot > 0.0 ? dot : 0.0;
            total += wI[h] * relu;
        }
        scores[s] = total;
    }
}

/* ------------------------------------------------------------------------------------
 * Top-k selection, [P1] section 7: keep the k entries of largest score among the
 * visible ones.  Ties (silent on the pages) go to the smaller index: a full sort of
 * (-score, s) pairs, first min(k, nvis) taken, the rest of idx padded with -1.
 * The selection is written in sorted order (score descending, index ascending).
 * ---------------------------------------------------------------------------------- */
typedef struct {
    double score;
    int64_t s;
} oracle_pair;

static int oracle_pair_cmp(const void* x, const void* y)
{
    const oracle_pair* a = (const oracle_pair*)x;
    const oracle_pair* b = (const oracle_pair*)y;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    if (a->s < b->s) return -1;
    if (a->s > b->s) return 1;
    return 0;
}

void oracle_topk(const double* scores, int64_t nvis, int64_t k, int32_t* idx)
{
    oracle_pair* p = (oracle_pair*)malloc(sizeof(oracle_pair) * (nvis > 0 ? nvis : 1));
    for (int64_t s = 0; s < nvis; ++s) {
        p[s].score = scores[s];
        p[s].s = s;
    }
    qsort(p, (size_t)nvis, sizeof(oracle_pair), oracle_pair_cmp);
    for (int64_t r = 0; r < k; ++r) idx[r] = r < nvis ? (int32_t)p[r].s : -1;
    free(p);
}

/* ------------------------------------------------------------------------------------
 * Shared-KV multi-query attention over a chosen set of compressed entries,
 * [P1] section 8:  o[h] = sum_{s in sel} Softmax_s(q[h] . C[s] * scale) * C[s]
 * with key = value = the compressed entry, scale = 1/sqrt(c) on the pages.
 * HCA's dense attention ([P1] section 10) is the same with sel = all visible entries.
 *
 * q: [n_h, c]; cache: [N, c]; sel: [nsel] entry ids, entries < 0 are padding and are
 * skipped.  out: [n_h, c]; lse: [n_h] natural-log sum of exp(logits), or NULL.
 * With no valid entry the output row is 0 and lse is -infinity (pages silent).
 * ---------------------------------------------------------------------------------- */
void oracle_mqa(const double* q, const double* cache, const int32_t* sel, int64_t nsel,
                int64_t n_h, int64_t c, double scale, double* out, double* lse)
{
    double* logit = (double*)malloc(sizeof(double) * (nsel > 0 ? nsel : 1));
    for (int64_t h = 0; h < n_h; ++h) {
        double mx = -INFINITY;
        for (int64_t r = 0; r < nsel; ++r) {
            if (sel[r] < 0) continue;
            double dot = 0.0;
            for (int64_t j = 0; j < c; ++j) dot += q[h * c + j] * cache[(int64_t)sel[r] * c + j];
            logit[r] = dot * scale;
            if (logit[r] > mx) mx = logit[r];
        }
        for (int64_t j = 0; j < c; ++j) out[h * c + j] = 0.0;
        if (mx == -INFINITY) {
            if (lse) lse[h] = -INFINITY;
            continue;
        }
        double denom = 0.0;
        for (int64_t r = 0; r < nsel; ++r)
            if (sel[r] >= 0) denom += exp(logit[r] - mx);
        for (int64_t r = 0; r < nsel; ++r) {
            if (sel[r] < 0) continue;
            double p = exp(logit[r] - mx) / denom;
            for (int64_t j = 0; j < c; ++j) out[h * c + j] += p * cache[(int64_t)sel[r] * c + j];
        }
        if (lse) lse[h] = mx + log(denom);
    }
    free(logit);
}

/* Sliding-window branch: the raw-token positions the query at position t attends to
 * besides the compressed entries.  bhhxx.wiki "MHA -> ... -> CSA/HCA", section 6 (HCA and
 * CSA paths) defines W_t = {max(1, t - n_window + 1), ..., t} on 1-based positions; with
 * this library's 0-based positions that is {max(0, t - n_win + 1), ..., t}, the current
 * token included.  Writes the positions in ascending order into pos (capacity n_win)
 * and returns their count (0 when t < 0 or n_win <= 0). */
int64_t oracle_window(int64_t t, int64_t n_win, int64_t* pos)
{
    if (t < 0 || n_win <= 0) return 0;
    int64_t lo = t - n_win + 1;
    if (lo < 0) lo = 0;
    int64_t n = 0;
    for (int64_t p = lo; p <= t; ++p) pos[n++] = p;
    return n;
}
