/*
 * hils_oracle.c -- float64 CPU reference of the forward pass of Hierarchical
 * Landmark Sparse (HiLS) attention.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
 * baseline load this file.  It shares no code, header, table or helper with the
 * CUDA library, and nothing in the library calls it.
 *
 * Source: "Hierarchical Sparse Attention Done Right: Toward Infinite Context
 * Modeling" (arXiv 2607.02980v1, paperlayer summary page):
 *   - Abstract: each query attends independently inside every retrieved chunk,
 *     and the per-chunk outputs are fused according to the chunk retrieval
 *     scores.
 *   - Sec. 3 Methodology, "Sparse training": a query scores every chunk summary
 *     and keeps the top-K chunks; only the selected tokens are touched.
 *   - Sec. 3 Methodology, "Hierarchical softmax": normalisation inside each
 *     chunk, then a softmax over the chunks' surrogate masses.
 *   - Sec. 4 Practical Design Choices, "Architecture" (GQA): the query heads of
 *     one group share one retrieved chunk set.
 *   - Sec. 2 Preliminary: chunks are a uniform partition of the sequence.
 * The surrogate mass used here is the scaled query-landmark dot product
 * q.L_c / sqrt(d) (the entropy bias the summary mentions is not part of this
 * definition); the query's own chunk is always fused in addition to the K
 * retrieved past chunks, causally masked.
 *
 * Readings where the page is silent (the plainest ones the rest of the page
 * supports):
 *   - one scale (1/sqrt(d) by default) for retrieval scores and token logits;
 *   - the own chunk c_i = floor(p_i / C) is scored with its own landmark;
 *   - a query with fewer than K past chunks takes all of them;
 *   - GQA selection ranks chunks by the mean over the group's heads of the
 *     per-head scores, while the fusion weights stay per head.  The pages do
 *     not fix this group rule: parity unpinned for G > 1 selection;
 *   - exact score ties go to the lower chunk index.
 *
 * Everything is float64, loops run in index order, no blocking or fusion.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- planted-mistake hook -------------------------------------------------
 * Zero in normal use.  The pin-strength tests set it to plant one known
 * mistake at a time and check that some pin fails.  Each use below is marked
 * "planted mistake N".                                                      */
static int g_mutant = 0;
void hils_oracle_set_mutant(int m) { g_mutant = m; }
#define PLANTED(n) (g_mutant == (n))

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += a[t] * b[t];
    return s;
}

/* Does candidate (sa, ia) rank before (sb, ib)?  Higher score first; equal
 * scores: lower chunk index first. */
static int ranks_before(double sa, int ia, double sb, int ib)
{
    if (sa != sb) return sa > sb;
    if (PLANTED(3)) return ia > ib;               /* planted mistake 3: ties to the higher index */
    return ia < ib;
}

/* Retrieval score of chunk landmark Lc for one head (Sec. 3, surrogate mass). */
static double retrieval_score(const double *qh, const double *Lc, int d, double scale)
{
    if (PLANTED(1)) return dot(qh, Lc, d);        /* planted mistake 1: scale dropped */
    return scale * dot(qh, Lc, d);
}

/* Group score of chunks 0..n_cand-1: mean over the G heads of the per-head
 * retrieval scores.  q is [G][d], L is [n_cand][d]. */
void hils_oracle_group_scores(int G, int d, int n_cand, double scale,
                              const double *q, const double *L, double *shat)
{
    for (int c = 0; c < n_cand; ++c) {
        const double *Lc = L + (size_t)(PLANTED(11) ? (c + 1 < n_cand ? c + 1 : c) : c) * d;
                                                  /* planted mistake 11: neighbouring landmark */
        double s = 0.0;
        for (int h = 0; h < G; ++h) s += retrieval_score(q + (size_t)h * d, Lc, d, scale);
        shat[c] = s / G;
    }
}

/* Top-k of the n_past candidates 0..n_past-1 by repeated selection of the best
 * remaining one.  Writes min(k, n_past) indices in rank order, then -1.
 * Returns the number selected. */
int hils_oracle_topk(int n_past, int k, const double *shat, int *sel)
{
    int m = k < n_past ? k : n_past;
    char *used = (char *)calloc((size_t)(n_past > 0 ? n_past : 1), 1);
    for (int j = 0; j < m; ++j) {
        int best = -1;
        for (int c = 0; c < n_past; ++c)
            if (!used[c] && (best < 0 || ranks_before(shat[c], c, shat[best], best))) best = c;
        sel[j] = best;
        used[best] = 1;
    }
    for (int j = m; j < k; ++j) sel[j] = -1;
    free(used);
    return m;
}

/* Chunk selection for one query group.
 *   q    [G][d]        queries of the group's heads at position pos
 *   L    [c_i+1][d]    landmarks of chunks 0..c_i, c_i = pos / C
 *   sel  [k+1]         out: top-k past chunks in rank order (-1 padded), then c_i
 *   shat [c_i+1]       out (may be NULL): group scores of chunks 0..c_i        */
void hils_oracle_select(int G, int d, int C, int k, long pos, double scale,
                        const double *q, const double *L, int *sel, double *shat_out)
{
    int ci = (int)(pos / C);
    double *shat = (double *)malloc(sizeof(double) * (size_t)(ci + 1));
    hils_oracle_group_scores(G, d, ci + 1, scale, q, L, shat);
    int n_past = PLANTED(6) ? ci + 1 : ci;        /* planted mistake 6: own chunk also a candidate */
    hils_oracle_topk(n_past, k, shat, sel);
    sel[k] = ci;
    if (shat_out) memcpy(shat_out, shat, sizeof(double) * (size_t)(ci + 1));
    free(shat);
}

/* Attention inside the selected chunks and their fusion, for one query group.
 *   q     [G][d]
 *   sel   [k+1]        chunk per slot (-1 = empty slot), slot k = own chunk
 *   Lsel  [k+1][d]     landmark of each slot's chunk
 *   Ksel, Vsel [k+1][C][d]  key/value rows c*C .. c*C+C-1 of each slot's chunk
 *   s     [G][k+1]     out: per-head retrieval score of each slot (-inf if empty)
 *   w     [G][k+1]     out: fusion weight of each slot (0 if empty)
 *   o     [G][d]       out: fused output
 *   oc    [G][k+1][d]  out (may be NULL): per-chunk outputs                   */
void hils_oracle_attend(int G, int d, int C, int k, long pos, double scale,
                        const double *q, const int *sel, const double *Lsel,
                        const double *Ksel, const double *Vsel,
                        double *s, double *w, double *o, double *oc)
{
    int ns = k + 1;
    double *ochunk = (double *)calloc((size_t)ns * d, sizeof(double));
    double *logit = (double *)malloc(sizeof(double) * (size_t)C);
    for (int h = 0; h < G; ++h) {
        const double *qh = q + (size_t)h * d;
        double *sh = s + (size_t)h * ns, *wh = w + (size_t)h * ns, *oh = o + (size_t)h * d;
        memset(ochunk, 0, sizeof(double) * (size_t)ns * d);
        for (int j = 0; j < ns; ++j) {
            int c = sel[j];
            if (c < 0 || (PLANTED(4) && j == k)) { sh[j] = -INFINITY; continue; }
                                                  /* planted mistake 4: own chunk dropped */
            sh[j] = retrieval_score(qh, Lsel + (size_t)j * d, d, scale);
            /* tokens of chunk c visible to the query: positions c*C+t <= pos */
            long first = (long)c * C;
            int n_vis = 0;
            for (int t = 0; t < C; ++t) {
                int visible = PLANTED(2) ? (first + t < pos) : (first + t <= pos);
                                                  /* planted mistake 2: query's own token masked */
                if (!visible) break;
                logit[t] = scale * dot(qh, Ksel + ((size_t)j * C + t) * d, d);
                n_vis = t + 1;
            }
            if (n_vis == 0) { sh[j] = -INFINITY; continue; }
            /* softmax over the visible tokens of this chunk only (Sec. 3, intra-chunk normalisation) */
            double m = logit[0];
            for (int t = 1; t < n_vis; ++t) if (logit[t] > m) m = logit[t];
            double den = 0.0;
            for (int t = 0; t < n_vis; ++t) den += exp(logit[t] - m);
            const double *Vj = PLANTED(7) ? Ksel : Vsel;   /* planted mistake 7: keys used as values */
            double *ocj = ochunk + (size_t)j * d;
            for (int t = 0; t < n_vis; ++t) {
                double p = exp(logit[t] - m) / den;
                const double *vt = Vj + ((size_t)j * C + t) * d;
                for (int x = 0; x < d; ++x) ocj[x] += p * vt[x];
            }
        }
        /* fusion: softmax over the selected chunks' retrieval scores (Abstract; Sec. 3) */
        double M = -INFINITY;
        for (int j = 0; j < ns; ++j) if (sh[j] > M) M = sh[j];
        double Z = 0.0;
        for (int j = 0; j < ns; ++j) wh[j] = (sh[j] == -INFINITY) ? 0.0 : exp(sh[j] - M);
        for (int j = 0; j < ns; ++j) Z += wh[j];
        for (int j = 0; j < ns; ++j) wh[j] /= Z;
        for (int x = 0; x < d; ++x) oh[x] = 0.0;
        for (int j = 0; j < ns; ++j)
            for (int x = 0; x < d; ++x) oh[x] += wh[j] * ochunk[(size_t)j * d + x];
        if (PLANTED(9)) {
            /* planted mistake 9: one softmax over all selected tokens jointly
             * (the flat block-sparse normalisation), no per-chunk fusion */
            double mm = -INFINITY, zz = 0.0;
            for (int x = 0; x < d; ++x) oh[x] = 0.0;
            for (int pass = 0; pass < 2; ++pass)
                for (int j = 0; j < ns; ++j) {
                    int c = sel[j];
                    if (c < 0) continue;
                    for (int t = 0; t < C && (long)c * C + t <= pos; ++t) {
                        double l = scale * dot(qh, Ksel + ((size_t)j * C + t) * d, d);
                        if (pass == 0) { if (l > mm) mm = l; continue; }
                        double p = exp(l - mm);
                        zz += p;
                        for (int x = 0; x < d; ++x) oh[x] += p * Vsel[((size_t)j * C + t) * d + x];
                    }
                }
            for (int x = 0; x < d; ++x) oh[x] /= zz;
        }
        if (oc) memcpy(oc + (size_t)h * ns * d, ochunk, sizeof(double) * (size_t)ns * d);
    }
    free(logit);
    free(ochunk);
}

/* Alternative selections under near ties.  Given the group scores of the
 * n_past candidates, the primary selection is hils_oracle_topk.  With t the
 * score of its last member, every candidate within eps of t may be swapped for
 * another such candidate by a computation whose scores err by less than eps/2.
 * Writes each alternative (k entries, rank order, -1 padded) to alts and
 * returns their number, or -1 if there are more than max_alts.  The first
 * alternative is the primary selection. */
int hils_oracle_tie_alternatives(int n_past, int k, const double *shat, double eps,
                                 int max_alts, int *alts)
{
    int *prim = (int *)malloc(sizeof(int) * (size_t)(k > 0 ? k : 1));
    int m = hils_oracle_topk(n_past, k, shat, prim);
    if (m == 0 || max_alts < 1) {
        if (max_alts >= 1) memcpy(alts, prim, sizeof(int) * (size_t)k);
        free(prim);
        return max_alts >= 1 ? 1 : -1;
    }
    double t = shat[prim[m - 1]];
    int n_fixed = 0, n_band = 0;
    int *band = (int *)malloc(sizeof(int) * (size_t)n_past);
    for (int c = 0; c < n_past; ++c) {
        if (shat[c] > t + eps) ++n_fixed;
        else if (fabs(shat[c] - t) <= eps) band[n_band++] = c;
    }
    int free_slots = m - n_fixed;
    /* count C(n_band, free_slots) with an early exit */
    double cnt = 1.0;
    for (int i = 0; i < free_slots; ++i) cnt = cnt * (n_band - i) / (i + 1);
    if (cnt > max_alts + 0.5) { free(band); free(prim); return -1; }
    int n_alt = 0;
    int *comb = (int *)malloc(sizeof(int) * (size_t)(free_slots > 0 ? free_slots : 1));
    for (int i = 0; i < free_slots; ++i) comb[i] = i;
    double *sub = (double *)malloc(sizeof(double) * (size_t)n_past);
    for (;;) {
        /* chosen set = fixed members + band[comb[...]]; rank it with the same order */
        for (int c = 0; c < n_past; ++c) sub[c] = -INFINITY;
        for (int c = 0; c < n_past; ++c) if (shat[c] > t + eps) sub[c] = shat[c];
        for (int i = 0; i < free_slots; ++i) sub[band[comb[i]]] = shat[band[comb[i]]];
        int *dst = alts + (size_t)n_alt * k;
        char *used = (char *)calloc((size_t)n_past, 1);
        for (int j = 0; j < m; ++j) {
            int best = -1;
            for (int c = 0; c < n_past; ++c)
                if (!used[c] && sub[c] != -INFINITY && (best < 0 || ranks_before(sub[c], c, sub[best], best))) best = c;
            dst[j] = best;
            used[best] = 1;
        }
        for (int j = m; j < k; ++j) dst[j] = -1;
        free(used);
        ++n_alt;
        /* next combination in lexicographic order */
        int i = free_slots - 1;
        while (i >= 0 && comb[i] == n_band - free_slots + i) --i;
        if (i < 0) break;
        ++comb[i];
        for (int j = i + 1; j < free_slots; ++j) comb[j] = comb[j - 1] + 1;
    }
    /* move the primary selection to the front */
    for (int a = 0; a < n_alt; ++a)
        if (memcmp(alts + (size_t)a * k, prim, sizeof(int) * (size_t)k) == 0) {
            for (int j = 0; j < k; ++j) {
                int tmp = alts[j];
                alts[j] = alts[(size_t)a * k + j];
                alts[(size_t)a * k + j] = tmp;
            }
            break;
        }
    free(sub); free(comb); free(band); free(prim);
    return n_alt;
}

/* Whole forward pass.
 *   Q [B][H][N][d], K, V [B][Hkv][T][d], L [B][Hkv][nL][d] with nL = ceil(T/C)
 *   query i sits at position q_offset + i (< T); head h uses kv-head h / (H/Hkv)
 *   O [B][H][N][d]; sel [B][Hkv][N][k+1]; s, w [B][H][N][k+1] (any may be NULL)
 * Parallel over (b, g, i) with OpenMP when nthreads > 1.  Returns 0, or -1 on
 * an invalid shape. */
int hils_oracle_forward(int B, int H, int Hkv, int N, int T, int d, int C, int k,
                        long q_offset, double scale,
                        const double *Q, const double *K, const double *V, const double *L,
                        double *O, int *sel_out, double *s_out, double *w_out, int nthreads)
{
    if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || N < 0 || T <= 0 || d <= 0 || C <= 0 || k < 0)
        return -1;
    if (q_offset < 0 || q_offset + N > T) return -1;
    int G = H / Hkv, nL = (T + C - 1) / C, ns = k + 1;
    long n_items = (long)B * Hkv * N;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *q = (double *)malloc(sizeof(double) * (size_t)G * d);
        double *Ls = (double *)malloc(sizeof(double) * (size_t)ns * d);
        double *Ks = (double *)calloc((size_t)ns * C * d, sizeof(double));
        double *Vs = (double *)calloc((size_t)ns * C * d, sizeof(double));
        double *s = (double *)malloc(sizeof(double) * (size_t)G * ns);
        double *w = (double *)malloc(sizeof(double) * (size_t)G * ns);
        double *o = (double *)malloc(sizeof(double) * (size_t)G * d);
        int *sel = (int *)malloc(sizeof(int) * (size_t)ns);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
        for (long it = 0; it < n_items; ++it) {
            int i = (int)(it % N), g = (int)((it / N) % Hkv), b = (int)(it / ((long)N * Hkv));
            long pos = q_offset + i;
            for (int h = 0; h < G; ++h)
                memcpy(q + (size_t)h * d, Q + ((((size_t)b * H + (size_t)g * G + h) * N) + i) * d,
                       sizeof(double) * (size_t)d);
            const double *Lbg = L + ((size_t)b * Hkv + g) * nL * d;
            const double *Kbg = K + ((size_t)b * Hkv + g) * T * d;
            const double *Vbg = V + ((size_t)b * Hkv + g) * T * d;
            hils_oracle_select(G, d, C, k, pos, scale, q, Lbg, sel, NULL);
            for (int j = 0; j < ns; ++j) {
                int c = sel[j];
                if (c < 0) continue;
                memcpy(Ls + (size_t)j * d, Lbg + (size_t)c * d, sizeof(double) * (size_t)d);
                int rows = (c + 1) * C <= T ? C : T - c * C;
                memcpy(Ks + (size_t)j * C * d, Kbg + (size_t)c * C * d, sizeof(double) * (size_t)rows * d);
                memcpy(Vs + (size_t)j * C * d, Vbg + (size_t)c * C * d, sizeof(double) * (size_t)rows * d);
            }
            hils_oracle_attend(G, d, C, k, pos, scale, q, sel, Ls, Ks, Vs, s, w, o, NULL);
            for (int h = 0; h < G; ++h) {
                size_t row = (((size_t)b * H + (size_t)g * G + h) * N) + i;
                if (O) memcpy(O + row * d, o + (size_t)h * d, sizeof(double) * (size_t)d);
                if (s_out) memcpy(s_out + row * ns, s + (size_t)h * ns, sizeof(double) * (size_t)ns);
                if (w_out) memcpy(w_out + row * ns, w + (size_t)h * ns, sizeof(double) * (size_t)ns);
            }
            if (sel_out) memcpy(sel_out + ((((size_t)b * Hkv + g) * N) + i) * ns, sel, sizeof(int) * (size_t)ns);
        }
        free(q); free(Ls); free(Ks); free(Vs); free(s); free(w); free(o); free(sel);
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Extension for the next rows of the method (the local window and the bias of
 * the surrogate mass).  The functions above are unchanged; these reduce to them
 * with wc = 1 and no bias.
 *
 * Local window (Sec. 2 Preliminary: block-sparse attention combines a local
 * sliding window with K retrieved chunks, the window aligned to chunk
 * boundaries so that it never overlaps a retrieved chunk; Sec. 5, Experimental
 * setup: a 512-token window with 64-token chunks): the window is the query's own
 * chunk and the wc - 1 chunks before it; every one is attended like a retrieved
 * chunk and fused by the same softmax over retrieval scores, and retrieval
 * ranks only the chunks before the window.  (Reading: the pages do not say how
 * the window enters the fusion; treating its chunks as always-retrieved chunks
 * is the one that keeps a single hierarchical softmax, and with wc = 1 it is the
 * method above.)
 *
 * Bias (Sec. 3, Linear surrogate for chunk mass: an affine surrogate of the
 * chunk mass, query-summary relevance plus an entropy-based bias per chunk):
 * bias[c] is added to every head's retrieval score of chunk c, so to the group
 * score as well; the fusion weights use the biased scores.
 * ------------------------------------------------------------------------- */

/* Selection with a window of wc >= 1 chunks for one query group.
 *   q    [G][d], L [c_i+1][d], bias [c_i+1] or NULL
 *   sel  [k+wc]   out: top-min(k, #candidates) of chunks 0..c_i-wc in rank order
 *                 (-1 padded), then the window chunks c_i-wc+1 .. c_i ascending
 *                 (-1 for the ones before chunk 0)
 *   shat [c_i+1]  out (may be NULL): biased group scores of chunks 0..c_i      */
void hils_oracle_select_window(int G, int d, int C, int k, int wc, long pos, double scale,
                               const double *q, const double *L, const double *bias, int *sel,
                               double *shat_out)
{
    int ci = (int)(pos / C);
    double *shat = (double *)malloc(sizeof(double) * (size_t)(ci + 1));
    hils_oracle_group_scores(G, d, ci + 1, scale, q, L, shat);
    if (bias)
        for (int c = 0; c <= ci; ++c) shat[c] += bias[c];
    int n_cand = PLANTED(14) ? ci : ci - wc + 1;  /* planted mistake 14: window chunks also candidates */
    if (n_cand < 0) n_cand = 0;
    hils_oracle_topk(n_cand, k, shat, sel);
    for (int j = 0; j < wc; ++j) {
        int c = ci - wc + 1 + j - (PLANTED(12) ? 1 : 0);   /* planted mistake 12: window one chunk early */
        sel[k + j] = c >= 0 ? c : -1;
    }
    if (shat_out) memcpy(shat_out, shat, sizeof(double) * (size_t)(ci + 1));
    free(shat);
}

/* Attention inside ns slots and their fusion, for one query group.
 *   sel [ns] chunk per slot (-1 = empty); Lsel [ns][d]; bsel [ns] or NULL: the
 *   slots' biases; Ksel, Vsel [ns][C][d]; s, w [G][ns]; o [G][d] (as
 *   hils_oracle_attend, with s_{h,c} = scale q_h . L_c + bias_c).             */
void hils_oracle_attend_slots(int G, int d, int C, int ns, long pos, double scale,
                              const double *q, const int *sel, const double *Lsel, const double *bsel,
                              const double *Ksel, const double *Vsel, double *s, double *w, double *o)
{
    double *ochunk = (double *)calloc((size_t)ns * d, sizeof(double));
    double *logit = (double *)malloc(sizeof(double) * (size_t)C);
    for (int h = 0; h < G; ++h) {
        const double *qh = q + (size_t)h * d;
        double *sh = s + (size_t)h * ns, *wh = w + (size_t)h * ns, *oh = o + (size_t)h * d;
        memset(ochunk, 0, sizeof(double) * (size_t)ns * d);
        for (int j = 0; j < ns; ++j) {
            int c = sel[j];
            if (c < 0) { sh[j] = -INFINITY; continue; }
            sh[j] = retrieval_score(qh, Lsel + (size_t)j * d, d, scale) + ((bsel && !PLANTED(13)) ? bsel[j] : 0.0);
                                                  /* planted mistake 13: bias left out of the fusion */
            long first = (long)c * C;
            int n_vis = 0;
            for (int t = 0; t < C && first + t <= pos; ++t) {
                logit[t] = scale * dot(qh, Ksel + ((size_t)j * C + t) * d, d);
                n_vis = t + 1;
            }
            if (n_vis == 0) { sh[j] = -INFINITY; continue; }
            double m = logit[0];
            for (int t = 1; t < n_vis; ++t) if (logit[t] > m) m = logit[t];
            double den = 0.0;
            for (int t = 0; t < n_vis; ++t) den += exp(logit[t] - m);
            double *ocj = ochunk + (size_t)j * d;
            for (int t = 0; t < n_vis; ++t) {
                double p = exp(logit[t] - m) / den;
                const double *vt = Vsel + ((size_t)j * C + t) * d;
                for (int x = 0; x < d; ++x) ocj[x] += p * vt[x];
            }
        }
        double M = -INFINITY;
        for (int j = 0; j < ns; ++j) if (sh[j] > M) M = sh[j];
        double Z = 0.0;
        for (int j = 0; j < ns; ++j) wh[j] = (sh[j] == -INFINITY) ? 0.0 : exp(sh[j] - M);
        for (int j = 0; j < ns; ++j) Z += wh[j];
        for (int j = 0; j < ns; ++j) wh[j] /= Z;
        for (int x = 0; x < d; ++x) oh[x] = 0.0;
        for (int j = 0; j < ns; ++j)
            for (int x = 0; x < d; ++x) oh[x] += wh[j] * ochunk[(size_t)j * d + x];
    }
    free(logit);
    free(ochunk);
}

/* Whole forward pass with a window of wc chunks and an optional bias
 * [B][Hkv][nL]; layouts as hils_oracle_forward with k+wc slots per query. */
int hils_oracle_forward_window(int B, int H, int Hkv, int N, int T, int d, int C, int k, int wc,
                               long q_offset, double scale,
                               const double *Q, const double *K, const double *V, const double *L,
                               const double *bias, double *O, int *sel_out, double *s_out, double *w_out,
                               int nthreads)
{
    if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv || N < 0 || T <= 0 || d <= 0 || C <= 0 || k < 0 || wc < 1)
        return -1;
    if (q_offset < 0 || q_offset + N > T) return -1;
    int G = H / Hkv, nL = (T + C - 1) / C, ns = k + wc;
    long n_items = (long)B * Hkv * N;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *q = (double *)malloc(sizeof(double) * (size_t)G * d);
        double *Ls = (double *)malloc(sizeof(double) * (size_t)ns * d);
        double *bs = (double *)malloc(sizeof(double) * (size_t)ns);
        double *Ks = (double *)calloc((size_t)ns * C * d, sizeof(double));
        double *Vs = (double *)calloc((size_t)ns * C * d, sizeof(double));
        double *s = (double *)malloc(sizeof(double) * (size_t)G * ns);
        double *w = (double *)malloc(sizeof(double) * (size_t)G * ns);
        double *o = (double *)malloc(sizeof(double) * (size_t)G * d);
        int *sel = (int *)malloc(sizeof(int) * (size_t)ns);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
        for (long it = 0; it < n_items; ++it) {
            int i = (int)(it % N), g = (int)((it / N) % Hkv), b = (int)(it / ((long)N * Hkv));
            long pos = q_offset + i;
            for (int h = 0; h < G; ++h)
                memcpy(q + (size_t)h * d, Q + ((((size_t)b * H + (size_t)g * G + h) * N) + i) * d,
                       sizeof(double) * (size_t)d);
            const double *Lbg = L + ((size_t)b * Hkv + g) * nL * d;
            const double *Kbg = K + ((size_t)b * Hkv + g) * T * d;
            const double *Vbg = V + ((size_t)b * Hkv + g) * T * d;
            const double *bbg = bias ? bias + ((size_t)b * Hkv + g) * nL : NULL;
            hils_oracle_select_window(G, d, C, k, wc, pos, scale, q, Lbg, bbg, sel, NULL);
            for (int j = 0; j < ns; ++j) {
                int c = sel[j];
                bs[j] = 0.0;
                if (c < 0) continue;
                bs[j] = bbg ? bbg[c] : 0.0;
                memcpy(Ls + (size_t)j * d, Lbg + (size_t)c * d, sizeof(double) * (size_t)d);
                int rows = (c + 1) * C <= T ? C : T - c * C;
                memcpy(Ks + (size_t)j * C * d, Kbg + (size_t)c * C * d, sizeof(double) * (size_t)rows * d);
                memcpy(Vs + (size_t)j * C * d, Vbg + (size_t)c * C * d, sizeof(double) * (size_t)rows * d);
            }
            hils_oracle_attend_slots(G, d, C, ns, pos, scale, q, sel, Ls, bbg ? bs : NULL, Ks, Vs, s, w, o);
            for (int h = 0; h < G; ++h) {
                size_t row = (((size_t)b * H + (size_t)g * G + h) * N) + i;
                if (O) memcpy(O + row * d, o + (size_t)h * d, sizeof(double) * (size_t)d);
                if (s_out) memcpy(s_out + row * ns, s + (size_t)h * ns, sizeof(double) * (size_t)ns);
                if (w_out) memcpy(w_out + row * ns, w + (size_t)h * ns, sizeof(double) * (size_t)ns);
            }
            if (sel_out) memcpy(sel_out + ((((size_t)b * Hkv + g) * N) + i) * ns, sel, sizeof(int) * (size_t)ns);
        }
        free(q); free(Ls); free(bs); free(Ks); free(Vs); free(s); free(w); free(o); free(sel);
    }
    return 0;
}

/* Landmarks and their biases from the chunks' keys (Sec. 3, Linear surrogate for
 * chunk mass: a landmark token appended to each chunk supplies a learned query;
 * that query's distribution over the chunk's keys weights the key sum that forms
 * the summary, and the entropy-based bias tends to log S for uniform scores and
 * to 0 when one score dominates).  For chunk c with landmark query u_c:
 *     p_t  = softmax_t(scale * u_c . k_t) over the chunk's keys (a partial last chunk
 *            uses the keys it has),
 *     L_c  = sum_t p_t k_t,
 *     beta_c = -sum_t p_t log p_t   (the entropy of p).
 * (Reading: the summary page names the ingredients, not the formula; this is the
 * plain one, and with it scale * q . L_c + beta_c never exceeds the chunk's
 * log-sum-exp mass log sum_t exp(scale * q . k_t), with equality for q = u_c.)
 *   K [T][d] of one (b, g); U [nL][d] landmark queries; L [nL][d], beta [nL] out. */
void hils_oracle_landmarks(int T, int d, int C, double scale, const double *K, const double *U,
                           double *L, double *beta)
{
    int nL = (T + C - 1) / C;
    double *sc = (double *)malloc(sizeof(double) * (size_t)C);
    for (int c = 0; c < nL; ++c) {
        int rows = (c + 1) * C <= T ? C : T - c * C;
        const double *u = U + (size_t)c * d;
        double m = -INFINITY;
        for (int t = 0; t < rows; ++t) {
            sc[t] = (PLANTED(15) ? 1.0 : scale) * dot(u, K + ((size_t)c * C + t) * d, d);
                                                  /* planted mistake 15: scale dropped from the landmark scores */
            if (sc[t] > m) m = sc[t];
        }
        double z = 0.0;
        for (int t = 0; t < rows; ++t) z += exp(sc[t] - m);
        double *Lc = L + (size_t)c * d, h = 0.0;
        for (int x = 0; x < d; ++x) Lc[x] = 0.0;
        for (int t = 0; t < rows; ++t) {
            double pt = exp(sc[t] - m) / z;
            const double *kt = K + ((size_t)c * C + t) * d;
            for (int x = 0; x < d; ++x) Lc[x] += pt * kt[x];
            if (pt > 0.0) h -= pt * log(pt);
        }
        beta[c] = PLANTED(16) ? -h : PLANTED(17) ? log((double)rows) : h;
                                                  /* planted mistakes 16, 17: entropy negated; log C always */
    }
    free(sc);
}

/* Threads the OpenMP runtime would use (1 without OpenMP). */
int hils_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
