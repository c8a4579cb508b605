/*
 * blasst_oracle.c -- plain, slow fp64 CPU oracle of BLASST's blocked attention
 * with softmax-threshold block skipping.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, __graft_entry__.smoke() and the
 * bench's CPU-baseline / reference legs may load this library.  It shares no
 * code, header, table or helper with the CUDA path in the package.
 *
 * What it computes (BLASST: "Dynamic BLocked Attention Sparsity via Softmax
 * Thresholding", arXiv:2512.12087):
 *   - attention = softmax(Q K^T * scale) V  (xllm-io review, section 3, the
 *     standard-attention formula);
 *   - FlashAttention-style pass over KV blocks in increasing order, keeping a
 *     running row max m, row sum l and accumulator (xllm-io review section 3,
 *     "solution overview"; nervesearch commentary on online softmax);
 *   - skip rule: a block j is skipped when its row max m~ and the running max
 *     after the block, m = max(m_prev, m~), satisfy m~ - m < ln(lambda)
 *     (xllm-io review section 3 skip condition exp(m~ - m) < lambda; gist.de
 *     section 2 "Kernidee"; gist.ja section 2.1);
 *   - the decision is taken for the whole tile: skip only if every row of the
 *     tile satisfies the rule (rows that see no key of the block abstain),
 *     i.e. skip <=> max_r (m~_r - m_r) < ln(lambda);
 *   - the first visited block of a tile (of a split, in decode) is never
 *     skipped (nervesearch commentary: six-block figure, "the first is always
 *     processed");  lambda = 0 means ln(lambda) = -inf: dense;
 *   - a skipped block adds nothing to l or O (gist.de section 2: the exp,
 *     the V block load and the P.V product are all omitted).
 * Readings where the pages are silent: strict "<"; causal alignment
 * bottom-right (query r sits at key r + Lk - Lq); decode tiles are all G = Hq/Hkv heads x Lq rows of one KV head;
 * decode splits are independent online-softmax passes over contiguous chunks
 * of ceil(nb/num_splits) blocks, merged exactly on lse; lse = M + ln(l) over
 * kept blocks, natural log.
 * Split seeding (decode, optional; not on the pages): every split after the
 * first starts its running max at the row maxima of block 0 instead of -inf
 * and has no forced first block.  Block 0 then adds nothing to that split's l
 * or O; only its maxima enter the comparison.  This is the single-pass rule
 * with the blocks between block 0 and the split start left out of the max.
 *
 * Everything is fp64: bf16 inputs are widened exactly.  Parallel over tiles
 * with OpenMP; each tile's arithmetic is a plain sequential loop nest.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_FORCED 2
#define ORACLE_NOMEM 3

static double bf16_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Number of query tiles and of KV blocks for the call. */
static void shape_counts(int is_decode, int B, int Hq, int Hkv, int Lq, int Lk, int BM, int BN,
                         long long *n_tiles, int *tiles_per_head, int *nb)
{
    int G = Hq / Hkv;
    *nb = (Lk + BN - 1) / BN;
    if (is_decode) {
        *tiles_per_head = (G * Lq + BM - 1) / BM;
        *n_tiles = (long long)B * Hkv * (*tiles_per_head);
    } else {
        *tiles_per_head = (Lq + BM - 1) / BM;
        *n_tiles = (long long)B * Hq * (*tiles_per_head);
    }
}

long long blasst_oracle_num_tiles(int is_decode, int B, int Hq, int Hkv, int Lq, int Lk, int BM, int BN)
{
    long long nt;
    int tph, nb;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lq <= 0 || Lk <= 0 || BM <= 0 || BN <= 0) return -1;
    shape_counts(is_decode, B, Hq, Hkv, Lq, Lk, BM, BN, &nt, &tph, &nb);
    return nt;
}

/*
 * One tile.  Rows of a prefill tile: queries t*BM .. of head hq.  Rows of a
 * decode tile: flat index rho = g*Lq + i over the G heads of KV head hkv and
 * the Lq queries, rows t*BM .. of that list.
 */
static int run_tile(long long tile, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv,
                    long long k_row_stride, long long v_row_stride,
                    double scale, double lambda, int causal, int BM, int BN, int is_decode, int num_splits,
                    int seed_splits, int tiles_per_head, int nb, const uint8_t *forced_skip,
                    double *o, double *lse, uint8_t *skip, uint8_t *visited, double *gaps,
                    long long *n_skipped, long long *n_visited)
{
    (void)B;
    const int G = Hq / Hkv;
    const double ln_lambda = lambda > 0.0 ? log(lambda) : -INFINITY;
    const int t = (int)(tile % tiles_per_head);
    const long long bh = tile / tiles_per_head;
    int b, hkv;
    if (is_decode) {
        b = (int)(bh / Hkv);
        hkv = (int)(bh % Hkv);
    } else {
        int hq = (int)(bh % Hq);
        b = (int)(bh / Hq);
        hkv = hq / G;
    }
    const int rows_total = is_decode ? G * Lq : Lq;
    const int r0 = t * BM;
    const int nrows = (rows_total - r0 < BM) ? rows_total - r0 : BM;

    /* Per row: which query head and query position it is. */
    int *row_head = malloc(sizeof(int) * nrows);
    int *row_pos = malloc(sizeof(int) * nrows);
    double *qrow = malloc(sizeof(double) * (size_t)nrows * d);
    double *s = malloc(sizeof(double) * (size_t)nrows * BN);
    double *M = malloc(sizeof(double) * nrows);
    double *Mn = malloc(sizeof(double) * nrows);
    double *mt = malloc(sizeof(double) * nrows);
    double *l = malloc(sizeof(double) * nrows);
    double *acc = malloc(sizeof(double) * (size_t)nrows * dv);
    /* decode: per-split partial results, merged at the end */
    int S = is_decode ? num_splits : 1;
    double *o_part = malloc(sizeof(double) * (size_t)S * nrows * dv);
    double *lse_part = malloc(sizeof(double) * (size_t)S * nrows);
    if (!row_head || !row_pos || !qrow || !s || !M || !Mn || !mt || !l || !acc || !o_part || !lse_part) {
        free(row_head); free(row_pos); free(qrow); free(s); free(M); free(Mn); free(mt); free(l);
        free(acc); free(o_part); free(lse_part);
        return ORACLE_NOMEM;
    }
    int status = ORACLE_OK;

    for (int r = 0; r < nrows; r++) {
        int rho = r0 + r;
        int hq, pos;
        if (is_decode) {
            hq = hkv * G + rho / Lq;
            pos = rho % Lq;
        } else {
            hq = (int)(bh % Hq);
            pos = rho;
        }
        row_head[r] = hq;
        row_pos[r] = pos;
        const uint16_t *qp = q + (((long long)b * Hq + hq) * Lq + pos) * d;
        for (int x = 0; x < d; x++) qrow[(size_t)r * d + x] = bf16_to_double(qp[x]);
    }

    const uint16_t *kbase = k + ((long long)b * Hkv + hkv) * (long long)Lk * k_row_stride;
    const uint16_t *vbase = v + ((long long)b * Hkv + hkv) * (long long)Lk * v_row_stride;
    const int per_split = (nb + S - 1) / S;
    long long my_skipped = 0, my_visited = 0;

    for (int sp = 0; sp < S; sp++) {
        int j0 = sp * per_split;
        int j1 = j0 + per_split < nb ? j0 + per_split : nb;
        for (int r = 0; r < nrows; r++) {
            M[r] = -INFINITY;
            l[r] = 0.0;
            for (int x = 0; x < dv; x++) acc[(size_t)r * dv + x] = 0.0;
        }
        int first = 1;
        if (is_decode && seed_splits && sp > 0 && j0 < j1) {
            /* seed: the running max starts at block 0's row maxima */
            for (int r = 0; r < nrows; r++) {
                int last_key = causal ? row_pos[r] + (Lk - Lq) : Lk - 1;
                double m = -INFINITY;
                for (int cc = 0; cc < BN; cc++) {
                    int key = cc;
                    if (key < Lk && key <= last_key) {
                        const uint16_t *kp = kbase + (long long)key * k_row_stride;
                        double dot = 0.0;
                        for (int x = 0; x < d; x++) dot += qrow[(size_t)r * d + x] * bf16_to_double(kp[x]);
                        if (scale * dot > m) m = scale * dot;
                    }
                }
                M[r] = m;
            }
            first = 0;
        }
        for (int j = j0; j < j1; j++) {
            long long pair = tile * nb + j;
            /* scores of the block; masked entries are -inf */
            int any_visible = 0;
            for (int r = 0; r < nrows; r++) {
                int last_key = causal ? row_pos[r] + (Lk - Lq) : Lk - 1;
                for (int cc = 0; cc < BN; cc++) {
                    int key = j * BN + cc;
                    double val = -INFINITY;
                    if (key < Lk && key <= last_key) {
                        const uint16_t *kp = kbase + (long long)key * k_row_stride;
                        double dot = 0.0;
                        for (int x = 0; x < d; x++) dot += qrow[(size_t)r * d + x] * bf16_to_double(kp[x]);
                        val = scale * dot;
                        any_visible = 1;
                    }
                    s[(size_t)r * BN + cc] = val;
                }
            }
            if (!any_visible) continue; /* block not visited by this tile */

            /* block row max, running max after the block, tile-wide gap */
            double gap = -INFINITY;
            for (int r = 0; r < nrows; r++) {
                double m = -INFINITY;
                for (int cc = 0; cc < BN; cc++)
                    if (s[(size_t)r * BN + cc] > m) m = s[(size_t)r * BN + cc];
                mt[r] = m;
                Mn[r] = M[r] > m ? M[r] : m;
                if (m > -INFINITY && m - Mn[r] > gap) gap = m - Mn[r];
            }
            int do_skip = (!first) && (lambda > 0.0) && (gap < ln_lambda);
            if (forced_skip) {
                do_skip = forced_skip[pair] != 0;
                if (first && do_skip) status = ORACLE_BAD_FORCED;
            }
            visited[pair] = 1;
            skip[pair] = (uint8_t)do_skip;
            gaps[pair] = first ? INFINITY : gap;
            my_visited++;
            my_skipped += do_skip;
            first = 0;
            if (do_skip) continue;

            /* online softmax update with the kept block */
            for (int r = 0; r < nrows; r++) {
                if (Mn[r] == -INFINITY) continue; /* row has seen nothing yet */
                double alpha = (M[r] == -INFINITY) ? 0.0 : exp(M[r] - Mn[r]);
                double *ar = acc + (size_t)r * dv;
                for (int x = 0; x < dv; x++) ar[x] *= alpha;
                l[r] *= alpha;
                for (int cc = 0; cc < BN; cc++) {
                    double sv = s[(size_t)r * BN + cc];
                    if (sv == -INFINITY) continue;
                    double p = exp(sv - Mn[r]);
                    l[r] += p;
                    const uint16_t *vp = vbase + (long long)(j * BN + cc) * v_row_stride;
                    for (int x = 0; x < dv; x++) ar[x] += p * bf16_to_double(vp[x]);
                }
                M[r] = Mn[r];
            }
        }
        for (int r = 0; r < nrows; r++) {
            double *op = o_part + ((size_t)sp * nrows + r) * dv;
            if (l[r] > 0.0) {
                for (int x = 0; x < dv; x++) op[x] = acc[(size_t)r * dv + x] / l[r];
                lse_part[(size_t)sp * nrows + r] = M[r] + log(l[r]);
            } else {
                for (int x = 0; x < dv; x++) op[x] = 0.0;
                lse_part[(size_t)sp * nrows + r] = -INFINITY;
            }
        }
    }

    /* merge splits on lse (prefill: S == 1, a copy) */
    for (int r = 0; r < nrows; r++) {
        double mx = -INFINITY;
        for (int sp = 0; sp < S; sp++)
            if (lse_part[(size_t)sp * nrows + r] > mx) mx = lse_part[(size_t)sp * nrows + r];
        double sum = 0.0;
        for (int sp = 0; sp < S; sp++) {
            double ls = lse_part[(size_t)sp * nrows + r];
            if (ls > -INFINITY) sum += exp(ls - mx);
        }
        double L_all = (mx > -INFINITY) ? mx + log(sum) : -INFINITY;
        long long orow = ((long long)b * Hq + row_head[r]) * Lq + row_pos[r];
        lse[orow] = L_all;
        double *out = o + orow * dv;
        for (int x = 0; x < dv; x++) out[x] = 0.0;
        for (int sp = 0; sp < S; sp++) {
            double ls = lse_part[(size_t)sp * nrows + r];
            if (ls == -INFINITY) continue;
            double w = exp(ls - L_all);
            const double *op = o_part + ((size_t)sp * nrows + r) * dv;
            for (int x = 0; x < dv; x++) out[x] += w * op[x];
        }
    }

    *n_skipped += my_skipped;
    *n_visited += my_visited;
    free(row_head); free(row_pos); free(qrow); free(s); free(M); free(Mn); free(mt); free(l);
    free(acc); free(o_part); free(lse_part);
    return status;
}

/*
 * Blocked attention with softmax-threshold skipping.
 *
 * q  [B, Hq, Lq, d]            bf16 bits, contiguous
 * k  [B, Hkv, Lk, *] rows of k_row_stride elements, the first d used
 * v  [B, Hkv, Lk, *] rows of v_row_stride elements, the first dv used
 * tiles / n_tiles: which tiles to compute (NULL: all); outputs of the other
 *     tiles are left untouched.
 * forced_skip [n_tiles_total * nb] or NULL: use this skip decision instead of
 *     the rule (marking a first block is an error, ORACLE_BAD_FORCED).
 * seed_splits: decode only; nonzero seeds the running max of every split
 *     after the first with block 0's row maxima (see the header).
 * Outputs: o [B, Hq, Lq, dv], lse [B, Hq, Lq] (natural log), and per
 *     (tile, block) pair: skip (1 = skipped), visited (1 = at least one
 *     unmasked score), gaps (max over voting rows of m~ - m; +inf on a first
 *     block; untouched if not visited).  counts[0] = skipped, counts[1] =
 *     visited, over the computed tiles.
 * Returns 0 on success.
 */
int blasst_oracle_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            int B, int Hq, int Hkv, int Lq, int Lk, int d, int dv,
                            long long k_row_stride, long long v_row_stride,
                            double scale, double lambda, int causal,
                            int BM, int BN, int is_decode, int num_splits, int seed_splits,
                            const long long *tiles, long long n_tiles, const uint8_t *forced_skip,
                            double *o, double *lse, uint8_t *skip, uint8_t *visited, double *gaps,
                            long long *counts)
{
    if (!q || !k || !v || !o || !lse || !skip || !visited || !gaps || !counts) return ORACLE_BAD_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || Lq <= 0 || Lk <= 0 || d <= 0 || dv <= 0) return ORACLE_BAD_ARG;
    if (BM <= 0 || BN <= 0 || k_row_stride < d || v_row_stride < dv) return ORACLE_BAD_ARG;
    if (!(lambda >= 0.0 && lambda < 1.0)) return ORACLE_BAD_ARG;
    if (causal && Lq > Lk) return ORACLE_BAD_ARG;
    if (!is_decode) num_splits = 1;
    if (num_splits <= 0) return ORACLE_BAD_ARG;

    long long nt_total;
    int tph, nb;
    shape_counts(is_decode, B, Hq, Hkv, Lq, Lk, BM, BN, &nt_total, &tph, &nb);
    long long n = tiles ? n_tiles : nt_total;
    for (long long i = 0; i < n; i++)
        if (tiles && (tiles[i] < 0 || tiles[i] >= nt_total)) return ORACLE_BAD_ARG;

    long long skipped = 0, vis = 0;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : skipped, vis)
    for (long long i = 0; i < n; i++) {
        long long tile = tiles ? tiles[i] : i;
        long long sk = 0, vi = 0;
        int st = run_tile(tile, q, k, v, B, Hq, Hkv, Lq, Lk, d, dv, k_row_stride, v_row_stride, scale, lambda,
                          causal, BM, BN, is_decode, num_splits, seed_splits, tph, nb, forced_skip, o, lse, skip,
                          visited,
                          gaps, &sk, &vi);
        skipped += sk;
        vis += vi;
        if (st != ORACLE_OK) {
#pragma omp critical
            status = st;
        }
    }
    counts[0] = skipped;
    counts[1] = vis;
    return status;
}
