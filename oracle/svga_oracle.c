/*
 * svga_oracle.c -- plain fp64 CPU oracle for block-sparse spatio-temporal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU
 * baseline may load this file's library.  It shares no code, header, table or
 * helper with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes, and where the method is stated ("Accelerating Spatio-Temporal
 * Attention for Video Diffusion on TPUs", summarised on three pages):
 *   - spatial heads keep keys of the same or nearby frames; temporal heads keep keys
 *     at nearby in-frame positions over all frames (aihirek.info, section "A Sparse
 *     VideoGen a figyelmi fejeket osztalyozza");
 *   - both masks keep every key of the first frame, the attention anchor (same
 *     section);
 *   - sparsity skips (query tile, key tile) pairs; visited tiles are either fully kept
 *     ("full") or partly kept ("boundary", masked element by element) (aihirek.info,
 *     section "A TPU-kernel kialakitasa dontonek bizonyult"; ainews.tenesys.com,
 *     "Co sie zmienilo?" items 1-2);
 *   - the token order of temporal heads is changed from frame-major to
 *     temporal-major (ainews.tenesys.com, "Co sie zmienilo?" item 5).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - predicates: spatial keeps |f_q - f_k| <= w_f, temporal keeps |s_q - s_k| <= w_s on
 *     the flattened in-frame index s = row * W + col; bands inclusive;
 *   - anchor is key-side: every query keeps all keys with f_k == 0;
 *   - temporal-major order "anchor-first": frame-0 tokens first (position s), then the
 *     other frames s-major: position S + s*(F-1) + (f-1).  The literal order s*F + f is
 *     kept as the "strict" variant;
 *   - a tile that holds padding (positions >= N) is never full: padded pairs are not kept;
 *   - an empty row gives O = 0 and LSE = -inf;
 *   - the tile-aligned traversal (B3: ainews.tenesys.com, "Co sie zmienilo?" item 4;
 *     oossa.com, opening paragraph) has two readings, both here: the mask snapped to
 *     tiles (orc_attention_rows_tile_aligned), and an exact layout in which each frame
 *     of a frame-major head starts at a multiple of a frame stride Sp >= S (positions
 *     f * Sp + s, positions f * Sp + s with s >= S hold no token); temporal-major heads
 *     keep their order and the positions from N on hold no token
 *     (orc_order_coords_padded, orc_tile_counts_padded).  The padded layout changes
 *     which pairs share a tile, not which pairs are kept, so its attention is the
 *     plain one.
 *
 * The attention is the plain definition: for each query row, the masked softmax of
 * scale * q . k over the kept keys, applied to V, computed in double precision from the
 * bf16-rounded inputs (passed in as float32 arrays holding bf16 values).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_FRAME_MAJOR = 0, ORC_TEMPORAL_ANCHOR_FIRST = 1, ORC_TEMPORAL_STRICT = 2 };
enum { ORC_SPATIAL = 0, ORC_TEMPORAL = 1, ORC_DENSE = 2 };

/* Position of token (frame f, in-frame index s) in the given order. */
long long orc_position(int order, int F, int S, int f, int s)
{
    if (order == ORC_FRAME_MAJOR) return (long long)f * S + s;
    if (order == ORC_TEMPORAL_STRICT) return (long long)s * F + f;
    /* anchor-first temporal-major */
    if (f == 0) return s;
    return (long long)S + (long long)s * (F - 1) + (f - 1);
}

/* Coordinates of every position of an order, found by scattering the forward map
 * over all tokens (no closed-form inverse).  Returns 0 if the map is a bijection. */
int orc_order_coords(int order, int F, int S, int32_t *f_of_pos, int32_t *s_of_pos)
{
    long long N = (long long)F * S;
    for (long long i = 0; i < N; ++i) { f_of_pos[i] = -1; s_of_pos[i] = -1; }
    for (int f = 0; f < F; ++f)
        for (int s = 0; s < S; ++s) {
            long long p = orc_position(order, F, S, f, s);
            if (p < 0 || p >= N || f_of_pos[p] != -1) return -1;
            f_of_pos[p] = f;
            s_of_pos[p] = s;
        }
    return 0;
}

/* The keep predicate M(q, k) on original coordinates. */
int orc_keep(int type, int band, int anchor, int fq, int sq, int fk, int sk)
{
    if (type == ORC_DENSE) return 1;
    if (anchor && fk == 0) return 1;
    if (type == ORC_SPATIAL) return abs(fq - fk) <= band;
    return abs(sq - sk) <= band;
}

/* Number of kept (q, k) pairs of one head, by enumerating all pairs. */
long long orc_kept_count(int type, int band, int anchor, int F, int S)
{
    long long N = (long long)F * S, total = 0;
#pragma omp parallel for reduction(+ : total) schedule(dynamic, 16)
    for (long long q = 0; q < N; ++q) {
        int fq = (int)(q / S), sq = (int)(q % S);
        long long c = 0;
        for (long long k = 0; k < N; ++k)
            c += orc_keep(type, band, anchor, fq, sq, (int)(k / S), (int)(k % S));
        total += c;
    }
    return total;
}

/* The element mask of one head in frame-major order, N x N bytes. */
void orc_mask(int type, int band, int anchor, int F, int S, uint8_t *mask)
{
    long long N = (long long)F * S;
#pragma omp parallel for schedule(static)
    for (long long q = 0; q < N; ++q)
        for (long long k = 0; k < N; ++k)
            mask[q * N + k] = (uint8_t)orc_keep(type, band, anchor, (int)(q / S), (int)(q % S),
                                                (int)(k / S), (int)(k % S));
}

int orc_tile_counts_range(int type, int band, int anchor, int order, int F, int S,
                          int tq, int tk, long long i0, long long i1, int64_t *counts);

/* The padded layout: position of token (f, s) when frame-major frames are laid out
 * with stride Sp (Sp >= S); the temporal-major orders are not padded. */
long long orc_position_padded(int order, int F, int S, int Sp, int f, int s)
{
    if (order == ORC_FRAME_MAJOR) return (long long)f * Sp + s;
    return orc_position(order, F, S, f, s);
}

/* Coordinates at every position 0 .. F * Sp - 1 of the padded layout, -1 / -1 where a
 * position holds no token; found by scattering the forward map over all tokens.
 * Returns 0 if every token lands on its own position inside the range. */
int orc_order_coords_padded(int order, int F, int S, int Sp, int32_t *f_of_pos,
                            int32_t *s_of_pos)
{
    long long NP = (long long)F * Sp;
    if (Sp < S) return -2;
    for (long long i = 0; i < NP; ++i) { f_of_pos[i] = -1; s_of_pos[i] = -1; }
    for (int f = 0; f < F; ++f)
        for (int s = 0; s < S; ++s) {
            long long p = orc_position_padded(order, F, S, Sp, f, s);
            if (p < 0 || p >= NP || f_of_pos[p] != -1) return -1;
            f_of_pos[p] = f;
            s_of_pos[p] = s;
        }
    return 0;
}

/* Kept-element counts of every (q-tile, k-tile) pair of one head in the padded layout
 * (F * Sp positions, tiles tq x tk over positions, the grid padded to whole tiles);
 * a position without a token keeps nothing.  counts has n_q * n_k entries. */
int orc_tile_counts_padded(int type, int band, int anchor, int order, int F, int S, int Sp,
                           int tq, int tk, int64_t *counts)
{
    long long NP = (long long)F * Sp;
    long long nq = (NP + tq - 1) / tq, nk = (NP + tk - 1) / tk;
    int32_t *fp = (int32_t *)malloc(sizeof(int32_t) * NP);
    int32_t *sp = (int32_t *)malloc(sizeof(int32_t) * NP);
    if (!fp || !sp) { free(fp); free(sp); return -2; }
    if (orc_order_coords_padded(order, F, S, Sp, fp, sp) != 0) { free(fp); free(sp); return -1; }
    memset(counts, 0, sizeof(int64_t) * nq * nk);
#pragma omp parallel for schedule(dynamic, 1)
    for (long long i = 0; i < nq; ++i) {
        int64_t *row = counts + i * nk;
        for (long long q = i * tq; q < (i + 1) * tq && q < NP; ++q) {
            if (fp[q] < 0) continue;
            for (long long k = 0; k < NP; ++k)
                if (fp[k] >= 0) row[k / tk] += orc_keep(type, band, anchor, fp[q], sp[q], fp[k], sp[k]);
        }
    }
    free(fp);
    free(sp);
    return 0;
}

/* Kept-element count of every (q-tile, k-tile) pair of one head whose tokens are
 * laid out in `order`, on the grid padded to whole tiles (padded pairs not kept).
 * counts has n_q * n_k entries, row-major over (q-tile, k-tile). */
int orc_tile_counts(int type, int band, int anchor, int order, int F, int S,
                    int tq, int tk, int64_t *counts)
{
    long long N = (long long)F * S;
    return orc_tile_counts_range(type, band, anchor, order, F, S, tq, tk, 0,
                                 (N + tq - 1) / tq, counts);
}

/* The same counts for the q-tiles i0 <= i < i1 only (counts has (i1 - i0) * n_k
 * entries): what a check of a few query rows of a large problem needs. */
int orc_tile_counts_range(int type, int band, int anchor, int order, int F, int S,
                          int tq, int tk, long long i0, long long i1, int64_t *counts)
{
    long long N = (long long)F * S;
    long long nq = (N + tq - 1) / tq, nk = (N + tk - 1) / tk;
    if (i0 < 0 || i1 > nq || i0 > i1) return -3;
    int32_t *fp = (int32_t *)malloc(sizeof(int32_t) * N);
    int32_t *sp = (int32_t *)malloc(sizeof(int32_t) * N);
    if (!fp || !sp) { free(fp); free(sp); return -2; }
    if (orc_order_coords(order, F, S, fp, sp) != 0) { free(fp); free(sp); return -1; }
    memset(counts, 0, sizeof(int64_t) * (i1 - i0) * nk);
#pragma omp parallel for schedule(dynamic, 1)
    for (long long i = i0; i < i1; ++i) {
        int64_t *row = counts + (i - i0) * nk;
        for (long long q = i * tq; q < (i + 1) * tq && q < N; ++q) {
            int fq = fp[q], sq = sp[q];
            for (long long k = 0; k < N; ++k)
                row[k / tk] += orc_keep(type, band, anchor, fq, sq, fp[k], sp[k]);
        }
    }
    free(fp);
    free(sp);
    return 0;
}

/* Tile classes from element counts: 0 = no kept element, 1 = every one of the
 * tq * tk pairs kept, 2 = otherwise.  Then, per q-tile, the ascending lists of full
 * and of boundary k-tiles (CSR: ptr has n_q + 1 entries).  Arrays are caller-owned;
 * full_idx / bnd_idx must hold n_q * n_k entries. */
void orc_classes_and_lists(const int64_t *counts, long long nq, long long nk, int tq, int tk,
                           uint8_t *cls, int32_t *full_ptr, int32_t *full_idx,
                           int32_t *bnd_ptr, int32_t *bnd_idx)
{
    long long nf = 0, nb = 0;
    for (long long i = 0; i < nq; ++i) {
        full_ptr[i] = (int32_t)nf;
        bnd_ptr[i] = (int32_t)nb;
        for (long long j = 0; j < nk; ++j) {
            int64_t c = counts[i * nk + j];
            uint8_t k = (c == 0) ? 0 : (c == (int64_t)tq * tk ? 1 : 2);
            cls[i * nk + j] = k;
            if (k == 1) full_idx[nf++] = (int32_t)j;
            if (k == 2) bnd_idx[nb++] = (int32_t)j;
        }
    }
    full_ptr[nq] = (int32_t)nf;
    bnd_ptr[nq] = (int32_t)nb;
}

/* Masked attention of one head for selected query rows, in frame-major order.
 *   q, k, v : [N, d] float32 holding bf16 values (frame-major)
 *   rows    : frame-major token indices of the query rows to compute
 *   o       : [nrows, d] double;  lse : [nrows] double (natural log)
 * For row q:  x_k = scale * q . k over kept k;  m = max x_k;
 *             O = sum exp(x_k - m) v_k / sum exp(x_k - m);  LSE = m + ln sum exp(x_k - m). */
void orc_attention_rows(const float *q, const float *k, const float *v, int F, int S, int d,
                        double scale, int type, int band, int anchor,
                        const int32_t *rows, int nrows, double *o, double *lse)
{
    long long N = (long long)F * S;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * N);
        double *qd = (double *)malloc(sizeof(double) * d);
        double *acc = (double *)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            long long t = rows[r];
            int fq = (int)(t / S), sq = (int)(t % S);
            for (int c = 0; c < d; ++c) qd[c] = (double)q[t * d + c];
            double m = -INFINITY;
            for (long long kk = 0; kk < N; ++kk) {
                if (!orc_keep(type, band, anchor, fq, sq, (int)(kk / S), (int)(kk % S))) {
                    x[kk] = -INFINITY;
                    continue;
                }
                const float *kr = k + kk * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qd[c] * (double)kr[c];
                x[kk] = scale * dot;
                if (x[kk] > m) m = x[kk];
            }
            for (int c = 0; c < d; ++c) acc[c] = 0.0;
            double l = 0.0;
            if (m != -INFINITY) {
                for (long long kk = 0; kk < N; ++kk) {
                    if (x[kk] == -INFINITY) continue;
                    double p = exp(x[kk] - m);
                    l += p;
                    const float *vr = v + kk * d;
                    for (int c = 0; c < d; ++c) acc[c] += p * (double)vr[c];
                }
            }
            for (int c = 0; c < d; ++c) o[(long long)r * d + c] = (l > 0.0) ? acc[c] / l : 0.0;
            lse[r] = (l > 0.0) ? m + log(l) : -INFINITY;
        }
        free(x);
        free(qd);
        free(acc);
    }
}

/* Tile-aligned traversal (B3: ainews.tenesys.com, "Co sie zmienilo?" item 4; oossa.com,
 * opening paragraph: the mask is aligned with the tiles the kernel computes), read as
 * the mask snapped to tiles: query token t keeps key token u iff the tile
 * (pos(t) / tq, pos(u) / tk) holds at least one pair the exact mask keeps, pos being
 * the position in the head's token order.  Then the plain masked softmax over that set.
 *   counts : kept-element counts of q-tiles i0 .. i0 + n_cnt - 1 (orc_tile_counts_range),
 *            n_k entries per q-tile; every row's q-tile must lie in that range
 *   rows, o, lse: as in orc_attention_rows (frame-major token indices).
 * Returns 0, or -1 when a row's q-tile is outside the counts given. */
int orc_attention_rows_tile_aligned(const float *q, const float *k, const float *v, int F,
                                    int S, int d, double scale, int order, int tq, int tk,
                                    const int64_t *counts, long long i0, long long n_cnt,
                                    const int32_t *rows, int nrows, double *o, double *lse)
{
    long long N = (long long)F * S, nk = (N + tk - 1) / tk;
    for (int r = 0; r < nrows; ++r) {
        long long t = rows[r];
        long long i = orc_position(order, F, S, (int)(t / S), (int)(t % S)) / tq;
        if (i < i0 || i >= i0 + n_cnt) return -1;
    }
    /* k-tile of every frame-major key token */
    int64_t *ktile = (int64_t *)malloc(sizeof(int64_t) * N);
    if (!ktile) return -2;
    for (long long u = 0; u < N; ++u)
        ktile[u] = orc_position(order, F, S, (int)(u / S), (int)(u % S)) / tk;
#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * N);
        double *qd = (double *)malloc(sizeof(double) * d);
        double *acc = (double *)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            long long t = rows[r];
            long long i = orc_position(order, F, S, (int)(t / S), (int)(t % S)) / tq;
            const int64_t *crow = counts + (i - i0) * nk;
            for (int c = 0; c < d; ++c) qd[c] = (double)q[t * d + c];
            double m = -INFINITY;
            for (long long u = 0; u < N; ++u) {
                if (crow[ktile[u]] == 0) {
                    x[u] = -INFINITY;
                    continue;
                }
                const float *kr = k + u * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qd[c] * (double)kr[c];
                x[u] = scale * dot;
                if (x[u] > m) m = x[u];
            }
            for (int c = 0; c < d; ++c) acc[c] = 0.0;
            double l = 0.0;
            if (m != -INFINITY) {
                for (long long u = 0; u < N; ++u) {
                    if (x[u] == -INFINITY) continue;
                    double p = exp(x[u] - m);
                    l += p;
                    const float *vr = v + u * d;
                    for (int c = 0; c < d; ++c) acc[c] += p * (double)vr[c];
                }
            }
            for (int c = 0; c < d; ++c) o[(long long)r * d + c] = (l > 0.0) ? acc[c] / l : 0.0;
            lse[r] = (l > 0.0) ? m + log(l) : -INFINITY;
        }
        free(x);
        free(qd);
        free(acc);
    }
    free(ktile);
    return 0;
}

int orc_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
