/*
 * oracle.c -- plain, slow, fp64 CPU oracle for zigzag-sharded causal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library and
 * its Python binding) may include, link or call this file.  Only tests/,
 * __graft_entry__.smoke() and the cpu_baseline / reference legs of bench.py use it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * What it follows:
 *  - "Folding Tensor and Sequence Parallelism" summary page (gist.science,
 *    2604.26294), section 2 "Metodologia", attention-layer bullets: an
 *    all-gather rebuilds the full K/V along the sequence and FlashAttention runs
 *    on it; a zigzag partition balances causal work so later tokens are not
 *    overloaded.
 *  - "AutoSP" summary page (gist.science, 2604.27089), section 2.A step 4: index
 *    tensors such as causal masks are recomputed for the distributed layout, i.e.
 *    the mask compares GLOBAL positions.
 *  - "Tensor, pipeline e sequence parallelism" tutorial page (llmdeepdive, 5.8),
 *    "01 Conceito": query heads share a smaller set of K/V heads (GQA, 24 q heads
 *    on 4 kv heads at head dim 256).
 *  The pages define no formula for the zigzag beyond its purpose.  The reading
 *  used here: the sequence is cut into 2D equal chunks of C = S/(2D) positions and
 *  shard r holds chunk r followed by chunk 2D-1-r.
 *
 * The attention itself is the plain definition, written out with no blocking,
 * no online softmax and no reordering: per query row, all visible scores, the
 * max, the exponentials, their sum, lse = m + ln(l), P = exp(s - lse), O = P V.
 * The backward pass is the exact gradient of L = <dO, O>:
 *   Delta = <dO, O>;  dP_k = <dO, v_k>;  dS_k = P_k (dP_k - Delta);
 *   dQ = scale * sum_k dS_k k_k;  dK_k += scale * dS_k q;  dV_k += P_k dO.
 *
 * Layouts (all row-major, doubles):
 *   Q, O, dO, dQ : [D][B][2C][Hq][d]   (shard-major: shard r's rows are its slab)
 *   K, V, dK, dV : [B][S][Hkv][d]      (natural position order, all-gathered)
 *   lse, Delta   : [D][B][Hq][2C]
 * GQA: q head h reads kv head h / (Hq/Hkv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Zigzag partition                                                    */
/* ------------------------------------------------------------------ */

/* Global position of row j (0 <= j < 2C) of shard r. */
static int64_t zigzag_position(int64_t S, int32_t D, int32_t r, int64_t j)
{
    int64_t C = S / (2 * (int64_t)D);
    if (j < C)
        return (int64_t)r * C + j;                       /* first chunk: r        */
    return (int64_t)(2 * D - 1 - r) * C + (j - C);       /* second chunk: 2D-1-r  */
}

/* perm[r*2C + j] = global position of shard-major row (r, j);
 * inv_perm[p]     = shard-major row index holding position p.
 * Returns 0, or -1 when S is not a multiple of 2D. */
int oracle_partition(int64_t S, int32_t D, int32_t *perm, int32_t *inv_perm)
{
    if (D <= 0 || S <= 0 || S % (2 * (int64_t)D) != 0)
        return -1;
    int64_t twoC = S / D;
    for (int32_t r = 0; r < D; ++r)
        for (int64_t j = 0; j < twoC; ++j) {
            int64_t p = zigzag_position(S, D, r, j);
            if (perm)
                perm[r * twoC + j] = (int32_t)p;
            if (inv_perm)
                inv_perm[p] = (int32_t)(r * twoC + j);
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Tile schedule (the build's own definition; the pages give none)     */
/* ------------------------------------------------------------------ */
/*
 * Tiling: a shard's 2C rows are cut into T = 2C/bq query tiles of bq rows; keys
 * into S/bk key tiles of bk.  A query tile's key-tile count kend is the number of
 * key tiles up to and including the one holding its largest visible key:
 *   kend = (largest position among the tile's rows) / bk + 1    (causal)
 *   kend = S / bk                                               (non-causal)
 * Per-shard work (QK^T tile products of size bq x bk, over all b and q heads):
 *   shard_tiles[r] = B * Hq * sum_i kend(r, i)
 * Work units: for each (b, kv head g, shard r) the T*G query slots are listed
 * tile-major, slot s = i*G + e meaning q tile i of q head g*G + e; consecutive
 * runs of `slots` slots form one unit (the last run may be short).  A unit row is
 *   {r, b, g, tile0, head0, tile1, head1, kend0, kend1}
 * with -1 / 0 for absent slots (slots == 1 leaves the second slot absent).
 * Order: by b, then g (ascending); within one (b, g) by max(kend0, kend1)
 * descending, then r, then the unit's index m within its (b, g, r) list (ascending).
 */
typedef struct {
    int32_t f[9];
    int64_t key_work, key_r, key_m, key_b, key_g;
} unit_rec;

static int unit_cmp(const void *pa, const void *pb)
{
    const unit_rec *a = (const unit_rec *)pa, *b = (const unit_rec *)pb;
    if (a->key_b != b->key_b) return a->key_b < b->key_b ? -1 : 1;
    if (a->key_g != b->key_g) return a->key_g < b->key_g ? -1 : 1;
    if (a->key_work != b->key_work) return a->key_work > b->key_work ? -1 : 1;
    if (a->key_r != b->key_r) return a->key_r < b->key_r ? -1 : 1;
    if (a->key_m != b->key_m) return a->key_m < b->key_m ? -1 : 1;
    return 0;
}

static int64_t tile_kend(int64_t S, int32_t D, int32_t r, int64_t i, int32_t bq,
                         int32_t bk, int32_t causal)
{
    if (!causal)
        return S / bk;
    int64_t largest = -1;
    for (int64_t j = i * bq; j < (i + 1) * bq; ++j) {   /* brute scan of the tile */
        int64_t p = zigzag_position(S, D, r, j);
        if (p > largest) largest = p;
    }
    return largest / bk + 1;
}

/* Returns the number of units (always written to *n_units), or -1 for an
 * invalid tiling.  units may be NULL (count only); at most cap rows written. */
int64_t oracle_schedule(int64_t S, int32_t D, int32_t B, int32_t Hq, int32_t Hkv,
                        int32_t causal, int32_t bq, int32_t bk, int32_t slots,
                        int64_t *shard_tiles, int32_t *units, int64_t cap)
{
    if (D <= 0 || B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || bq <= 0 ||
        bk <= 0 || (slots != 1 && slots != 2))
        return -1;
    if (S % (2 * (int64_t)D) != 0 || (S / D) % bq != 0 || S % bk != 0)
        return -1;
    int32_t G = Hq / Hkv;
    int64_t T = (S / D) / bq;
    int64_t *kend = (int64_t *)malloc(sizeof(int64_t) * (size_t)(D * T));
    for (int32_t r = 0; r < D; ++r)
        for (int64_t i = 0; i < T; ++i)
            kend[r * T + i] = tile_kend(S, D, r, i, bq, bk, causal);
    if (shard_tiles)
        for (int32_t r = 0; r < D; ++r) {
            int64_t w = 0;
            for (int64_t i = 0; i < T; ++i) w += kend[r * T + i];
            shard_tiles[r] = w * B * Hq;
        }
    int64_t per_group = (T * G + slots - 1) / slots;
    int64_t n = (int64_t)B * Hkv * D * per_group;
    if (units) {
        unit_rec *recs = (unit_rec *)malloc(sizeof(unit_rec) * (size_t)n);
        int64_t u = 0;
        for (int32_t b = 0; b < B; ++b)
            for (int32_t g = 0; g < Hkv; ++g)
                for (int32_t r = 0; r < D; ++r)
                    for (int64_t m = 0; m < per_group; ++m) {
                        unit_rec *x = &recs[u++];
                        int64_t s0 = m * slots;
                        int64_t s1 = s0 + 1;
                        int has1 = (slots == 2) && (s1 < T * G);
                        int64_t i0 = s0 / G, e0 = s0 % G;
                        x->f[0] = r; x->f[1] = b; x->f[2] = g;
                        x->f[3] = (int32_t)i0; x->f[4] = (int32_t)(g * G + e0);
                        x->f[7] = (int32_t)kend[r * T + i0];
                        if (has1) {
                            int64_t i1 = s1 / G, e1 = s1 % G;
                            x->f[5] = (int32_t)i1; x->f[6] = (int32_t)(g * G + e1);
                            x->f[8] = (int32_t)kend[r * T + i1];
                        } else {
                            x->f[5] = -1; x->f[6] = -1; x->f[8] = 0;
                        }
                        x->key_work = x->f[7] > x->f[8] ? x->f[7] : x->f[8];
                        x->key_r = r; x->key_m = m; x->key_b = b; x->key_g = g;
                    }
        qsort(recs, (size_t)n, sizeof(unit_rec), unit_cmp);
        for (int64_t k = 0; k < n && k < cap; ++k)
            memcpy(units + 9 * k, recs[k].f, sizeof(int32_t) * 9);
        free(recs);
    }
    free(kend);
    return n;
}

/* ------------------------------------------------------------------ */
/* Attention, forward, one query row                                   */
/* ------------------------------------------------------------------ */

/* Scores, probabilities and output of one (shard-major row, q head).
 *   q_row : [d] query vector;  p : its global position
 *   k, v  : [B][S][Hkv][d]
 *   s_buf : scratch of S doubles, left holding P_k for k < n_keys
 * Writes o_row[d], returns lse, sets *n_keys_out. */
static double attend_row(int64_t S, int32_t Hkv, int32_t d, int32_t causal,
                         double scale, const double *q_row, int64_t p,
                         const double *k, const double *v, int32_t b, int32_t kv,
                         double *s_buf, double *o_row, int64_t *n_keys_out)
{
    int64_t n_keys = causal ? p + 1 : S;      /* key k visible iff k <= p (global) */
    *n_keys_out = n_keys;
    double m = -INFINITY;
    for (int64_t key = 0; key < n_keys; ++key) {
        const double *kk = k + (((int64_t)b * S + key) * Hkv + kv) * d;
        double dot = 0.0;
        for (int32_t t = 0; t < d; ++t) dot += q_row[t] * kk[t];
        s_buf[key] = scale * dot;
        if (s_buf[key] > m) m = s_buf[key];
    }
    double l = 0.0;
    for (int64_t key = 0; key < n_keys; ++key) l += exp(s_buf[key] - m);
    double lse = m + log(l);
    for (int64_t key = 0; key < n_keys; ++key) s_buf[key] = exp(s_buf[key] - lse);
    for (int32_t t = 0; t < d; ++t) o_row[t] = 0.0;
    for (int64_t key = 0; key < n_keys; ++key) {
        const double *vv = v + (((int64_t)b * S + key) * Hkv + kv) * d;
        for (int32_t t = 0; t < d; ++t) o_row[t] += s_buf[key] * vv[t];
    }
    return lse;
}

static int check_problem(int32_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t d,
                         int32_t D)
{
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || D <= 0) return -1;
    if (Hq % Hkv != 0 || S % (2 * (int64_t)D) != 0) return -1;
    return 0;
}

/* Full forward.  o: [D][B][2C][Hq][d], lse: [D][B][Hq][2C]. */
int oracle_attn_fwd(int32_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t d,
                    int32_t D, int32_t causal, double scale, const double *q,
                    const double *k, const double *v, double *o, double *lse)
{
    if (check_problem(B, S, Hq, Hkv, d, D)) return -1;
    int64_t twoC = S / D;
    int32_t G = Hq / Hkv;
    int64_t n_rows = (int64_t)D * B * twoC;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 16)
        for (int64_t idx = 0; idx < n_rows * Hq; ++idx) {
            int64_t row = idx / Hq;                 /* (r, b, j) flattened */
            int32_t h = (int32_t)(idx % Hq);
            int32_t r = (int32_t)(row / ((int64_t)B * twoC));
            int32_t b = (int32_t)((row / twoC) % B);
            int64_t j = row % twoC;
            int64_t p = zigzag_position(S, D, r, j);
            int64_t nk;
            double l = attend_row(S, Hkv, d, causal, scale, q + (row * Hq + h) * d, p, k,
                                  v, b, h / G, s_buf, o + (row * Hq + h) * d, &nk);
            lse[(((int64_t)r * B + b) * Hq + h) * twoC + j] = l;
        }
        free(s_buf);
    }
    return 0;
}

/* Forward on selected shard-major rows only.
 *   rows   : [n] flattened (r, b, j) row indices, (r*B + b)*2C + j
 *   q_rows : [n][Hq][d] the query vectors of those rows
 *   o_rows : [n][Hq][d], lse_rows : [n][Hq] */
int oracle_attn_fwd_rows(int32_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t d,
                         int32_t D, int32_t causal, double scale, const int64_t *rows,
                         int64_t n, const double *q_rows, const double *k,
                         const double *v, double *o_rows, double *lse_rows)
{
    if (check_problem(B, S, Hq, Hkv, d, D)) return -1;
    int64_t twoC = S / D;
    int32_t G = Hq / Hkv;
    for (int64_t x = 0; x < n; ++x)
        if (rows[x] < 0 || rows[x] >= (int64_t)D * B * twoC) return -1;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 4)
        for (int64_t idx = 0; idx < n * Hq; ++idx) {
            int64_t x = idx / Hq;
            int32_t h = (int32_t)(idx % Hq);
            int64_t row = rows[x];
            int32_t r = (int32_t)(row / ((int64_t)B * twoC));
            int32_t b = (int32_t)((row / twoC) % B);
            int64_t j = row % twoC;
            int64_t p = zigzag_position(S, D, r, j);
            int64_t nk;
            lse_rows[x * Hq + h] =
                attend_row(S, Hkv, d, causal, scale, q_rows + (x * Hq + h) * d, p, k, v,
                           b, h / G, s_buf, o_rows + (x * Hq + h) * d, &nk);
        }
        free(s_buf);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Backward                                                            */
/* ------------------------------------------------------------------ */

/* Full backward of L = <dout, O>.  Also returns the forward o, lse and
 * delta = rowsum(dout * o) it used (all fp64).  dk, dv are sums over every
 * shard and every q head of the kv group (what a reduce-scatter would deliver).
 * Parallel over (b, kv head): each group owns its dk/dv slice outright. */
int oracle_attn_bwd(int32_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t d,
                    int32_t D, int32_t causal, double scale, const double *q,
                    const double *k, const double *v, const double *dout, double *dq,
                    double *dk, double *dv, double *o, double *lse, double *delta)
{
    if (check_problem(B, S, Hq, Hkv, d, D)) return -1;
    int64_t twoC = S / D;
    int32_t G = Hq / Hkv;
    memset(dk, 0, sizeof(double) * (size_t)((int64_t)B * S * Hkv * d));
    memset(dv, 0, sizeof(double) * (size_t)((int64_t)B * S * Hkv * d));
#pragma omp parallel
    {
        double *p_buf = (double *)malloc(sizeof(double) * (size_t)S);
        double *ds_buf = (double *)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 1)
        for (int64_t grp = 0; grp < (int64_t)B * Hkv; ++grp) {
            int32_t b = (int32_t)(grp / Hkv);
            int32_t kv = (int32_t)(grp % Hkv);
            for (int32_t e = 0; e < G; ++e) {
                int32_t h = kv * G + e;
                for (int32_t r = 0; r < D; ++r)
                    for (int64_t j = 0; j < twoC; ++j) {
                        int64_t row = ((int64_t)r * B + b) * twoC + j;
                        int64_t p = zigzag_position(S, D, r, j);
                        const double *q_row = q + (row * Hq + h) * d;
                        const double *do_row = dout + (row * Hq + h) * d;
                        double *o_row = o + (row * Hq + h) * d;
                        double *dq_row = dq + (row * Hq + h) * d;
                        int64_t nk;
                        double l = attend_row(S, Hkv, d, causal, scale, q_row, p, k, v, b,
                                              kv, p_buf, o_row, &nk);
                        int64_t stat = (((int64_t)r * B + b) * Hq + h) * twoC + j;
                        lse[stat] = l;
                        double dlt = 0.0;
                        for (int32_t t = 0; t < d; ++t) dlt += do_row[t] * o_row[t];
                        delta[stat] = dlt;
                        for (int64_t key = 0; key < nk; ++key) {
                            const double *vv = v + (((int64_t)b * S + key) * Hkv + kv) * d;
                            double dp = 0.0;
                            for (int32_t t = 0; t < d; ++t) dp += do_row[t] * vv[t];
                            ds_buf[key] = p_buf[key] * (dp - dlt);
                        }
                        for (int32_t t = 0; t < d; ++t) dq_row[t] = 0.0;
                        for (int64_t key = 0; key < nk; ++key) {
                            int64_t kofs = (((int64_t)b * S + key) * Hkv + kv) * d;
                            for (int32_t t = 0; t < d; ++t) {
                                dq_row[t] += scale * ds_buf[key] * k[kofs + t];
                                dk[kofs + t] += scale * ds_buf[key] * q_row[t];
                                dv[kofs + t] += p_buf[key] * do_row[t];
                            }
                        }
                    }
            }
        }
        free(p_buf);
        free(ds_buf);
    }
    return 0;
}

/* dQ of selected shard-major rows only (each row's dQ needs nothing but its own q, dO
 * and all of K, V: its forward is recomputed, Delta = <dO, O>, dS_k = P_k(dP_k -
 * Delta), dQ = scale * sum_k dS_k k_k).
 *   rows : [n] flattened (r*B + b)*2C + j;  q_rows, do_rows : [n][Hq][d]
 *   dq_rows : [n][Hq][d] */
int oracle_attn_dq_rows(int32_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t d,
                        int32_t D, int32_t causal, double scale, const int64_t *rows,
                        int64_t n, const double *q_rows, const double *do_rows,
                        const double *k, const double *v, double *dq_rows)
{
    if (check_problem(B, S, Hq, Hkv, d, D)) return -1;
    int64_t twoC = S / D;
    int32_t G = Hq / Hkv;
    for (int64_t x = 0; x < n; ++x)
        if (rows[x] < 0 || rows[x] >= (int64_t)D * B * twoC) return -1;
#pragma omp parallel
    {
        double *p_buf = (double *)malloc(sizeof(double) * (size_t)S);
        double *o_row = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (int64_t idx = 0; idx < n * Hq; ++idx) {
            int64_t x = idx / Hq;
            int32_t h = (int32_t)(idx % Hq);
            int64_t row = rows[x];
            int32_t r = (int32_t)(row / ((int64_t)B * twoC));
            int32_t b = (int32_t)((row / twoC) % B);
            int64_t j = row % twoC;
            int64_t p = zigzag_position(S, D, r, j);
            int32_t kv = h / G;
            const double *q_row = q_rows + (x * Hq + h) * d;
            const double *do_row = do_rows + (x * Hq + h) * d;
            double *dq_row = dq_rows + (x * Hq + h) * d;
            int64_t nk;
            attend_row(S, Hkv, d, causal, scale, q_row, p, k, v, b, kv, p_buf, o_row, &nk);
            double dlt = 0.0;
            for (int32_t t = 0; t < d; ++t) dlt += do_row[t] * o_row[t];
            for (int32_t t = 0; t < d; ++t) dq_row[t] = 0.0;
            for (int64_t key = 0; key < nk; ++key) {
                int64_t kofs = (((int64_t)b * S + key) * Hkv + kv) * d;
                double dp = 0.0;
                for (int32_t t = 0; t < d; ++t) dp += do_row[t] * v[kofs + t];
                double ds = p_buf[key] * (dp - dlt);
                for (int32_t t = 0; t < d; ++t) dq_row[t] += scale * ds * k[kofs + t];
            }
        }
        free(p_buf);
        free(o_row);
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Partial results over a key range, and their merge                   */
/* ------------------------------------------------------------------ */
/*
 * Ring attention ("AutoSP" summary page, sections 1 and 4, where it is the
 * sequence-parallel baseline) hands each rank's queries the K/V blocks one after
 * another; each block gives the softmax attention restricted to its keys, and the
 * pieces are combined.  The pages print no formula.  The reading taken is the
 * definition of a softmax over a union of disjoint key sets K_1, ..., K_n: with
 * lse_i = ln sum_{k in K_i} exp(s_k) and O_i = sum_{k in K_i} exp(s_k - lse_i) v_k,
 *   lse = ln sum_i exp(lse_i),   O = sum_i exp(lse_i - lse) O_i,
 * an empty K_i contributing lse_i = -inf and O_i = 0.
 */

/* Forward restricted to the keys at positions [key_lo, key_hi), intersected with the
 * causal set k <= p.  A row that sees no key gets lse = -inf and O = 0.
 * Layouts as oracle_attn_fwd. */
int oracle_attn_fwd_keys(int32_t B, int64_t S, int32_t Hq, int32_t Hkv, int32_t d,
                         int32_t D, int32_t causal, double scale, int64_t key_lo,
                         int64_t key_hi, const double *q, const double *k,
                         const double *v, double *o, double *lse)
{
    if (check_problem(B, S, Hq, Hkv, d, D)) return -1;
    if (key_lo < 0 || key_hi > S || key_lo > key_hi) return -1;
    int64_t twoC = S / D;
    int32_t G = Hq / Hkv;
    int64_t n_rows = (int64_t)D * B * twoC;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
#pragma omp for schedule(dynamic, 16)
        for (int64_t idx = 0; idx < n_rows * Hq; ++idx) {
            int64_t row = idx / Hq;
            int32_t h = (int32_t)(idx % Hq);
            int32_t r = (int32_t)(row / ((int64_t)B * twoC));
            int32_t b = (int32_t)((row / twoC) % B);
            int64_t j = row % twoC;
            int64_t p = zigzag_position(S, D, r, j);
            int32_t kv = h / G;
            const double *q_row = q + (row * Hq + h) * d;
            double *o_row = o + (row * Hq + h) * d;
            int64_t end = key_hi;
            if (causal && p + 1 < end) end = p + 1;          /* visible: key <= p */
            for (int32_t t = 0; t < d; ++t) o_row[t] = 0.0;
            double *lse_out = &lse[(((int64_t)r * B + b) * Hq + h) * twoC + j];
            if (end <= key_lo) {                              /* no visible key */
                *lse_out = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int64_t key = key_lo; key < end; ++key) {
                const double *kk = k + (((int64_t)b * S + key) * Hkv + kv) * d;
                double dot = 0.0;
                for (int32_t t = 0; t < d; ++t) dot += q_row[t] * kk[t];
                s_buf[key] = scale * dot;
                if (s_buf[key] > m) m = s_buf[key];
            }
            double l = 0.0;
            for (int64_t key = key_lo; key < end; ++key) l += exp(s_buf[key] - m);
            double lse_r = m + log(l);
            for (int64_t key = key_lo; key < end; ++key) {
                double pk = exp(s_buf[key] - lse_r);
                const double *vv = v + (((int64_t)b * S + key) * Hkv + kv) * d;
                for (int32_t t = 0; t < d; ++t) o_row[t] += pk * vv[t];
            }
            *lse_out = lse_r;
        }
        free(s_buf);
    }
    return 0;
}

/* Merge of n partial results.  o_parts [n][m][d] and lse_parts [n][m] hold, for the
 * same m (row, head) pairs in the same order, each part's O and lse; writes o [m][d]
 * and lse [m].  Pairs whose parts are all empty get lse = -inf and O = 0. */
int oracle_attn_merge(int32_t n, int64_t m, int32_t d, const double *o_parts,
                      const double *lse_parts, double *o, double *lse)
{
    if (n <= 0 || m < 0 || d <= 0) return -1;
    for (int64_t x = 0; x < m; ++x) {
        double mx = -INFINITY;
        for (int32_t i = 0; i < n; ++i)
            if (lse_parts[(int64_t)i * m + x] > mx) mx = lse_parts[(int64_t)i * m + x];
        double *o_row = o + x * d;
        for (int32_t t = 0; t < d; ++t) o_row[t] = 0.0;
        if (mx == -INFINITY) {
            lse[x] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int32_t i = 0; i < n; ++i) l += exp(lse_parts[(int64_t)i * m + x] - mx);
        double lse_x = mx + log(l);
        for (int32_t i = 0; i < n; ++i) {
            double w = exp(lse_parts[(int64_t)i * m + x] - lse_x);
            const double *oi = o_parts + ((int64_t)i * m + x) * d;
            for (int32_t t = 0; t < d; ++t) o_row[t] += w * oi[t];
        }
        lse[x] = lse_x;
    }
    return 0;
}
