/*
 * rtp_oracle.c -- plain, slow, fp64 CPU oracle for the RTPurbo attention hot
 * path (one attention layer with retrieval heads and local heads).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA path.
 *
 * Source of every rule below: the paper-graph-ui summary page of
 * "Full Attention Strikes Back: Transferring Full Attention into Sparse within
 * Hundred Training Steps" (arXiv 2605.16928), cited as [FASB §<section>].
 *
 * Arithmetic: every sum, product, exp and log is fp64.  Tensors arrive as
 * bf16 bit patterns (uint16_t); a bf16 value converts to fp64 exactly.  The
 * only rounding this file performs on purpose is the single bf16
 * round-to-nearest-even of the 16-dim projections (the quantisation point of
 * the indexer, see orc_project_rows).
 *
 * Parity pins for each function live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_D 128 /* head dimension d_h */
#define ORC_R 16  /* indexer dimension r */

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp64                                                             */
/* ------------------------------------------------------------------------ */

/* A bf16 pattern is the upper half of an IEEE binary32; widening is exact. */
double orc_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round an fp64 value to bf16 (8 significant bits, binary32 exponent range),
 * round-to-nearest, ties-to-even, in one step (no intermediate binary32). */
uint16_t orc_double_to_bf16(double x)
{
    if (isnan(x))
        return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (a == 0.0)
        return sign;
    if (isinf(a) || a >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    int e;
    (void)frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1) */
    int q = e - 8;               /* exponent of one unit in the 8th significant bit */
    if (q < -133)                /* below the binary32 normal range: fixed quantum 2^-133 */
        q = -133;
    double r = rint(ldexp(a, -q)); /* default rounding mode: nearest, ties to even */
    double v = ldexp(r, q);
    float f = (float)v;          /* exact (<= 8 significant bits) or +inf on overflow */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

void orc_bf16_round_array(const double* x, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_double_to_bf16(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Indexer projection  [FASB §Low-Dimensional Projection Mechanism]          */
/*   q16 = W^Q_h q,  k16 = W^K_h k,  W stored as [d_h=128][r=16]            */
/* ------------------------------------------------------------------------ */

/* out[i][c] = bf16_rne( sum_d x[i][d] * W[d][c] ), the sum exact-ish in fp64
 * (each product of two bf16 values is exact in fp64).  pre[i][c] (nullable)
 * receives the fp64 value before rounding. */
void orc_project_rows(const uint16_t* x, int64_t n_rows, int64_t x_stride,
                      const uint16_t* W, uint16_t* out, int64_t out_stride,
                      double* pre)
{
    double Wd[ORC_D * ORC_R];
    for (int i = 0; i < ORC_D * ORC_R; ++i)
        Wd[i] = orc_bf16_to_double(W[i]);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n_rows; ++i) {
        const uint16_t* xr = x + i * x_stride;
        for (int c = 0; c < ORC_R; ++c) {
            double acc = 0.0;
            for (int d = 0; d < ORC_D; ++d)
                acc += orc_bf16_to_double(xr[d]) * Wd[d * ORC_R + c];
            out[i * out_stride + c] = orc_double_to_bf16(acc);
            if (pre)
                pre[i * ORC_R + c] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Indexer score  s(m, n) = q16_m . k16_n   [FASB §Low-Dimensional ...]     */
/* ------------------------------------------------------------------------ */

void orc_scores(const uint16_t* q16, const uint16_t* k16, int64_t n_keys,
                int64_t k16_stride, double* s)
{
    double q[ORC_R];
    for (int c = 0; c < ORC_R; ++c)
        q[c] = orc_bf16_to_double(q16[c]);
    for (int64_t j = 0; j < n_keys; ++j) {
        const uint16_t* kr = k16 + j * k16_stride;
        double acc = 0.0;
        for (int c = 0; c < ORC_R; ++c)
            acc += q[c] * orc_bf16_to_double(kr[c]);
        s[j] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* Dynamic top-p  [FASB §Dynamic Top-p Selection Mechanism, Eq. 5]          */
/* ------------------------------------------------------------------------ */

typedef struct {
    double s;
    int64_t j;
} orc_key;

/* Order: score descending; equal scores by index ascending (lower index wins). */
static int orc_key_cmp(const void* a, const void* b)
{
    const orc_key* x = (const orc_key*)a;
    const orc_key* y = (const orc_key*)b;
    if (x->s > y->s)
        return -1;
    if (x->s < y->s)
        return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

/*
 * Top-P over the scores s[0..n-1] (n >= 1):
 *   w_j = exp(s_j - max s), Z = sum_j w_j (softmax with no temperature);
 *   walk the keys in (score desc, index asc) order accumulating w and keep the
 *   shortest prefix whose mass reaches or exceeds p * Z.  p >= 1 keeps every key;
 *   p <= 0 keeps exactly the first key of the order (the argmax, lowest index).
 * Outputs (each nullable):
 *   sel[j]    1 if key j is kept;
 *   t         score of the last kept key (the row threshold);
 *   jtie      index of the last kept key: every kept key has s > t, or s == t
 *             and index <= jtie;
 *   count     number of kept keys;
 *   mass_frac kept mass / Z;
 *   Z, m      the softmax normaliser and the max score.
 */
void orc_topp(const double* s, int64_t n, double p, uint8_t* sel, double* t,
              int64_t* jtie, int64_t* count, double* mass_frac, double* Zout,
              double* mout)
{
    double m = s[0];
    for (int64_t j = 1; j < n; ++j)
        if (s[j] > m)
            m = s[j];
    double Z = 0.0;
    for (int64_t j = 0; j < n; ++j)
        Z += exp(s[j] - m);

    orc_key* order = (orc_key*)malloc((size_t)n * sizeof(orc_key));
    for (int64_t j = 0; j < n; ++j) {
        order[j].s = s[j];
        order[j].j = j;
    }
    qsort(order, (size_t)n, sizeof(orc_key), orc_key_cmp);

    int64_t kept = 0;
    double acc = 0.0;
    if (p >= 1.0) {
        kept = n;
        for (int64_t k = 0; k < n; ++k)
            acc += exp(order[k].s - m);
    } else {
        double target = p * Z;
        while (kept < n) {
            acc += exp(order[kept].s - m);
            ++kept;
            if (acc >= target)
                break;
        }
    }
    if (sel) {
        memset(sel, 0, (size_t)n);
        for (int64_t k = 0; k < kept; ++k)
            sel[order[k].j] = 1;
    }
    if (t)
        *t = order[kept - 1].s;
    if (jtie)
        *jtie = order[kept - 1].j;
    if (count)
        *count = kept;
    if (mass_frac)
        *mass_frac = acc / Z;
    if (Zout)
        *Zout = Z;
    if (mout)
        *mout = m;
    free(order);
}

/* ------------------------------------------------------------------------ */
/* Static top-k  [FASB §5 Experimental Analysis: the top-k variant of the   */
/* method, k = 4096, the fixed-budget baseline of the top-p ablation]       */
/* ------------------------------------------------------------------------ */

/*
 * Keep the k highest-scoring keys of s[0..n-1] (n >= 1, k >= 1); equal scores
 * go to the lower index, the same (score desc, index asc) order as orc_topp.
 * k >= n keeps every key.  Outputs as orc_topp (each nullable): sel, the
 * threshold t (score of the last kept key), jtie (its index), count = min(k, n).
 */
void orc_topk(const double* s, int64_t n, int64_t k, uint8_t* sel, double* t,
              int64_t* jtie, int64_t* count)
{
    orc_key* order = (orc_key*)malloc((size_t)n * sizeof(orc_key));
    for (int64_t j = 0; j < n; ++j) {
        order[j].s = s[j];
        order[j].j = j;
    }
    qsort(order, (size_t)n, sizeof(orc_key), orc_key_cmp);
    const int64_t kept = k < n ? k : n;
    if (sel) {
        memset(sel, 0, (size_t)n);
        for (int64_t a = 0; a < kept; ++a)
            sel[order[a].j] = 1;
    }
    if (t)
        *t = order[kept - 1].s;
    if (jtie)
        *jtie = order[kept - 1].j;
    if (count)
        *count = kept;
    free(order);
}

/* ------------------------------------------------------------------------ */
/* Block-level approximate top-p, sort-free by a histogram                  */
/* [FASB §Hardware-Aware Fast Top-p Decoding Kernel, steps 1-5]             */
/* ------------------------------------------------------------------------ */

/*
 * The keys s[0..n-1] (n >= 1) in blocks of `block` consecutive keys (the last
 * one may be shorter), nb = ceil(n / block):
 *   1-2. per block b: m_b = max of its scores and l_b = log sum exp of its
 *        scores (the block's attention mass, in log form);
 *   3.   a histogram of nbins bins over the block maxima: the range
 *        [lo, hi] = [min m_b, max m_b] cut into nbins equal bins,
 *        bin(b) = min(nbins - 1, floor(((m_b - lo) / (hi - lo)) * nbins))
 *        (every block in the top bin when hi == lo); each bin accumulates the
 *        masses exp(l_b - hi) of its blocks (the log-sum-exp of their l_b);
 *   4.   walk the bins from the highest down, accumulating their masses; the
 *        first bin at which the running mass reaches p * (total mass) is the
 *        threshold bin (p >= 1: the lowest occupied bin);
 *   5.   block b is selected iff bin(b) >= the threshold bin: the threshold
 *        bin is kept whole, since the histogram cannot tell its blocks apart.
 * Outputs (each nullable): bsel[nb] (1 = selected), bin_of[nb], the threshold
 * bin kstar, the kept token count, and the kept share of the token-level
 * softmax mass sum_{kept j} exp(s_j - max) / sum_j exp(s_j - max).
 * The range arithmetic is written as above in fp64 so that a caller may feed
 * it binary32 scores and reproduce any implementation that evaluates the same
 * expression in fp64.
 */
void orc_block_topp(const double* s, int64_t n, double p, int64_t block, int64_t nbins,
                    uint8_t* bsel, int64_t* bin_of, int64_t* kstar_out,
                    int64_t* kept_count, double* kept_mass_frac)
{
    const int64_t nb = (n + block - 1) / block;
    double* mb = (double*)malloc((size_t)nb * sizeof(double));
    double* lb = (double*)malloc((size_t)nb * sizeof(double));
    int64_t* bin = (int64_t*)malloc((size_t)nb * sizeof(int64_t));
    double* hist = (double*)calloc((size_t)nbins, sizeof(double));
    for (int64_t b = 0; b < nb; ++b) {
        const int64_t j0 = b * block, j1 = (j0 + block < n) ? j0 + block : n;
        double m = s[j0];
        for (int64_t j = j0 + 1; j < j1; ++j)
            if (s[j] > m)
                m = s[j];
        double acc = 0.0;
        for (int64_t j = j0; j < j1; ++j)
            acc += exp(s[j] - m);
        mb[b] = m;
        lb[b] = m + log(acc);
    }
    double lo = mb[0], hi = mb[0];
    for (int64_t b = 1; b < nb; ++b) {
        if (mb[b] < lo)
            lo = mb[b];
        if (mb[b] > hi)
            hi = mb[b];
    }
    double total = 0.0;
    for (int64_t b = 0; b < nb; ++b) {
        int64_t k = nbins - 1;
        if (hi > lo) {
            const double x = floor(((mb[b] - lo) / (hi - lo)) * (double)nbins);
            k = x < (double)(nbins - 1) ? (int64_t)x : nbins - 1;
        }
        bin[b] = k;
        const double w = exp(lb[b] - hi);
        hist[k] += w;
        total += w;
    }
    int64_t kstar = 0;
    if (p >= 1.0) {
        for (kstar = 0; kstar < nbins && hist[kstar] == 0.0; ++kstar) {
        }
    } else {
        double cum = 0.0;
        for (int64_t k = nbins - 1; k >= 0; --k) {
            if (hist[k] == 0.0)
                continue;
            cum += hist[k];
            kstar = k;
            if (cum >= p * total)
                break;
        }
    }
    double m = hi, Z = 0.0, kept_m = 0.0;
    int64_t cnt = 0;
    for (int64_t b = 0; b < nb; ++b) {
        const int64_t j0 = b * block, j1 = (j0 + block < n) ? j0 + block : n;
        const int on = bin[b] >= kstar;
        for (int64_t j = j0; j < j1; ++j) {
            const double w = exp(s[j] - m);
            Z += w;
            if (on) {
                kept_m += w;
                ++cnt;
            }
        }
        if (bsel)
            bsel[b] = (uint8_t)on;
        if (bin_of)
            bin_of[b] = bin[b];
    }
    if (kstar_out)
        *kstar_out = kstar;
    if (kept_count)
        *kept_count = cnt;
    if (kept_mass_frac)
        *kept_mass_frac = kept_m / Z;
    free(mb);
    free(lb);
    free(bin);
    free(hist);
}

/* ------------------------------------------------------------------------ */
/* Exact attention over an index set  [FASB §Dynamic Top-p ..., sparse      */
/* attention formula]: O = sum_{n in S} softmax_S(q.k_n * scale) v_n        */
/* ------------------------------------------------------------------------ */

/* idx: ascending key indices (n_idx >= 1).  o: 128 fp64.  lse: log sum exp of
 * the scaled logits over the set. */
void orc_attend(const uint16_t* q, const uint16_t* K, int64_t k_stride,
                const uint16_t* V, int64_t v_stride, const int64_t* idx,
                int64_t n_idx, double scale, double* o, double* lse)
{
    double qd[ORC_D];
    for (int d = 0; d < ORC_D; ++d)
        qd[d] = orc_bf16_to_double(q[d]);
    double* logit = (double*)malloc((size_t)n_idx * sizeof(double));
    double mx = -INFINITY;
    for (int64_t a = 0; a < n_idx; ++a) {
        const uint16_t* kr = K + idx[a] * k_stride;
        double acc = 0.0;
        for (int d = 0; d < ORC_D; ++d)
            acc += qd[d] * orc_bf16_to_double(kr[d]);
        logit[a] = acc * scale;
        if (logit[a] > mx)
            mx = logit[a];
    }
    double den = 0.0;
    for (int d = 0; d < ORC_D; ++d)
        o[d] = 0.0;
    for (int64_t a = 0; a < n_idx; ++a) {
        double w = exp(logit[a] - mx);
        den += w;
        const uint16_t* vr = V + idx[a] * v_stride;
        for (int d = 0; d < ORC_D; ++d)
            o[d] += w * orc_bf16_to_double(vr[d]);
    }
    for (int d = 0; d < ORC_D; ++d)
        o[d] /= den;
    if (lse)
        *lse = mx + log(den);
    free(logit);
}

/* ------------------------------------------------------------------------ */
/* Local-head key set  [FASB §Local Head Attention Pattern]                  */
/*   keys j <= P with j < n_sink (attention sinks) or j > P - W (the W most  */
/*   recent positions, the query's own included).                            */
/* ------------------------------------------------------------------------ */

int64_t orc_local_set(int64_t P, int64_t window, int64_t n_sink, int64_t* idx)
{
    int64_t n = 0;
    for (int64_t j = 0; j <= P; ++j)
        if (j < n_sink || j > P - window)
            idx[n++] = j;
    return n;
}

/* ------------------------------------------------------------------------ */
/* Row drivers (OpenMP over independent rows).                              */
/* Layouts (bf16 bits, all contiguous):                                      */
/*   q   [B][Lq][H][128]      k, v [B][Lk][Hkv][128]                         */
/*   q16 [B][Lq][Hq16][16]    k16  [B][Lk][Hk16][16]                         */
/* A row is (b, i, h): batch b, query row i (position P = q_pos0 + i), query  */
/* head h.  Its keys are positions 0..P of batch b, kv head g = h / (H/Hkv). */
/* ------------------------------------------------------------------------ */

typedef struct {
    int64_t B, Lq, Lk, H, Hkv;
    int64_t q_pos0;
} orc_shape;

static inline int64_t orc_q_off(const orc_shape* S, int64_t b, int64_t i, int64_t h)
{
    return ((b * S->Lq + i) * S->H + h) * ORC_D;
}

static inline int64_t orc_kv_off(const orc_shape* S, int64_t b, int64_t j, int64_t g)
{
    return ((b * S->Lk + j) * S->Hkv + g) * ORC_D;
}

/*
 * Retrieval rows: indexer scores from (q16, k16) -> Top-P -> exact attention.
 * row_b/row_i/row_h: the rows; row_hq16/row_hk16: the head slot of that row's
 * indexer query in q16 and of its indexer keys in k16.  Hq16/Hk16: number of
 * head slots in q16/k16.  Outputs per row r: o[r*128..], lse[r], t[r],
 * jtie[r], count[r], mass_frac[r]; sel (nullable) receives P+1 flags per row
 * at offset sel_off[r].
 */
void orc_retrieval_rows(const int64_t* dims /* B, Lq, Lk, H, Hkv, q_pos0 */,
                        const uint16_t* q, const uint16_t* k, const uint16_t* v,
                        const uint16_t* q16, int64_t Hq16, const uint16_t* k16,
                        int64_t Hk16, int64_t n_rows, const int64_t* row_b,
                        const int64_t* row_i, const int64_t* row_h,
                        const int64_t* row_hq16, const int64_t* row_hk16,
                        double p, double scale, double* o, double* lse,
                        double* t, int64_t* jtie, int64_t* count,
                        double* mass_frac, uint8_t* sel, const int64_t* sel_off)
{
    orc_shape S = {dims[0], dims[1], dims[2], dims[3], dims[4], dims[5]};
    int64_t G = S.H / S.Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t b = row_b[r], i = row_i[r], h = row_h[r], g = h / G;
        int64_t P = S.q_pos0 + i;
        int64_t n = P + 1;
        double* s = (double*)malloc((size_t)n * sizeof(double));
        uint8_t* mask = sel ? sel + sel_off[r] : (uint8_t*)malloc((size_t)n);
        const uint16_t* q16r = q16 + ((b * S.Lq + i) * Hq16 + row_hq16[r]) * ORC_R;
        const uint16_t* k16b = k16 + (b * S.Lk * Hk16 + row_hk16[r]) * ORC_R;
        orc_scores(q16r, k16b, n, Hk16 * ORC_R, s);
        orc_topp(s, n, p, mask, &t[r], &jtie[r], &count[r], &mass_frac[r], NULL, NULL);
        int64_t* idx = (int64_t*)malloc((size_t)count[r] * sizeof(int64_t));
        int64_t c = 0;
        for (int64_t j = 0; j < n; ++j)
            if (mask[j])
                idx[c++] = j;
        orc_attend(q + orc_q_off(&S, b, i, h), k + orc_kv_off(&S, b, 0, g),
                   S.Hkv * ORC_D, v + orc_kv_off(&S, b, 0, g), S.Hkv * ORC_D,
                   idx, c, scale, o + r * ORC_D, &lse[r]);
        free(idx);
        free(s);
        if (!sel)
            free(mask);
    }
}

/* Local rows (window, n_sink) or, with window >= P + 1 and n_sink = 0, dense
 * causal rows.  Same row conventions as orc_retrieval_rows. */
void orc_local_rows(const int64_t* dims, const uint16_t* q, const uint16_t* k,
                    const uint16_t* v, int64_t n_rows, const int64_t* row_b,
                    const int64_t* row_i, const int64_t* row_h, int64_t window,
                    int64_t n_sink, double scale, double* o, double* lse)
{
    orc_shape S = {dims[0], dims[1], dims[2], dims[3], dims[4], dims[5]};
    int64_t G = S.H / S.Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t b = row_b[r], i = row_i[r], h = row_h[r], g = h / G;
        int64_t P = S.q_pos0 + i;
        int64_t* idx = (int64_t*)malloc((size_t)(P + 1) * sizeof(int64_t));
        int64_t c = orc_local_set(P, window, n_sink, idx);
        orc_attend(q + orc_q_off(&S, b, i, h), k + orc_kv_off(&S, b, 0, g),
                   S.Hkv * ORC_D, v + orc_kv_off(&S, b, 0, g), S.Hkv * ORC_D,
                   idx, c, scale, o + r * ORC_D, &lse[r]);
        free(idx);
    }
}
