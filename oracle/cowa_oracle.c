/*
 * CoWindow Attention (CoWA) -- fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * What it computes (plain definitions, no blocking, no fusion, no reordering):
 *
 *   Mask.  "CoWindow Attention: Full Causal Coverage Is a Collective Property"
 *   (paper digest, section "method key points"): every KV head has a shared
 *   prefix-sink window, a shared near-diagonal window and its own
 *   complementary long-range window, described by the quadruple
 *   (sink width S, near width N, gap G, long-range width W), with
 *   bottom-right-aligned causal distance.  The exact breakpoint rule is the
 *   one this library fixes: for query row i and key j, p = i + Lk - Lq and
 *   d = p - j; key j is visible to window index w iff d >= 0 and
 *   (j < S  or  d < N  or  N+G+w*W <= d < N+G+(w+1)*W).
 *   Query head hq uses KV head floor(hq / g), g = Hq / Hkv (contiguous GQA
 *   grouping); the window index is the global KV-head index
 *   (local head + kv_head_offset), or widx[global head] when a window map is
 *   given (the duplicated-window control of the paper's 8K ablation).
 *
 *   Forward.  s_ij = scale * <q_i, k_j> on visible pairs, -inf elsewhere;
 *   LSE_i = log sum_j exp(s_ij) (natural log); P_ij = exp(s_ij - LSE_i);
 *   O_i = sum_j P_ij v_j.  A row with no visible key has O = 0, LSE = -inf.
 *
 *   Backward (analytic gradients of the forward):
 *   dV_j = sum_i P_ij dO_i;  dP_ij = <dO_i, v_j>;  delta_i = <dO_i, O_i>;
 *   dS_ij = P_ij (dP_ij - delta_i);  dQ_i = scale sum_j dS_ij k_j;
 *   dK_j = scale sum_i dS_ij q_i;  dK and dV summed over the g query heads
 *   that share a KV head.
 *
 *   Decode.  The same forward with Lq = 1 over the first seqlens[b] keys of
 *   a KV cache, so p = seqlens[b] - 1 (the new token sees itself).
 *
 * Inputs are either fp64 or bf16 bit patterns (uint16), selected by a flag;
 * bf16 values are widened exactly to fp64 so both sides of a parity test
 * see the same numbers.  All tensors are contiguous: Q/O [B, Lq, Hq, d],
 * K/V [B, Lk, Hkv, d], LSE [B, Hq, Lq].  Arithmetic is fp64 throughout.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int64_t B, Lq, Lk, Hq, Hkv, D;   /* Hkv: heads present in the tensors */
    int64_t S, N, G, W;              /* window quadruple */
    int64_t kv_head_offset;          /* global index of local KV head 0 */
    const int64_t *widx;             /* optional window index per global head */
    double scale;
    int bf16;                        /* inputs are bf16 bit patterns */
} oracle_ctx;

static double widen(const void *base, int64_t idx, int bf16)
{
    if (!bf16) return ((const double *)base)[idx];
    uint32_t u = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Visibility of key j to aligned query position p under window index w. */
int cowa_ref_visible(int64_t p, int64_t j, int64_t w, int64_t S, int64_t N,
                     int64_t G, int64_t W)
{
    int64_t d = p - j;
    if (j < 0 || d < 0) return 0;
    if (j < S) return 1;
    if (d < N) return 1;
    return d >= N + G + w * W && d < N + G + (w + 1) * W;
}

/* Dense mask of one window index: out[i*Lk + j] in {0,1}. */
void cowa_ref_mask(int64_t Lq, int64_t Lk, int64_t w, int64_t S, int64_t N,
                   int64_t G, int64_t W, uint8_t *out)
{
    for (int64_t i = 0; i < Lq; ++i) {
        int64_t p = i + Lk - Lq;
        for (int64_t j = 0; j < Lk; ++j)
            out[i * Lk + j] = (uint8_t)cowa_ref_visible(p, j, w, S, N, G, W);
    }
}

int cowa_ref_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int64_t window_of(const oracle_ctx *c, int64_t hkv_local)
{
    int64_t hg = hkv_local + c->kv_head_offset;
    return c->widx ? c->widx[hg] : hg;
}

static int64_t q_index(const oracle_ctx *c, int64_t b, int64_t i, int64_t hq)
{
    return ((b * c->Lq + i) * c->Hq + hq) * c->D;
}

static int64_t k_index(const oracle_ctx *c, int64_t b, int64_t j, int64_t h)
{
    return ((b * c->Lk + j) * c->Hkv + h) * c->D;
}

/*
 * One query row of the forward.  Fills s[0..Lk) with exp-ready scores
 * (-inf where invisible), returns LSE, writes O_i (length D) and, when
 * prob != NULL, P_ij for every j.
 */
static double fwd_row(const oracle_ctx *c, const void *q, const void *k,
                      const void *v, int64_t b, int64_t hq, int64_t i,
                      double *o, double *s, double *prob)
{
    const int64_t g = c->Hq / c->Hkv, h = hq / g, w = window_of(c, h);
    const int64_t p = i + c->Lk - c->Lq, D = c->D;
    const int64_t qi = q_index(c, b, i, hq);
    double m = -INFINITY;
    for (int64_t j = 0; j < c->Lk; ++j) {
        if (!cowa_ref_visible(p, j, w, c->S, c->N, c->G, c->W)) {
            s[j] = -INFINITY;
            continue;
        }
        const int64_t kj = k_index(c, b, j, h);
        double dot = 0.0;
        for (int64_t x = 0; x < D; ++x)
            dot += widen(q, qi + x, c->bf16) * widen(k, kj + x, c->bf16);
        s[j] = c->scale * dot;
        if (s[j] > m) m = s[j];
    }
    for (int64_t x = 0; x < D; ++x) o[x] = 0.0;
    if (m == -INFINITY) {
        if (prob)
            for (int64_t j = 0; j < c->Lk; ++j) prob[j] = 0.0;
        return -INFINITY;
    }
    double sum = 0.0;
    for (int64_t j = 0; j < c->Lk; ++j)
        if (s[j] != -INFINITY) sum += exp(s[j] - m);
    const double lse = m + log(sum);
    for (int64_t j = 0; j < c->Lk; ++j) {
        double pj = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - lse);
        if (prob) prob[j] = pj;
        if (pj == 0.0) continue;
        const int64_t vj = k_index(c, b, j, h);
        for (int64_t x = 0; x < D; ++x) o[x] += pj * widen(v, vj + x, c->bf16);
    }
    return lse;
}

static void make_ctx(oracle_ctx *c, int64_t B, int64_t Lq, int64_t Lk,
                     int64_t Hq, int64_t Hkv, int64_t D, int64_t S, int64_t N,
                     int64_t G, int64_t W, int64_t off, const int64_t *widx,
                     double scale, int bf16)
{
    c->B = B; c->Lq = Lq; c->Lk = Lk; c->Hq = Hq; c->Hkv = Hkv; c->D = D;
    c->S = S; c->N = N; c->G = G; c->W = W;
    c->kv_head_offset = off; c->widx = widx; c->scale = scale; c->bf16 = bf16;
}

/* Full forward.  o [B,Lq,Hq,D], lse [B,Hq,Lq]. */
void cowa_ref_fwd(int64_t B, int64_t Lq, int64_t Lk, int64_t Hq, int64_t Hkv,
                  int64_t D, int64_t S, int64_t N, int64_t G, int64_t W,
                  int64_t off, const int64_t *widx, double scale, int bf16,
                  const void *q, const void *k, const void *v, double *o,
                  double *lse)
{
    oracle_ctx c;
    make_ctx(&c, B, Lq, Lk, Hq, Hkv, D, S, N, G, W, off, widx, scale, bf16);
    const int64_t total = B * Hq * Lq;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < total; ++t) {
            const int64_t i = t % Lq, hq = (t / Lq) % Hq, b = t / (Lq * Hq);
            lse[(b * Hq + hq) * Lq + i] =
                fwd_row(&c, q, k, v, b, hq, i, o + q_index(&c, b, i, hq), s, NULL);
        }
        free(s);
    }
}

/* Forward on selected rows.  rows: n triples (b, hq, i); o [n, D], lse [n]. */
void cowa_ref_fwd_rows(int64_t B, int64_t Lq, int64_t Lk, int64_t Hq,
                       int64_t Hkv, int64_t D, int64_t S, int64_t N, int64_t G,
                       int64_t W, int64_t off, const int64_t *widx,
                       double scale, int bf16, const void *q, const void *k,
                       const void *v, int64_t n, const int64_t *rows, double *o,
                       double *lse)
{
    oracle_ctx c;
    make_ctx(&c, B, Lq, Lk, Hq, Hkv, D, S, N, G, W, off, widx, scale, bf16);
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n; ++r) {
            const int64_t *t = rows + 3 * r;
            lse[r] = fwd_row(&c, q, k, v, t[0], t[1], t[2], o + r * D, s, NULL);
        }
        free(s);
    }
}

/*
 * Backward terms of one query row: accumulates dQ_i into dq_row and, when
 * dk/dv are given (per-head accumulators [Lk, D]), adds this row's share of
 * dK_j and dV_j for every visible j.
 */
static void bwd_row(const oracle_ctx *c, const void *q, const void *k,
                    const void *v, const void *dout, int64_t b, int64_t hq,
                    int64_t i, double *s, double *prob, double *o,
                    double *dq_row, double *dk, double *dv)
{
    const int64_t g = c->Hq / c->Hkv, h = hq / g, D = c->D;
    const int64_t qi = q_index(c, b, i, hq);
    const double lse = fwd_row(c, q, k, v, b, hq, i, o, s, prob);
    for (int64_t x = 0; x < D; ++x) dq_row[x] = 0.0;
    if (lse == -INFINITY) return;
    double delta = 0.0;
    for (int64_t x = 0; x < D; ++x) delta += widen(dout, qi + x, c->bf16) * o[x];
    for (int64_t j = 0; j < c->Lk; ++j) {
        const double pij = prob[j];
        if (s[j] == -INFINITY) continue;
        const int64_t kj = k_index(c, b, j, h);
        double dp = 0.0;
        for (int64_t x = 0; x < D; ++x)
            dp += widen(dout, qi + x, c->bf16) * widen(v, kj + x, c->bf16);
        const double ds = pij * (dp - delta);
        for (int64_t x = 0; x < D; ++x)
            dq_row[x] += c->scale * ds * widen(k, kj + x, c->bf16);
        if (dk)
            for (int64_t x = 0; x < D; ++x)
                dk[j * D + x] += c->scale * ds * widen(q, qi + x, c->bf16);
        if (dv)
            for (int64_t x = 0; x < D; ++x)
                dv[j * D + x] += pij * widen(dout, qi + x, c->bf16);
    }
}

/* Full backward.  dq [B,Lq,Hq,D], dk/dv [B,Lk,Hkv,D]. */
void cowa_ref_bwd(int64_t B, int64_t Lq, int64_t Lk, int64_t Hq, int64_t Hkv,
                  int64_t D, int64_t S, int64_t N, int64_t G, int64_t W,
                  int64_t off, const int64_t *widx, double scale, int bf16,
                  const void *q, const void *k, const void *v, const void *dout,
                  double *dq, double *dk, double *dv)
{
    oracle_ctx c;
    make_ctx(&c, B, Lq, Lk, Hq, Hkv, D, S, N, G, W, off, widx, scale, bf16);
    const int64_t g = Hq / Hkv;
    /* One (b, KV head) per task: its g query heads and all rows run in order,
       so the dK/dV accumulators of that head have a single writer. */
#pragma omp parallel
    {
        const size_t nl = (size_t)(Lk > 0 ? Lk : 1);
        double *s = (double *)malloc(sizeof(double) * nl);
        double *prob = (double *)malloc(sizeof(double) * nl);
        double *o = (double *)malloc(sizeof(double) * (size_t)D);
        double *dkh = (double *)malloc(sizeof(double) * nl * (size_t)D);
        double *dvh = (double *)malloc(sizeof(double) * nl * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < B * Hkv; ++t) {
            const int64_t b = t / Hkv, h = t % Hkv;
            memset(dkh, 0, sizeof(double) * (size_t)(Lk * D));
            memset(dvh, 0, sizeof(double) * (size_t)(Lk * D));
            for (int64_t hq = h * g; hq < (h + 1) * g; ++hq)
                for (int64_t i = 0; i < Lq; ++i)
                    bwd_row(&c, q, k, v, dout, b, hq, i, s, prob, o,
                            dq + q_index(&c, b, i, hq), dkh, dvh);
            for (int64_t j = 0; j < Lk; ++j)
                for (int64_t x = 0; x < D; ++x) {
                    dk[k_index(&c, b, j, h) + x] = dkh[j * D + x];
                    dv[k_index(&c, b, j, h) + x] = dvh[j * D + x];
                }
        }
        free(s); free(prob); free(o); free(dkh); free(dvh);
    }
}

/* dQ of selected rows.  rows: n triples (b, hq, i); dq [n, D]. */
void cowa_ref_bwd_dq_rows(int64_t B, int64_t Lq, int64_t Lk, int64_t Hq,
                          int64_t Hkv, int64_t D, int64_t S, int64_t N,
                          int64_t G, int64_t W, int64_t off,
                          const int64_t *widx, double scale, int bf16,
                          const void *q, const void *k, const void *v,
                          const void *dout, int64_t n, const int64_t *rows,
                          double *dq)
{
    oracle_ctx c;
    make_ctx(&c, B, Lq, Lk, Hq, Hkv, D, S, N, G, W, off, widx, scale, bf16);
#pragma omp parallel
    {
        const size_t nl = (size_t)(Lk > 0 ? Lk : 1);
        double *s = (double *)malloc(sizeof(double) * nl);
        double *prob = (double *)malloc(sizeof(double) * nl);
        double *o = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n; ++r) {
            const int64_t *t = rows + 3 * r;
            bwd_row(&c, q, k, v, dout, t[0], t[1], t[2], s, prob, o, dq + r * D,
                    NULL, NULL);
        }
        free(s); free(prob); free(o);
    }
}

/*
 * dK and dV of selected key columns.  cols: n triples (b, hkv, j);
 * dk/dv [n, D].  Every (query head of the group, row) that sees key j
 * contributes; the rows are independent and summed in a fixed order per
 * thread, then across threads.
 */
void cowa_ref_bwd_dkv_cols(int64_t B, int64_t Lq, int64_t Lk, int64_t Hq,
                           int64_t Hkv, int64_t D, int64_t S, int64_t N,
                           int64_t G, int64_t W, int64_t off,
                           const int64_t *widx, double scale, int bf16,
                           const void *q, const void *k, const void *v,
                           const void *dout, int64_t n, const int64_t *cols,
                           double *dk, double *dv)
{
    oracle_ctx c;
    make_ctx(&c, B, Lq, Lk, Hq, Hkv, D, S, N, G, W, off, widx, scale, bf16);
    const int64_t g = Hq / Hkv;
    for (int64_t r = 0; r < n; ++r) {
        const int64_t b = cols[3 * r], h = cols[3 * r + 1], j = cols[3 * r + 2];
        const int64_t w = window_of(&c, h);
        for (int64_t x = 0; x < D; ++x) dk[r * D + x] = dv[r * D + x] = 0.0;
#pragma omp parallel
        {
            const size_t nl = (size_t)(Lk > 0 ? Lk : 1);
            double *s = (double *)malloc(sizeof(double) * nl);
            double *prob = (double *)malloc(sizeof(double) * nl);
            double *o = (double *)malloc(sizeof(double) * (size_t)D);
            double *acc_k = (double *)calloc((size_t)D, sizeof(double));
            double *acc_v = (double *)calloc((size_t)D, sizeof(double));
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = 0; t < g * Lq; ++t) {
                const int64_t hq = h * g + t / Lq, i = t % Lq;
                const int64_t p = i + Lk - Lq;
                if (!cowa_ref_visible(p, j, w, S, N, G, W)) continue;
                const int64_t qi = q_index(&c, b, i, hq), kj = k_index(&c, b, j, h);
                const double lse = fwd_row(&c, q, k, v, b, hq, i, o, s, prob);
                double delta = 0.0, dp = 0.0;
                for (int64_t x = 0; x < D; ++x) {
                    delta += widen(dout, qi + x, bf16) * o[x];
                    dp += widen(dout, qi + x, bf16) * widen(v, kj + x, bf16);
                }
                (void)lse;
                const double pij = prob[j];
                const double ds = pij * (dp - delta);
                for (int64_t x = 0; x < D; ++x) {
                    acc_k[x] += scale * ds * widen(q, qi + x, bf16);
                    acc_v[x] += pij * widen(dout, qi + x, bf16);
                }
            }
#pragma omp critical
            for (int64_t x = 0; x < D; ++x) {
                dk[r * D + x] += acc_k[x];
                dv[r * D + x] += acc_v[x];
            }
            free(s); free(prob); free(o); free(acc_k); free(acc_v);
        }
    }
}

/*
 * Single-token decode over a KV cache.  q [B, Hq, D]; kc/vc
 * [B, Lcap, Hkv, D]; seqlens [B] (keys 0..seqlens[b]-1 are valid and the
 * new token is the last of them); o [B, Hq, D]; lse [B, Hq].
 */
void cowa_ref_decode(int64_t B, int64_t Lcap, int64_t Hq, int64_t Hkv,
                     int64_t D, int64_t S, int64_t N, int64_t G, int64_t W,
                     int64_t off, const int64_t *widx, double scale, int bf16,
                     const void *q, const void *kc, const void *vc,
                     const int32_t *seqlens, double *o, double *lse)
{
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lcap > 0 ? Lcap : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < B * Hq; ++t) {
            const int64_t b = t / Hq, hq = t % Hq;
            /* View batch row b as a forward problem with Lq = 1 over the
               first seqlens[b] keys of its cache. */
            oracle_ctx c;
            make_ctx(&c, 1, 1, seqlens[b], Hq, Hkv, D, S, N, G, W, off, widx,
                     scale, bf16);
            const size_t esz = bf16 ? 2 : 8;
            const char *qb = (const char *)q + (size_t)(b * Hq * D) * esz;
            const char *kb = (const char *)kc + (size_t)(b * Lcap * Hkv * D) * esz;
            const char *vb = (const char *)vc + (size_t)(b * Lcap * Hkv * D) * esz;
            lse[t] = fwd_row(&c, qb, kb, vb, 0, hq, 0, o + t * D, s, NULL);
        }
        free(s);
    }
}

/*
 * Brute-force visible-pair counts per tile of one window index, for checking
 * the visible-tile schedule: out[qt * nkt + kt] = number of (i, j) with
 * i in [qt*BM, min((qt+1)*BM, Lq)), j in [kt*BN, min((kt+1)*BN, Lk)) and key
 * j visible to row i.
 */
void cowa_ref_tile_counts(int64_t Lq, int64_t Lk, int64_t w, int64_t S,
                          int64_t N, int64_t G, int64_t W, int64_t BM,
                          int64_t BN, int64_t *out)
{
    const int64_t nqt = (Lq + BM - 1) / BM, nkt = (Lk + BN - 1) / BN;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t qt = 0; qt < nqt; ++qt) {
        for (int64_t kt = 0; kt < nkt; ++kt) out[qt * nkt + kt] = 0;
        const int64_t i1 = (qt + 1) * BM < Lq ? (qt + 1) * BM : Lq;
        for (int64_t i = qt * BM; i < i1; ++i) {
            const int64_t p = i + Lk - Lq;
            for (int64_t j = 0; j < Lk; ++j)
                out[qt * nkt + j / BN] += cowa_ref_visible(p, j, w, S, N, G, W);
        }
    }
}
