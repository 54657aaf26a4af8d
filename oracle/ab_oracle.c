/*
 * ab_oracle.c -- plain, slow CPU oracle for the AB-Attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call this
 * file: only the tests, the smoke check and the benchmark's CPU-baseline leg do. It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Source of the method: the news page "AB-Attention ускорил генерацию видео до 2,23×
 * и пропускает 92% внимания" (app.hamidun.com), section «Три приёма AB-Attention»:
 *   - IBCS: queries in 128-token blocks, 8 clusters per block, each with a centroid
 *     and a weight equal to its share of the block's queries; a key block is scored
 *     by the weighted attention of the centroids to its mean key;
 *   - SIP: key blocks drawn with probability proportional to the score, the most
 *     important always kept, each kept block weighted by 1/p (Horvitz-Thompson) in
 *     both the numerator and the softmax normaliser, i.e. a logit shift;
 *   - section «Где ломаются прежние разреженные схемы»: top-k keeps the K best blocks
 *     and drops the rest from numerator and normaliser.
 * Points the page leaves open are fixed here as plain readings (listed in the design
 * notes): deterministic k-means init, squared Euclidean distance on raw Q, ties to the
 * lowest cluster, 1/sqrt(d) score scale with the softmax over all key blocks, exact
 * integer water-filling for p_j = min(1, c s_j), Philox4x32-10 draws keyed by
 * (seed) with counter (kb, qb, h, b).
 *
 * Inputs Q, K, V are raw bf16 bit patterns (uint16), read exactly as fp32 values;
 * all arithmetic is fp64 unless a step says otherwise. Layout BHND, contiguous.
 * Every function returns 0 on success or a negative code on bad arguments.
 *
 * Parity pins (tests/): hand-worked golden fixtures for k-means, IBCS scores and SIP;
 * closed forms (sum of scores = 1, sum of p = K, p = 1/4 -> w = 4); torch SDPA in fp64
 * for the all-blocks case, top-k case and integer-weight duplication case; exact
 * rational water-filling; Monte Carlo unbiasedness; Philox against an independent
 * implementation; torch autograd in fp64 of the masked, log-weight-shifted softmax
 * attention for the gradients, and the softmax's shift invariance (sum_t dK_t = 0).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_BLOCK 128

static double bf16_val(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int64_t n_blocks_of(int N_pad) { return N_pad / ORC_BLOCK; }

static int check_shape(int B, int H, int N, int N_pad, int d)
{
    if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return -1;
    if (N_pad % ORC_BLOCK != 0 || N > N_pad || N_pad - N >= ORC_BLOCK) return -1;
    return 0;
}

/* ------------------------------------------------------------------------------
 * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
 * 1, 2, 3", SC'11): 10 rounds of the 4x32 S-box on a 128-bit counter, with the
 * 64-bit key bumped by the Weyl constants between rounds.
 * ------------------------------------------------------------------------------ */
void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    const uint32_t mul0 = 0xD2511F53u, mul1 = 0xCD9E8D57u;
    const uint32_t weyl0 = 0x9E3779B9u, weyl1 = 0xBB67AE85u;
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += weyl0;
            k1 += weyl1;
        }
        uint64_t prod0 = (uint64_t)mul0 * c0;
        uint64_t prod1 = (uint64_t)mul1 * c2;
        uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
        uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* ------------------------------------------------------------------------------
 * Mean key of each key unit of U tokens (IBCS: "its averaged keys"; U = 128 is the
 * key block, U = 4 the page's fine-grained selection unit, third technique), over
 * the valid tokens t < N only. A unit with no valid token does not exist: its row is
 * 0 (the score gives it nothing). kbar: [B, H, N_pad / U, d].
 * ------------------------------------------------------------------------------ */
int orc_mean_key_u(const uint16_t *K, int B, int H, int N, int N_pad, int d, int U, double *kbar)
{
    if (!K || !kbar || check_shape(B, H, N, N_pad, d) || U < 1 || N_pad % U != 0) return -1;
    const int64_t nku = N_pad / U;
    const int64_t rows = (int64_t)B * H * nku;
#pragma omp parallel for schedule(dynamic, 64)
    for (int64_t r = 0; r < rows; ++r) {
        const int64_t bh = r / nku, j = r % nku;
        const int64_t t0 = j * U;
        int64_t t1 = t0 + U;
        if (t1 > N) t1 = N;
        double *out = kbar + r * d;
        for (int i = 0; i < d; ++i) out[i] = 0.0;
        if (t1 <= t0) continue;
        for (int64_t t = t0; t < t1; ++t) {
            const uint16_t *row = K + (bh * N_pad + t) * d;
            for (int i = 0; i < d; ++i) out[i] += bf16_val(row[i]);
        }
        for (int i = 0; i < d; ++i) out[i] /= (double)(t1 - t0);
    }
    return 0;
}

int orc_mean_key(const uint16_t *K, int B, int H, int N, int N_pad, int d, double *kbar)
{
    return orc_mean_key_u(K, B, H, N, N_pad, d, ORC_BLOCK, kbar);
}

/* ------------------------------------------------------------------------------
 * IBCS per-block k-means (Lloyd iterations), C clusters, T iterations.
 *   init   : centroid c = query at block-local index c*floor(n_v/C) (n_v >= C), else
 *            index min(c, n_v-1);
 *   assign : argmin over c of the squared Euclidean distance |q - c_c|^2, ties to the
 *            lowest c;
 *   update : c_c = mean of its members; an empty cluster keeps its centroid;
 *   output : centroids after the T-th update, weights = member count / n_v from the
 *            T-th assignment (each cluster weighted by its share of the block's queries:
 *            AB-Attention news page, «Три приёма AB-Attention», first technique IBCS).
 * cent [B,H,nqb,C,d], wts [B,H,nqb,C], assign [B,H,N_pad] (optional; 255 on padding),
 * min_gap [B,H,nqb] (optional): the smallest relative gap (d2 - d1) / d2 between the
 * best and second-best distance seen by any query in any iteration (1 when C = 1).
 * inertia [B,H,nqb,T] (optional): sum of squared distances to the assigned centroid
 * at each assignment.
 * ------------------------------------------------------------------------------ */
int orc_kmeans(const uint16_t *Q, int B, int H, int N, int N_pad, int d, int C, int T,
               double *cent, double *wts, uint8_t *assign, double *min_gap, double *inertia)
{
    if (!Q || !cent || !wts || check_shape(B, H, N, N_pad, d)) return -1;
    if (C < 1 || C > 64 || T < 1) return -1;
    const int64_t nqb = n_blocks_of(N_pad);
    const int64_t rows = (int64_t)B * H * nqb;
    int rc = 0;
#pragma omp parallel
    {
        double *q = (double *)malloc(sizeof(double) * ORC_BLOCK * d);
        double *sum = (double *)malloc(sizeof(double) * C * d);
        int *cnt = (int *)malloc(sizeof(int) * C);
        int *lab = (int *)malloc(sizeof(int) * ORC_BLOCK);
        if (!q || !sum || !cnt || !lab) {
#pragma omp atomic write
            rc = -2;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < rows; ++r) {
            if (rc) continue;
            const int64_t bh = r / nqb, qb = r % nqb;
            const int64_t t0 = qb * ORC_BLOCK;
            int nv = (int)((N - t0) < ORC_BLOCK ? (N - t0) : ORC_BLOCK);
            for (int t = 0; t < nv; ++t)
                for (int i = 0; i < d; ++i) q[t * d + i] = bf16_val(Q[(bh * N_pad + t0 + t) * d + i]);
            double *cc = cent + r * (int64_t)C * d;
            for (int c = 0; c < C; ++c) {
                int src = nv >= C ? c * (nv / C) : (c < nv - 1 ? c : nv - 1);
                for (int i = 0; i < d; ++i) cc[c * d + i] = q[src * d + i];
            }
            double gap_min = 1.0;
            for (int it = 0; it < T; ++it) {
                double inert = 0.0;
                for (int t = 0; t < nv; ++t) {
                    double best = INFINITY, second = INFINITY;
                    int arg = 0;
                    for (int c = 0; c < C; ++c) {
                        double dist = 0.0;
                        for (int i = 0; i < d; ++i) {
                            double diff = q[t * d + i] - cc[c * d + i];
                            dist += diff * diff;
                        }
                        if (dist < best) {
                            second = best;
                            best = dist;
                            arg = c;
                        } else if (dist < second) {
                            second = dist;
                        }
                    }
                    lab[t] = arg;
                    inert += best;
                    if (C > 1) {
                        double g = second > 0.0 ? (second - best) / second : 0.0;
                        if (g < gap_min) gap_min = g;
                    }
                }
                if (inertia) inertia[r * T + it] = inert;
                for (int c = 0; c < C; ++c) {
                    cnt[c] = 0;
                    for (int i = 0; i < d; ++i) sum[c * d + i] = 0.0;
                }
                for (int t = 0; t < nv; ++t) {
                    cnt[lab[t]] += 1;
                    for (int i = 0; i < d; ++i) sum[lab[t] * d + i] += q[t * d + i];
                }
                for (int c = 0; c < C; ++c)
                    if (cnt[c] > 0)
                        for (int i = 0; i < d; ++i) cc[c * d + i] = sum[c * d + i] / cnt[c];
            }
            for (int c = 0; c < C; ++c) wts[r * C + c] = (double)cnt[c] / (double)nv;
            if (assign) {
                uint8_t *a = assign + bh * N_pad + t0;
                for (int t = 0; t < ORC_BLOCK; ++t) a[t] = t < nv ? (uint8_t)lab[t] : 255;
            }
            if (min_gap) min_gap[r] = gap_min;
        }
        free(q);
        free(sum);
        free(cnt);
        free(lab);
    }
    return rc;
}

/* ------------------------------------------------------------------------------
 * IBCS block score: for each query block, L[c, j] = cent_c . kbar_j / sqrt(d); a
 * softmax over the existing key units j < nkb_valid for each centroid c;
 * s_j = sum_c w_c softmax_j(L[c,.]), and s_j = 0 for j >= nkb_valid (units past the
 * sequence end).
 * cent [B,H,nqb,C,d], wts [B,H,nqb,C], kbar [B,H,nkb,d] -> scores [B,H,nqb,nkb].
 * ------------------------------------------------------------------------------ */
int orc_score_u(const double *cent, const double *wts, const double *kbar, int B, int H,
                int nqb, int nkb, int nkb_valid, int C, int d, double *scores)
{
    if (!cent || !wts || !kbar || !scores || B <= 0 || H <= 0 || nqb <= 0 || nkb <= 0 ||
        nkb_valid < 1 || nkb_valid > nkb || C < 1 || d <= 0)
        return -1;
    const int64_t rows = (int64_t)B * H * nqb;
    const double scale = 1.0 / sqrt((double)d);
    int rc = 0;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * nkb);
        if (!logit) {
#pragma omp atomic write
            rc = -2;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < rows; ++r) {
            if (rc) continue;
            const int64_t bh = r / nqb;
            const double *kb = kbar + bh * (int64_t)nkb * d;
            double *s = scores + r * nkb;
            for (int j = 0; j < nkb; ++j) s[j] = 0.0;
            for (int c = 0; c < C; ++c) {
                const double *cv = cent + (r * C + c) * (int64_t)d;
                double m = -INFINITY;
                for (int j = 0; j < nkb_valid; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < d; ++i) acc += cv[i] * kb[(int64_t)j * d + i];
                    logit[j] = acc * scale;
                    if (logit[j] > m) m = logit[j];
                }
                double z = 0.0;
                for (int j = 0; j < nkb_valid; ++j) z += exp(logit[j] - m);
                const double wc = wts[r * C + c];
                for (int j = 0; j < nkb_valid; ++j) s[j] += wc * exp(logit[j] - m) / z;
            }
        }
        free(logit);
    }
    return rc;
}

int orc_score(const double *cent, const double *wts, const double *kbar, int B, int H,
              int nqb, int nkb, int C, int d, double *scores)
{
    return orc_score_u(cent, wts, kbar, B, H, nqb, nkb, nkb, C, d, scores);
}

/* ------------------------------------------------------------------------------
 * SIP selection for one row, in exact integer arithmetic so that any implementation
 * reproduces it bit for bit:
 *   u_j = floor(s_j * 2^50) (exact), U = sum u_j (exact), K = min(budget, nkb);
 *   if #{u_j > 0} <= K every positive block is kept with p = 1;
 *   otherwise grow the saturated set S from empty by S <- S + {j : k u_j >= R} with
 *   k = K - |S| and R = U - sum_S u, until no block joins; then p_j = 1 on S and
 *   p_j = (double)(k u_j) / (double)R elsewhere (IEEE divide), so sum p = K;
 *   draw: Philox4x32-10, key (lo32 seed, hi32 seed), counter (kb, qb, h, b);
 *   R53 = ((x0 << 32) | x1) >> 11; keep iff (double)R53 < p_j * 2^53;
 *   kept blocks in ascending order, w_j = (float)(1 / p_j).
 * Returns 1 in *bad when a score is not finite or outside [0, 2], or when the exact sum
 * U does not fit in 64 bits (sum of the row's scores of 2^14 or more: never for IBCS
 * scores, whose rows sum to 1), so that every integer above stays exact.
 * ------------------------------------------------------------------------------ */
static int sip_row(const float *s, int nkb, int K, uint64_t seed, int b, int h, int qb,
                   int32_t *idx, int32_t *cnt_out, float *w, double *p, uint64_t *u)
{
    for (int j = 0; j < nkb; ++j) {
        float v = s[j];
        if (!(v >= 0.0f && v <= 2.0f)) return 1;
        u[j] = (uint64_t)floor(ldexp((double)v, 50));
    }
    unsigned __int128 U128 = 0;
    int positive = 0;
    for (int j = 0; j < nkb; ++j) {
        U128 += u[j];
        positive += u[j] > 0;
    }
    if (U128 >> 64) return 1;
    const uint64_t U = (uint64_t)U128;
    unsigned char *inS = (unsigned char *)calloc((size_t)nkb, 1);
    if (!inS) return 2;
    uint64_t k = 0, R = 0;
    if (positive <= K) {
        for (int j = 0; j < nkb; ++j) inS[j] = u[j] > 0;
    } else {
        int sizeS = 0;
        uint64_t sumS = 0;
        for (;;) {
            k = (uint64_t)(K - sizeS);
            R = U - sumS;
            int added = 0;
            for (int j = 0; j < nkb; ++j) {
                if (inS[j]) continue;
                if ((unsigned __int128)k * u[j] >= (unsigned __int128)R) {
                    inS[j] = 2; /* joins in this pass */
                    added += 1;
                }
            }
            if (!added) break;
            for (int j = 0; j < nkb; ++j)
                if (inS[j] == 2) {
                    inS[j] = 1;
                    sizeS += 1;
                    sumS += u[j];
                }
        }
    }
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    int c = 0;
    for (int j = 0; j < nkb; ++j) {
        double pj;
        if (inS[j]) pj = 1.0;
        else if (u[j] == 0 || positive <= K) pj = 0.0;
        else pj = (double)(k * u[j]) / (double)R;
        if (p) p[j] = pj;
        uint32_t ctr[4] = {(uint32_t)j, (uint32_t)qb, (uint32_t)h, (uint32_t)b};
        uint32_t x[4];
        orc_philox4x32_10(ctr, key, x);
        uint64_t r53 = (((uint64_t)x[0] << 32) | x[1]) >> 11;
        if ((double)r53 < ldexp(pj, 53)) {
            idx[c] = j;
            w[c] = (float)(1.0 / pj);
            c += 1;
        }
    }
    for (int j = c; j < nkb; ++j) {
        idx[j] = -1;
        w[j] = 0.0f;
    }
    *cnt_out = c;
    free(inS);
    return 0;
}

int orc_sip(const float *scores, int B, int H, int nqb, int nkb, int budget, uint64_t seed,
            int32_t *idx, int32_t *cnt, float *w, double *p, int32_t *bad_rows)
{
    if (!scores || !idx || !cnt || !w || B <= 0 || H <= 0 || nqb <= 0 || nkb <= 0 ||
        budget < 1)
        return -1;
    const int K = budget < nkb ? budget : nkb;
    const int64_t rows = (int64_t)B * H * nqb;
    int rc = 0;
#pragma omp parallel
    {
        uint64_t *u = (uint64_t *)malloc(sizeof(uint64_t) * nkb);
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < rows; ++r) {
            if (!u) continue;
            const int b = (int)(r / ((int64_t)H * nqb));
            const int h = (int)((r / nqb) % H);
            const int qb = (int)(r % nqb);
            int e = sip_row(scores + r * nkb, nkb, K, seed, b, h, qb, idx + r * nkb, cnt + r,
                            w + r * nkb, p ? p + r * nkb : NULL, u);
            if (bad_rows) bad_rows[r] = e;
            if (e) {
                cnt[r] = 0;
                for (int j = 0; j < nkb; ++j) {
                    idx[r * nkb + j] = -1;
                    w[r * nkb + j] = 0.0f;
                }
#pragma omp atomic write
                rc = 1;
            }
        }
        if (!u) {
#pragma omp atomic write
            rc = -2;
        }
        free(u);
    }
    return rc;
}

/* ------------------------------------------------------------------------------
 * Top-k selection: order blocks by (score descending, index ascending), keep the first
 * K = min(budget, nkb), report them in ascending order, weights 1.
 * ------------------------------------------------------------------------------ */
typedef struct {
    float s;
    int32_t j;
} orc_pair;

static int by_score_desc(const void *a, const void *b)
{
    const orc_pair *x = (const orc_pair *)a, *y = (const orc_pair *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int by_index(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

int orc_topk(const float *scores, int B, int H, int nqb, int nkb, int budget, int32_t *idx,
             int32_t *cnt, float *w)
{
    if (!scores || !idx || !cnt || B <= 0 || H <= 0 || nqb <= 0 || nkb <= 0 || budget < 1)
        return -1;
    const int K = budget < nkb ? budget : nkb;
    const int64_t rows = (int64_t)B * H * nqb;
    int rc = 0;
#pragma omp parallel
    {
        orc_pair *pr = (orc_pair *)malloc(sizeof(orc_pair) * nkb);
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < rows; ++r) {
            if (!pr) continue;
            const float *s = scores + r * nkb;
            int ok = 1;
            for (int j = 0; j < nkb; ++j) {
                if (!(s[j] >= 0.0f && s[j] <= 2.0f)) ok = 0;
                pr[j].s = s[j];
                pr[j].j = j;
            }
            int32_t *out = idx + r * nkb;
            if (!ok) {
                cnt[r] = 0;
                for (int j = 0; j < nkb; ++j) out[j] = -1;
#pragma omp atomic write
                rc = 1;
                continue;
            }
            qsort(pr, (size_t)nkb, sizeof(orc_pair), by_score_desc);
            for (int j = 0; j < K; ++j) out[j] = pr[j].j;
            qsort(out, (size_t)K, sizeof(int32_t), by_index);
            for (int j = K; j < nkb; ++j) out[j] = -1;
            cnt[r] = K;
            if (w)
                for (int j = 0; j < nkb; ++j) w[r * nkb + j] = j < K ? 1.0f : 0.0f;
        }
        if (!pr) {
#pragma omp atomic write
            rc = -2;
        }
        free(pr);
    }
    return rc;
}

/* ------------------------------------------------------------------------------
 * Block-sparse attention with Horvitz-Thompson weights over key units of U tokens
 * (U = 128: key blocks; U = 4: the page's fine-grained units), per query row i of
 * query block qb (128 queries):
 *   O_i = sum_{j in sel} w_j sum_{t in j, t<N} e^{q_i.k_t/sqrt(d)} v_t
 *         / sum_{j in sel} w_j sum_{t in j, t<N} e^{q_i.k_t/sqrt(d)}
 * (w = NULL means all weights 1, the top-k mode); unit j holds tokens
 * [j U, j U + U). Rows i >= N are 0 (lse 0); a row with an empty selection (or only
 * units past the sequence end) is 0 with lse = -inf. idx / w rows have N_pad / U
 * entries.
 * The `rows` list picks which (b, h, qb) blocks to compute: flat index
 * (b*H + h)*nqb + qb; NULL means all, in order. Outputs are per listed block:
 * out [n_rows, 128, d], lse [n_rows, 128] (ln of the denominator), and optionally
 * the unshifted numerator num [n_rows, 128, d] and denominator den [n_rows, 128].
 * ------------------------------------------------------------------------------ */
int orc_attn_rows_u(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B, int H,
                    int N, int N_pad, int d, int U, const int32_t *idx, const int32_t *cnt,
                    const float *w, int64_t n_rows, const int64_t *rows, double *out,
                    double *lse, double *num, double *den)
{
    if (!Q || !K || !V || !idx || !cnt || !out || check_shape(B, H, N, N_pad, d) || U < 1 ||
        N_pad % U != 0)
        return -1;
    const int64_t nqb = n_blocks_of(N_pad), nkb = N_pad / U;
    const int64_t total = (int64_t)B * H * nqb;
    if (!rows) n_rows = total;
    for (int64_t n = 0; n < n_rows; ++n)
        if (rows && (rows[n] < 0 || rows[n] >= total)) return -1;
    for (int64_t n = 0; n < n_rows; ++n) {
        const int64_t r = rows ? rows[n] : n;
        if (cnt[r] < 0 || cnt[r] > nkb) return -1;
        for (int32_t c = 0; c < cnt[r]; ++c)
            if (idx[r * nkb + c] < 0 || idx[r * nkb + c] >= nkb) return -1;
    }
    const double scale = 1.0 / sqrt((double)d);
    int rc = 0;
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * nkb * U);
        double *qv = (double *)malloc(sizeof(double) * d);
        double *acc = (double *)malloc(sizeof(double) * d);
        if (!logit || !qv || !acc) {
#pragma omp atomic write
            rc = -2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = 0; n < n_rows; ++n) {
            if (rc) continue;
            const int64_t r = rows ? rows[n] : n;
            const int64_t bh = r / nqb, qb = r % nqb;
            const int32_t nsel = cnt[r];
            const int32_t *sel = idx + r * nkb;
            for (int i = 0; i < ORC_BLOCK; ++i) {
                const int64_t tq = qb * ORC_BLOCK + i;
                double *o = out + (n * ORC_BLOCK + i) * d;
                double *nm = num ? num + (n * ORC_BLOCK + i) * d : NULL;
                if (tq >= N) {
                    for (int e = 0; e < d; ++e) o[e] = 0.0;
                    if (nm)
                        for (int e = 0; e < d; ++e) nm[e] = 0.0;
                    if (lse) lse[n * ORC_BLOCK + i] = 0.0;
                    if (den) den[n * ORC_BLOCK + i] = 0.0;
                    continue;
                }
                for (int e = 0; e < d; ++e) qv[e] = bf16_val(Q[(bh * N_pad + tq) * d + e]);
                /* logits of every valid key in the selected blocks, plus ln w_j */
                double m = -INFINITY;
                int64_t nl = 0;
                for (int32_t c = 0; c < nsel; ++c) {
                    const int64_t j = sel[c];
                    const double lw = w ? log((double)w[r * nkb + c]) : 0.0;
                    for (int t = 0; t < U; ++t) {
                        const int64_t tk = j * U + t;
                        if (tk >= N) break;
                        double dot = 0.0;
                        for (int e = 0; e < d; ++e)
                            dot += qv[e] * bf16_val(K[(bh * N_pad + tk) * d + e]);
                        logit[nl] = dot * scale + lw;
                        if (logit[nl] > m) m = logit[nl];
                        ++nl;
                    }
                }
                if (nl == 0) {
                    for (int e = 0; e < d; ++e) o[e] = 0.0;
                    if (nm)
                        for (int e = 0; e < d; ++e) nm[e] = 0.0;
                    if (lse) lse[n * ORC_BLOCK + i] = -INFINITY;
                    if (den) den[n * ORC_BLOCK + i] = 0.0;
                    continue;
                }
                double z = 0.0;
                for (int e = 0; e < d; ++e) acc[e] = 0.0;
                nl = 0;
                for (int32_t c = 0; c < nsel; ++c) {
                    const int64_t j = sel[c];
                    for (int t = 0; t < U; ++t) {
                        const int64_t tk = j * U + t;
                        if (tk >= N) break;
                        const double pexp = exp(logit[nl++] - m);
                        z += pexp;
                        for (int e = 0; e < d; ++e)
                            acc[e] += pexp * bf16_val(V[(bh * N_pad + tk) * d + e]);
                    }
                }
                for (int e = 0; e < d; ++e) o[e] = acc[e] / z;
                if (lse) lse[n * ORC_BLOCK + i] = m + log(z);
                if (nm) {
                    const double em = exp(m);
                    for (int e = 0; e < d; ++e) nm[e] = acc[e] * em;
                }
                if (den) den[n * ORC_BLOCK + i] = z * exp(m);
            }
        }
        free(logit);
        free(qv);
        free(acc);
    }
    return rc;
}

int orc_attn_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B, int H, int N,
                  int N_pad, int d, const int32_t *idx, const int32_t *cnt, const float *w,
                  int64_t n_rows, const int64_t *rows, double *out, double *lse, double *num,
                  double *den)
{
    return orc_attn_rows_u(Q, K, V, B, H, N, N_pad, d, ORC_BLOCK, idx, cnt, w, n_rows, rows, out,
                           lse, num, den);
}

/* ------------------------------------------------------------------------------
 * Dense softmax attention over all valid keys (the budget = all blocks case),
 * written independently of the block loop above: full row of N logits, softmax,
 * weighted sum. out [B,H,N_pad,d], lse [B,H,N_pad] (optional). Rows i >= N are 0.
 * ------------------------------------------------------------------------------ */
int orc_dense_attn(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int B, int H,
                   int N, int N_pad, int d, double *out, double *lse)
{
    if (!Q || !K || !V || !out || check_shape(B, H, N, N_pad, d)) return -1;
    const double scale = 1.0 / sqrt((double)d);
    const int64_t rows = (int64_t)B * H * N_pad;
    int rc = 0;
#pragma omp parallel
    {
        double *row = (double *)malloc(sizeof(double) * N);
        if (!row) {
#pragma omp atomic write
            rc = -2;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            if (rc) continue;
            const int64_t bh = r / N_pad, i = r % N_pad;
            double *o = out + r * d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            if (i >= N) {
                if (lse) lse[r] = 0.0;
                continue;
            }
            const uint16_t *q = Q + r * d;
            double m = -INFINITY;
            for (int64_t t = 0; t < N; ++t) {
                const uint16_t *kr = K + (bh * N_pad + t) * d;
                double dot = 0.0;
                for (int e = 0; e < d; ++e) dot += bf16_val(q[e]) * bf16_val(kr[e]);
                row[t] = dot * scale;
                if (row[t] > m) m = row[t];
            }
            double z = 0.0;
            for (int64_t t = 0; t < N; ++t) {
                row[t] = exp(row[t] - m);
                z += row[t];
            }
            for (int64_t t = 0; t < N; ++t) {
                const uint16_t *vr = V + (bh * N_pad + t) * d;
                const double pw = row[t] / z;
                for (int e = 0; e < d; ++e) o[e] += pw * bf16_val(vr[e]);
            }
            if (lse) lse[r] = m + log(z);
        }
        free(row);
    }
    return rc;
}

/* ------------------------------------------------------------------------------
 * Gradient of the block-sparse HT attention above (key blocks of 128 tokens) with
 * respect to Q, K and V, for an upstream gradient dO of the output. The weights and
 * the selection are constants (the selection is a sample, not a differentiable
 * function of Q or K). With the loss L = sum_i dO_i . O_i, per valid query row i of
 * query block qb and every valid key t of its kept blocks j:
 *   P_it  = w_j e^{q_i.k_t/sqrt(d)} / sum_{j',t'} w_j' e^{q_i.k_t'/sqrt(d)}  (O_i = sum_t P_it v_t)
 *   dV_t += P_it dO_i
 *   dP_it = dO_i . v_t,   D_i = dO_i . O_i = sum_t P_it dP_it
 *   dS_it = P_it (dP_it - D_i)          (derivative through the softmax)
 *   dQ_i += dS_it k_t / sqrt(d),   dK_t += dS_it q_i / sqrt(d)
 * Rows i >= N and rows with an empty selection contribute nothing and get dQ_i = 0;
 * keys t >= N get dK_t = dV_t = 0. dO is bf16 bits like Q, K, V; dQ, dK, dV are fp64
 * [B,H,N_pad,d]. w = NULL means all weights 1 (top-k). Work is split over the (b, h)
 * pairs, each pair's rows taken in order, so the sums over query rows into dK and dV
 * run in a fixed order.
 * ------------------------------------------------------------------------------ */
int orc_attn_bwd(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const uint16_t *dO,
                 int B, int H, int N, int N_pad, int d, const int32_t *idx, const int32_t *cnt,
                 const float *w, double *dQ, double *dK, double *dV)
{
    if (!Q || !K || !V || !dO || !idx || !cnt || !dQ || !dK || !dV ||
        check_shape(B, H, N, N_pad, d))
        return -1;
    const int64_t nb = n_blocks_of(N_pad);
    const int64_t BH = (int64_t)B * H;
    for (int64_t r = 0; r < BH * nb; ++r) {
        if (cnt[r] < 0 || cnt[r] > nb) return -1;
        for (int32_t c = 0; c < cnt[r]; ++c) {
            if (idx[r * nb + c] < 0 || idx[r * nb + c] >= nb) return -1;
            if (w && !(w[r * nb + c] > 0.0f && isfinite(w[r * nb + c]))) return -1;
        }
    }
    const int64_t total = BH * N_pad * d;
    for (int64_t e = 0; e < total; ++e) dQ[e] = dK[e] = dV[e] = 0.0;
    const double scale = 1.0 / sqrt((double)d);
    int rc = 0;
#pragma omp parallel
    {
        const int64_t max_keys = nb * ORC_BLOCK;
        double *pr = (double *)malloc(sizeof(double) * max_keys);
        int64_t *key = (int64_t *)malloc(sizeof(int64_t) * max_keys);
        double *qv = (double *)malloc(sizeof(double) * d);
        double *gv = (double *)malloc(sizeof(double) * d);
        double *ov = (double *)malloc(sizeof(double) * d);
        if (!pr || !key || !qv || !gv || !ov) {
#pragma omp atomic write
            rc = -2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < BH; ++bh) {
            if (rc) continue;
            const uint16_t *Qh = Q + bh * N_pad * d, *Kh = K + bh * N_pad * d;
            const uint16_t *Vh = V + bh * N_pad * d, *Gh = dO + bh * N_pad * d;
            double *dQh = dQ + bh * N_pad * d, *dKh = dK + bh * N_pad * d;
            double *dVh = dV + bh * N_pad * d;
            for (int64_t qb = 0; qb < nb; ++qb) {
                const int64_t r = bh * nb + qb;
                for (int i = 0; i < ORC_BLOCK; ++i) {
                    const int64_t tq = qb * ORC_BLOCK + i;
                    if (tq >= N) continue;
                    for (int e = 0; e < d; ++e) {
                        qv[e] = bf16_val(Qh[tq * d + e]);
                        gv[e] = bf16_val(Gh[tq * d + e]);
                    }
                    /* logits (with ln w_j) of the valid keys of the kept blocks */
                    int64_t nk = 0;
                    double m = -INFINITY;
                    for (int32_t c = 0; c < cnt[r]; ++c) {
                        const int64_t j = idx[r * nb + c];
                        const double lw = w ? log((double)w[r * nb + c]) : 0.0;
                        for (int t = 0; t < ORC_BLOCK; ++t) {
                            const int64_t tk = j * ORC_BLOCK + t;
                            if (tk >= N) break;
                            double dot = 0.0;
                            for (int e = 0; e < d; ++e) dot += qv[e] * bf16_val(Kh[tk * d + e]);
                            pr[nk] = dot * scale + lw;
                            key[nk] = tk;
                            if (pr[nk] > m) m = pr[nk];
                            ++nk;
                        }
                    }
                    if (nk == 0) continue;
                    /* softmax probabilities and the output row */
                    double z = 0.0;
                    for (int64_t a = 0; a < nk; ++a) {
                        pr[a] = exp(pr[a] - m);
                        z += pr[a];
                    }
                    for (int e = 0; e < d; ++e) ov[e] = 0.0;
                    for (int64_t a = 0; a < nk; ++a) {
                        pr[a] /= z;
                        for (int e = 0; e < d; ++e) ov[e] += pr[a] * bf16_val(Vh[key[a] * d + e]);
                    }
                    double Di = 0.0;
                    for (int e = 0; e < d; ++e) Di += gv[e] * ov[e];
                    /* gradients */
                    for (int64_t a = 0; a < nk; ++a) {
                        const int64_t tk = key[a];
                        double dp = 0.0;
                        for (int e = 0; e < d; ++e) dp += gv[e] * bf16_val(Vh[tk * d + e]);
                        const double ds = pr[a] * (dp - Di);
                        for (int e = 0; e < d; ++e) {
                            dVh[tk * d + e] += pr[a] * gv[e];
                            dQh[tq * d + e] += ds * bf16_val(Kh[tk * d + e]) * scale;
                            dKh[tk * d + e] += ds * qv[e] * scale;
                        }
                    }
                }
            }
        }
        free(pr);
        free(key);
        free(qv);
        free(gv);
        free(ov);
    }
    return rc;
}

/* Number of OpenMP threads the oracle runs with (reported beside its timings). */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
