/*
 * attn_oracle.c -- plain, slow, double-precision CPU oracle of multi-head
 * causal scaled dot-product self-attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this:
 * only the tests, the smoke check and the bench's CPU-baseline leg load it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes, per head (b, h), for rows i and columns j of [T, T]:
 *
 *   S_ij = scale * <q_i, k_j>              affinity = dot product of a token's
 *                                          query with the keys of the tokens
 *                                          up to it, divided by sqrt(head dim)
 *   S_ij = -inf for j > i                  upper triangle masked before the
 *                                          softmax: no look into the future
 *   P_i. = softmax(S_i.)                   row-normalised weights
 *   O_i  = sum_j P_ij v_j                  values aggregated by the weights
 *   lse_i = ln sum_{j<=i} exp(S_ij)        natural log, of the scaled scores
 *
 * Sources: "How Andrej Karpathy built GPT from 200 lines of code" (rdly.ru
 * summary of the "Let's build GPT" video), section "Self-Attention: the
 * mathematical trick" [43:56]-[55:20] (tril, row normalisation, -inf upper
 * triangle, softmax) and section "Implementing the attention heads (Query,
 * Key, Value)" [1:04:00]-[1:22:27] (query/key affinities, values, division by
 * the square root of the head size, heads in parallel).  Heads are independent
 * and dropout is 0 (nanoGPT skill card, Workflow 2 config: dropout = 0.0).
 *
 * The backward pass is the exact derivative of the forward for the loss
 * L = sum(O * dO); the pages do not spell it out, so it is the textbook
 * chain rule through O = P V and the row softmax:
 *
 *   dV_j  = sum_{i>=j} P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   Delta_i = <dO_i, O_i>              (= sum_j P_ij dP_ij)
 *   dS_ij = P_ij (dP_ij - Delta_i)
 *   dQ_i  = scale * sum_{j<=i} dS_ij k_j
 *   dK_j  = scale * sum_{i>=j} dS_ij q_i
 *
 * Non-causal variant (the "_nc" entry points): the same computation with no
 * mask, every query attending to all T keys -- the encoder-style attention the
 * pages contrast with the decoder's masked one when they introduce the -inf
 * upper triangle ([55:20]); the backward is the same derivative with sums over
 * all i and j.
 *
 * Attention dropout (the "_dropout" entry points): the pages give a model
 * dropout rate ("GPT da zero", table "Come funziona": 0.1; the nanoGPT skill
 * card's GPT-2 config: 0.0) but not where inside attention it acts.  Read
 * plainly, attention dropout zeroes attention weights after the softmax and
 * before they meet the values, scaling the kept weights so their expectation
 * is unchanged.  With a keep mask M_ij in {0, 1} and keep scale c:
 *
 *   Z_ij = c * M_ij * P_ij               dropped weights (lse, P unchanged)
 *   O_i  = sum_j Z_ij v_j
 *   dV_j = sum_i Z_ij dO_i
 *   dS_ij = P_ij (c * M_ij * <dO_i, v_j> - Delta_i),  Delta_i = <dO_i, O_i>
 *
 * The mask is the counter-based generator Philox4x32-10 (Salmon, Moraes, Dror
 * and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011): key =
 * (seed low word, seed high word), counter = (i, j / 8, b * H + h, offset);
 * the four 32-bit outputs give eight 16-bit values, value (j mod 8) = bits
 * 16 * (j mod 2) .. +15 of output word (j mod 8) / 2.  Element (i, j) is kept
 * iff that value is >= t, t = floor(p * 65536 + 1/2) for the drop probability
 * p, and c = 65536 / (65536 - t), so E[c M] = 1 exactly.
 *
 * Decode ("oracle_attn_decode"): generating text appends one token at a time
 * and each new token's query attends to every earlier token and itself
 * ("nanoGPT — 架构与原理", section 5 "边界与局限": generate recomputes the
 * whole forward for every new token, with no KV cache).  With the keys
 * and values of all Tk tokens kept, the Tq newest queries (positions
 * Tk - Tq .. Tk - 1) need only their own rows of the causal attention: query
 * r sees keys 0 .. Tk - Tq + r.
 *
 * Layout: every tensor is [B, H, T, D] contiguous float64; lse is [B, H, T].
 * No blocking, no fusion, no reordering beyond the definition.  The softmax
 * subtracts the row maximum before exponentiating, which changes nothing in
 * exact arithmetic and keeps exp() finite.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Row i of the softmax of one head over keys 0..last (last = i when causal,
 * T - 1 otherwise): fills p[0..last] (later entries untouched), returns lse_i.
 * q_i is one query row, kh the head's keys. */
static double softmax_row(const double *qi, const double *kh, int last, int D, double scale,
                          double *p)
{
    const int i = last;
    double m = -INFINITY;
    for (int j = 0; j <= i; ++j) {
        double s = 0.0;
        for (int d = 0; d < D; ++d) s += qi[d] * kh[(int64_t)j * D + d];
        s *= scale;
        p[j] = s;
        if (s > m) m = s;
    }
    double l = 0.0;
    for (int j = 0; j <= i; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    for (int j = 0; j <= i; ++j) p[j] /= l;
    return m + log(l);
}

/* ---- Philox4x32-10: ten rounds of the round function below, the key
 * bumped by the Weyl increments between rounds. */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u /* golden ratio - 1, times 2^32 */
#define PHILOX_W1 0xBB67AE85u /* sqrt(3) - 1, times 2^32 */

void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        const uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        const uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* The drop threshold t for probability p (see the header comment). */
static uint32_t drop_threshold(double p) { return (uint32_t)floor(p * 65536.0 + 0.5); }

/* Keep bit of element (i, j) of head bh. */
static int keep_bit(uint64_t seed, uint32_t offset, int64_t bh, int i, int j, uint32_t t)
{
    const uint32_t ctr[4] = {(uint32_t)i, (uint32_t)j >> 3, (uint32_t)bh, offset};
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t x[4];
    oracle_philox4x32_10(ctr, key, x);
    const uint32_t u = (x[(j & 7) >> 1] >> (16 * (j & 1))) & 0xFFFFu;
    return u >= t;
}

/* Dropout parameters of one call; p = 0 means no dropout.  head0 is the flat
 * head index (b * H + h) of the first head held by the tensors, so that a
 * subset of a larger problem's heads draws that problem's masks. */
typedef struct {
    double p;
    uint64_t seed;
    uint32_t offset;
    int64_t head0;
} dropout_t;

static const dropout_t no_dropout = {0.0, 0, 0, 0};

/* Keep scale c * M_ij of element (i, j) of head bh (1 when p = 0). */
static double keep_factor(const dropout_t *dr, int64_t bh, int i, int j)
{
    if (dr->p == 0.0) return 1.0;
    const uint32_t t = drop_threshold(dr->p);
    if (!keep_bit(dr->seed, dr->offset, dr->head0 + bh, i, j, t)) return 0.0;
    return 65536.0 / (65536.0 - (double)t);
}

/* The keep mask M [B,H,T,T] as bytes (1 = kept), over all (i, j). */
void oracle_dropout_mask(int B, int H, int T, double p, uint64_t seed, uint32_t offset,
                         uint8_t *mask)
{
    const uint32_t t = drop_threshold(p);
    const int64_t heads = (int64_t)B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh)
        for (int i = 0; i < T; ++i)
            for (int j = 0; j < T; ++j)
                mask[(bh * T + i) * (int64_t)T + j] = (uint8_t)keep_bit(seed, offset, bh, i, j, t);
}

static int num_threads_used = 1;

/* Number of OpenMP threads the last call ran on. */
int oracle_threads(void) { return num_threads_used; }

/* Last key row i attends to: itself when causal, the final token otherwise. */
static int last_key(int i, int T, int causal) { return causal ? i : T - 1; }

/* First query row that attends to key j: j itself when causal, else row 0. */
static int first_query(int j, int causal) { return causal ? j : 0; }

/* Forward: o [B,H,T,D], lse [B,H,T] (lse may be NULL). */
static void attn_fwd(const double *q, const double *k, const double *v,
                     double *o, double *lse, int B, int H, int T, int D, double scale,
                     int causal, const dropout_t *dr)
{
    const int64_t heads = (int64_t)B * H;
    const int64_t hs = (int64_t)T * D;
#pragma omp parallel
    {
#ifdef _OPENMP
#pragma omp single
        num_threads_used = omp_get_num_threads();
#endif
        double *p = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < heads; ++bh) {
            const double *qh = q + bh * hs, *kh = k + bh * hs, *vh = v + bh * hs;
            double *oh = o + bh * hs;
            for (int i = 0; i < T; ++i) {
                const int last = last_key(i, T, causal);
                double li = softmax_row(qh + (int64_t)i * D, kh, last, D, scale, p);
                if (lse) lse[bh * T + i] = li;
                for (int j = 0; j <= last; ++j) p[j] *= keep_factor(dr, bh, i, j);  /* Z_i. */
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j <= last; ++j) acc += p[j] * vh[(int64_t)j * D + d];
                    oh[(int64_t)i * D + d] = acc;
                }
            }
        }
        free(p);
    }
}

/* The full probability matrices P [B,H,T,T] (zeros above the diagonal when
 * causal). */
static void attn_probs(const double *q, const double *k, double *p,
                       int B, int H, int T, int D, double scale, int causal)
{
    const int64_t heads = (int64_t)B * H;
    const int64_t hs = (int64_t)T * D;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh) {
        double *ph = p + bh * (int64_t)T * T;
        memset(ph, 0, sizeof(double) * (size_t)T * (size_t)T);
        for (int i = 0; i < T; ++i)
            softmax_row(q + bh * hs + (int64_t)i * D, k + bh * hs, last_key(i, T, causal), D,
                        scale, ph + (int64_t)i * T);
    }
}

/* Backward: dq, dk, dv [B,H,T,D] from q, k, v and the upstream gradient dO.
 * The forward (P, O) is recomputed here from q, k, v in double. */
static void attn_bwd(const double *q, const double *k, const double *v, const double *dO,
                     double *dq, double *dk, double *dv,
                     int B, int H, int T, int D, double scale, int causal, const dropout_t *dr)
{
    const int64_t heads = (int64_t)B * H;
    const int64_t hs = (int64_t)T * D;
#pragma omp parallel
    {
#ifdef _OPENMP
#pragma omp single
        num_threads_used = omp_get_num_threads();
#endif
        const size_t tt = (size_t)(T > 0 ? T : 1) * (size_t)(T > 0 ? T : 1);
        double *P = (double *)malloc(sizeof(double) * tt);    /* P_ij  */
        double *dS = (double *)malloc(sizeof(double) * tt);   /* dS_ij */
        double *Z = (double *)malloc(sizeof(double) * tt);    /* Z_ij = c M_ij P_ij */
        double *O = (double *)malloc(sizeof(double) * (size_t)(hs > 0 ? hs : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < heads; ++bh) {
            const double *qh = q + bh * hs, *kh = k + bh * hs, *vh = v + bh * hs;
            const double *gh = dO + bh * hs;
            double *dqh = dq + bh * hs, *dkh = dk + bh * hs, *dvh = dv + bh * hs;
            memset(P, 0, sizeof(double) * tt);
            memset(dS, 0, sizeof(double) * tt);
            memset(Z, 0, sizeof(double) * tt);
            /* forward recompute: P, Z and O */
            for (int i = 0; i < T; ++i) {
                const int last = last_key(i, T, causal);
                softmax_row(qh + (int64_t)i * D, kh, last, D, scale, P + (int64_t)i * T);
                for (int j = 0; j <= last; ++j)
                    Z[(int64_t)i * T + j] = keep_factor(dr, bh, i, j) * P[(int64_t)i * T + j];
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j <= last; ++j) acc += Z[(int64_t)i * T + j] * vh[(int64_t)j * D + d];
                    O[(int64_t)i * D + d] = acc;
                }
            }
            /* dV_j = sum_{i>=j} Z_ij dO_i (all i when not causal) */
            for (int j = 0; j < T; ++j)
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int i = first_query(j, causal); i < T; ++i) acc += Z[(int64_t)i * T + j] * gh[(int64_t)i * D + d];
                    dvh[(int64_t)j * D + d] = acc;
                }
            /* dS_ij = P_ij (c M_ij dP_ij - Delta_i), dP_ij = <dO_i, v_j>, Delta_i = <dO_i, O_i> */
            for (int i = 0; i < T; ++i) {
                double delta = 0.0;
                for (int d = 0; d < D; ++d) delta += gh[(int64_t)i * D + d] * O[(int64_t)i * D + d];
                for (int j = 0; j <= last_key(i, T, causal); ++j) {
                    double dp = 0.0;
                    for (int d = 0; d < D; ++d) dp += gh[(int64_t)i * D + d] * vh[(int64_t)j * D + d];
                    dS[(int64_t)i * T + j] = P[(int64_t)i * T + j] * (keep_factor(dr, bh, i, j) * dp - delta);
                }
            }
            /* dQ_i = scale * sum_{j<=i} dS_ij k_j (all j when not causal) */
            for (int i = 0; i < T; ++i)
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j <= last_key(i, T, causal); ++j) acc += dS[(int64_t)i * T + j] * kh[(int64_t)j * D + d];
                    dqh[(int64_t)i * D + d] = scale * acc;
                }
            /* dK_j = scale * sum_{i>=j} dS_ij q_i (all i when not causal) */
            for (int j = 0; j < T; ++j)
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int i = first_query(j, causal); i < T; ++i) acc += dS[(int64_t)i * T + j] * qh[(int64_t)i * D + d];
                    dkh[(int64_t)j * D + d] = scale * acc;
                }
        }
        free(P);
        free(dS);
        free(Z);
        free(O);
    }
}

/* Exported entry points: the causal attention of the decoder, and the same
 * computation without the mask ("_nc"). */
void oracle_attn_fwd(const double *q, const double *k, const double *v, double *o, double *lse,
                     int B, int H, int T, int D, double scale)
{
    attn_fwd(q, k, v, o, lse, B, H, T, D, scale, 1, &no_dropout);
}

void oracle_attn_fwd_nc(const double *q, const double *k, const double *v, double *o,
                        double *lse, int B, int H, int T, int D, double scale)
{
    attn_fwd(q, k, v, o, lse, B, H, T, D, scale, 0, &no_dropout);
}

void oracle_attn_probs(const double *q, const double *k, double *p, int B, int H, int T, int D,
                       double scale)
{
    attn_probs(q, k, p, B, H, T, D, scale, 1);
}

void oracle_attn_probs_nc(const double *q, const double *k, double *p, int B, int H, int T,
                          int D, double scale)
{
    attn_probs(q, k, p, B, H, T, D, scale, 0);
}

void oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dO,
                     double *dq, double *dk, double *dv, int B, int H, int T, int D, double scale)
{
    attn_bwd(q, k, v, dO, dq, dk, dv, B, H, T, D, scale, 1, &no_dropout);
}

void oracle_attn_bwd_nc(const double *q, const double *k, const double *v, const double *dO,
                        double *dq, double *dk, double *dv, int B, int H, int T, int D,
                        double scale)
{
    attn_bwd(q, k, v, dO, dq, dk, dv, B, H, T, D, scale, 0, &no_dropout);
}

/* Attention with dropout on the weights (either mask): p in [0, 1), the
 * generator's seed and counter offset as in the header comment. */
void oracle_attn_fwd_dropout(const double *q, const double *k, const double *v, double *o,
                             double *lse, int B, int H, int T, int D, double scale, int causal,
                             double p, uint64_t seed, uint32_t offset, int64_t head0)
{
    const dropout_t dr = {p, seed, offset, head0};
    attn_fwd(q, k, v, o, lse, B, H, T, D, scale, causal, &dr);
}

void oracle_attn_bwd_dropout(const double *q, const double *k, const double *v,
                             const double *dO, double *dq, double *dk, double *dv, int B, int H,
                             int T, int D, double scale, int causal, double p, uint64_t seed,
                             uint32_t offset, int64_t head0)
{
    const dropout_t dr = {p, seed, offset, head0};
    attn_bwd(q, k, v, dO, dq, dk, dv, B, H, T, D, scale, causal, &dr);
}

/* Decode: q, o [B,H,Tq,D], k, v [B,H,Tk,D], lse [B,H,Tq] (may be NULL);
 * query r is the token at position Tk - Tq + r and sees keys 0 .. Tk - Tq + r. */
void oracle_attn_decode(const double *q, const double *k, const double *v, double *o,
                        double *lse, int B, int H, int Tq, int Tk, int D, double scale)
{
    const int64_t heads = (int64_t)B * H;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)(Tk > 0 ? Tk : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < heads; ++bh) {
            const double *kh = k + bh * (int64_t)Tk * D, *vh = v + bh * (int64_t)Tk * D;
            for (int r = 0; r < Tq; ++r) {
                const int last = Tk - Tq + r;
                const double *qr = q + (bh * Tq + r) * (int64_t)D;
                double li = softmax_row(qr, kh, last, D, scale, p);
                if (lse) lse[bh * Tq + r] = li;
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int j = 0; j <= last; ++j) acc += p[j] * vh[(int64_t)j * D + d];
                    o[(bh * Tq + r) * (int64_t)D + d] = acc;
                }
            }
        }
        free(p);
    }
}
