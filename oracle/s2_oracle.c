/*
 * s2_oracle.c -- plain fp64 CPU oracle for HHST sparse attention.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg load this file's library. The CUDA library never
 * calls it, and the two share no code, header, table or helper: this file
 * includes nothing but the C standard library and pthreads.
 *
 * What it computes. "S2-Attention: Hardware-aware context sharding among
 * attention heads" (OpenReview forum page, Abstract; arXiv 2407.17678 abstract)
 * describes HHST only in words: attention is sparse, the pattern can differ per
 * head, each head attends to a different strided subset of the context while
 * the heads together cover all of it, and sparse heads can be mixed with dense
 * ones ("hybrid"). The pages give no formula, so the oracle uses this explicit
 * block rule, with query block i = q / B and key block j = k / B:
 *
 *     active(h, i, j) = j <= i and (dense[h] or i - j < L or (j + h) mod S == 0)
 *
 * and causality inside the diagonal block (key k visible to query q iff k <= q).
 * The method reaches exactly (up to rounding order) masked softmax attention, so
 * the oracle is that definition written out in fp64, on inputs given as bf16
 * bit patterns (widened exactly to double):
 *
 *     s_k  = scale * sum_d Q[q,d] K[k,d]            for every visible key k
 *     m    = max_k s_k,  den = sum_k exp(s_k - m)
 *     O[q] = sum_k exp(s_k - m) / den * V[k]
 *     LSE  = m + log(den)
 *
 * Decode is the same definition for one query at position n-1 of a context of
 * n tokens whose keys and values sit in a paged cache addressed through a block
 * table (PagedAttention is in the arXiv page's reference list).
 *
 * Two generalisations follow the same definition with another block rule.
 * (1) Per-context-range patterns: the arXiv abstract says the patterns can be
 * customised per head and per context range. Here a head's key-block axis is
 * cut into consecutive ranges, each with its own (S, L, dense), and key block j
 * takes the parameters of the range that holds it (s2o_range_block_active).
 * (2) Any per-head block mask, given as [H][nb][nb] bytes (the *_mask entry
 * points), with the same token-level causality inside the diagonal block.
 * The *_mask entry points also take a number of key/value heads Hkv dividing H:
 * query head h reads key/value head h / (H / Hkv) (grouped-query attention; the
 * pages do not mention it; Hkv = H is plain multi-head attention).
 * A query that sees no key at all (possible only under a given mask) gets a
 * zero output row and LSE = -inf: the softmax over an empty set is undefined,
 * and zero is the value whose weight in any later merge is nil.
 *
 * Backward. The arXiv abstract reports training speedups, so the gradients of
 * the same definition are part of the method. With an upstream gradient dO,
 * P[q,k] = exp(s_qk - LSE_q) over the visible keys of row q, and
 *
 *     dV[k]  = sum_q P[q,k] dO[q]
 *     dP[q,k] = dO[q] . V[k]
 *     Dq     = sum_k P[q,k] dP[q,k]
 *     dS[q,k] = P[q,k] (dP[q,k] - Dq)
 *     dQ[q]  = scale * sum_k dS[q,k] K[k]
 *     dK[k]  = scale * sum_q dS[q,k] Q[q]
 *
 * (the chain rule through the softmax and the scaled dot products; with
 * grouped K/V heads, dK and dV of a K/V head sum over its query heads).
 *
 * Every loop visits keys in ascending order; nothing is blocked, fused or
 * reordered beyond the definition.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* bf16 bit pattern -> double: the bf16 value is the top half of an fp32. */
static double bf16_bits_to_double(uint16_t u)
{
    uint32_t bits = ((uint32_t)u) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* The block rule above. Returns 1 when key block j is visible to query block i
 * of head h, 0 otherwise (including j > i and negative indices). */
int s2o_block_active(int64_t h, int64_t i, int64_t j, int64_t S, int64_t L, int dense)
{
    if (j < 0 || i < 0 || j > i) return 0;
    if (dense) return 1;
    if (i - j < L) return 1;
    return ((j + h) % S) == 0;
}

/* Full block mask, mask[(h * nb + i) * nb + j] in {0,1}. dense may be NULL. */
void s2o_block_mask(int64_t H, int64_t nb, int64_t S, int64_t L,
                    const uint8_t* dense, uint8_t* mask)
{
    for (int64_t h = 0; h < H; ++h)
        for (int64_t i = 0; i < nb; ++i)
            for (int64_t j = 0; j < nb; ++j)
                mask[(h * nb + i) * nb + j] =
                    (uint8_t)s2o_block_active(h, i, j, S, L, dense ? dense[h] != 0 : 0);
}

/* Per-context-range rule for one head. The head's ranges r = 0..nr-1 cover key
 * blocks [end[r-1], end[r]) (end[-1] = 0), ends strictly ascending. Key block j
 * uses the parameters of its range: visible iff j <= i and (dense[r] or
 * i - j < L[r] or (S[r] > 0 and (j + h) mod S[r] == 0)). S[r] = 0 means the
 * range has no strided blocks. Blocks past the last range are not visible. */
int s2o_range_block_active(int64_t h, int64_t i, int64_t j, int64_t nr, const int64_t* end,
                           const int64_t* S, const int64_t* L, const uint8_t* dense)
{
    if (j < 0 || i < 0 || j > i) return 0;
    for (int64_t r = 0; r < nr; ++r) {
        if (j >= end[r]) continue;
        if (dense[r]) return 1;
        if (i - j < L[r]) return 1;
        return S[r] > 0 && ((j + h) % S[r]) == 0;
    }
    return 0;
}

/* Block mask [H][nb][nb] of per-head context ranges: head h owns ranges
 * range_ptr[h] .. range_ptr[h+1]-1 of the flat arrays end/S/L/dense. */
void s2o_range_block_mask(int64_t H, int64_t nb, const int64_t* range_ptr, const int64_t* end,
                          const int64_t* S, const int64_t* L, const uint8_t* dense,
                          uint8_t* mask)
{
    for (int64_t h = 0; h < H; ++h) {
        const int64_t r0 = range_ptr[h], nr = range_ptr[h + 1] - r0;
        for (int64_t i = 0; i < nb; ++i)
            for (int64_t j = 0; j < nb; ++j)
                mask[(h * nb + i) * nb + j] = (uint8_t)s2o_range_block_active(
                    h, i, j, nr, end + r0, S + r0, L + r0, dense + r0);
    }
}

/* ------------------------------------------------------------------------- */
/* Work distribution: a pool of pthreads pulls item indices from a counter.   */
/* ------------------------------------------------------------------------- */

typedef struct {
    int kind; /* 0 = prefill rows, 1 = decode items, 2 = backward planes, 3 = chunk rows,
                 4 = row statistics of sampled planes, 5 = sampled gradient rows */
    const uint16_t *q, *k, *v, *dout;
    double *dq, *dk, *dv; /* backward outputs */
    const int32_t *block_table, *ctx_lens, *q_start;
    int64_t batch, H, seq, D, B, S, L, page_size, max_pages;
    const uint8_t* dense;
    const uint8_t* bmask; /* NULL: the block rule above; else [H][nbm][nbm] */
    int64_t nbm, Hkv;     /* mask side; key/value heads (query head h reads h / (H / Hkv)) */
    double scale;
    int64_t n_items;
    const int64_t* items;
    double *out, *lse;
    /* sampled backward: K/V planes b * Hkv + g, query rows hh * seq + q of the
     * group's heads, key positions; row statistics from q_lo on */
    int64_t n_planes, nq, nk, q_lo;
    const int64_t *planes, *qrows, *krows;
    double *st_lse, *st_D;
    int64_t next;
    int failed;
    pthread_mutex_t lock;
} job_t;

static int64_t take(job_t* J)
{
    pthread_mutex_lock(&J->lock);
    int64_t r = J->next++;
    pthread_mutex_unlock(&J->lock);
    return r;
}

/* Is key block j visible to query block i of head h under this job's rule? */
static int visible(const job_t* J, int64_t h, int64_t i, int64_t j, int dense)
{
    if (J->bmask) return j <= i && j < J->nbm && i < J->nbm && J->bmask[(h * J->nbm + i) * J->nbm + j] != 0;
    return s2o_block_active(h, i, j, J->S, J->L, dense);
}

/* Prefill row r = (b * H + h) * seq + q: keys 0..q of the same batch entry, read
 * from key/value head h / (H / Hkv). */
static void prefill_row(const job_t* J, int64_t r, double* s, double* qd,
                        double* out, double* lse)
{
    const int64_t D = J->D, seq = J->seq;
    const int64_t q = r % seq;
    const int64_t bh = r / seq;
    const int64_t h = bh % J->H;
    const int64_t i = q / J->B;
    const int dense = J->dense ? J->dense[h] != 0 : 0;
    const int64_t kvh = (bh / J->H) * J->Hkv + h / (J->H / J->Hkv);
    const uint16_t* Q = J->q + r * D;
    const uint16_t* K = J->k + kvh * seq * D;
    const uint16_t* V = J->v + kvh * seq * D;

    for (int64_t d = 0; d < D; ++d) qd[d] = bf16_bits_to_double(Q[d]);

    double m = -INFINITY;
    for (int64_t k = 0; k <= q; ++k) {
        if (!visible(J, h, i, k / J->B, dense)) continue;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qd[d] * bf16_bits_to_double(K[k * D + d]);
        s[k] = J->scale * dot;
        if (s[k] > m) m = s[k];
    }
    double den = 0.0;
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    for (int64_t k = 0; k <= q; ++k) {
        if (!visible(J, h, i, k / J->B, dense)) continue;
        const double p = exp(s[k] - m);
        den += p;
        for (int64_t d = 0; d < D; ++d) out[d] += p * bf16_bits_to_double(V[k * D + d]);
    }
    if (den == 0.0) { /* no visible key */
        *lse = -INFINITY;
        return;
    }
    for (int64_t d = 0; d < D; ++d) out[d] /= den;
    *lse = m + log(den);
}

/* One query of sequence sq and head h at position pos of a paged context:
 * keys 0..pos, token t being row t % page_size of page block_table[sq][t /
 * page_size] in a [pages][Hkv][page_size][D] cache, key/value head
 * h / (H / Hkv). Q points at the query's D bf16 values. */
static int paged_row(const job_t* J, int64_t sq, int64_t h, int64_t pos, const uint16_t* Q,
                     double* s, double* qd, double* out, double* lse)
{
    const int64_t D = J->D, H = J->H, P = J->page_size;
    const int64_t i = pos / J->B;
    const int dense = J->dense ? J->dense[h] != 0 : 0;
    const int64_t Hkv = J->Hkv, kvh = h / (H / Hkv);

    for (int64_t d = 0; d < D; ++d) qd[d] = bf16_bits_to_double(Q[d]);

    double m = -INFINITY;
    for (int64_t k = 0; k <= pos; ++k) {
        if (!visible(J, h, i, k / J->B, dense)) continue;
        const int64_t page = J->block_table[sq * J->max_pages + k / P];
        if (page < 0) return -1;
        const uint16_t* Krow = J->k + ((page * Hkv + kvh) * P + k % P) * D;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qd[d] * bf16_bits_to_double(Krow[d]);
        s[k] = J->scale * dot;
        if (s[k] > m) m = s[k];
    }
    double den = 0.0;
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    for (int64_t k = 0; k <= pos; ++k) {
        if (!visible(J, h, i, k / J->B, dense)) continue;
        const int64_t page = J->block_table[sq * J->max_pages + k / P];
        const uint16_t* Vrow = J->v + ((page * Hkv + kvh) * P + k % P) * D;
        const double p = exp(s[k] - m);
        den += p;
        for (int64_t d = 0; d < D; ++d) out[d] += p * bf16_bits_to_double(Vrow[d]);
    }
    if (den == 0.0) { /* no visible key */
        *lse = -INFINITY;
        return 0;
    }
    for (int64_t d = 0; d < D; ++d) out[d] /= den;
    *lse = m + log(den);
    return 0;
}

/* Decode item e = seq_index * H + h: the query of sequence s sits at position
 * n-1 (n = ctx_lens[s]) and sees keys 0..n-1 of its paged context. */
static int decode_item(const job_t* J, int64_t e, double* s, double* qd,
                       double* out, double* lse)
{
    const int64_t sq = e / J->H, h = e % J->H;
    const int64_t n = J->ctx_lens[sq];
    if (n < 1) return -1;
    return paged_row(J, sq, h, n - 1, J->q + e * J->D, s, qd, out, lse);
}

/* Chunk item e = t * H + h, t a row of the packed chunk queries: sequence sq
 * holds rows q_start[sq] .. q_start[sq+1]-1, its last chunk of a context of
 * n = ctx_lens[sq] tokens, so row t sits at position n - (q_start[sq+1] - t). */
static int chunk_item(const job_t* J, int64_t e, double* s, double* qd, double* out,
                      double* lse)
{
    const int64_t t = e / J->H, h = e % J->H;
    int64_t sq = 0;
    while (sq + 1 < J->batch && J->q_start[sq + 1] <= t) ++sq;
    const int64_t n = J->ctx_lens[sq];
    const int64_t pos = n - (J->q_start[sq + 1] - t);
    if (pos < 0 || pos >= n) return -1;
    return paged_row(J, sq, h, pos, J->q + e * J->D, s, qd, out, lse);
}

/* Backward item e = b * Hkv + g: every query head h of K/V head g (h / (H / Hkv)
 * == g) and every row of batch entry b. dQ rows of those heads and the dK, dV
 * rows of plane e are written by this item alone. */
static void backward_plane(const job_t* J, int64_t e, double* s, double* p, double* qd,
                           double* dod)
{
    const int64_t D = J->D, seq = J->seq, H = J->H, Hkv = J->Hkv, grp = H / Hkv;
    const int64_t b = e / Hkv, g = e % Hkv;
    const uint16_t* K = J->k + e * seq * D;
    const uint16_t* V = J->v + e * seq * D;
    double* dK = J->dk + e * seq * D;
    double* dV = J->dv + e * seq * D;
    for (int64_t t = 0; t < seq * D; ++t) dK[t] = dV[t] = 0.0;
    for (int64_t h = g * grp; h < (g + 1) * grp; ++h) {
        const int dense = J->dense ? J->dense[h] != 0 : 0;
        const int64_t plane = b * H + h;
        for (int64_t q = 0; q < seq; ++q) {
            const int64_t i = q / J->B;
            const uint16_t* Q = J->q + (plane * seq + q) * D;
            const uint16_t* dO = J->dout + (plane * seq + q) * D;
            double* dQ = J->dq + (plane * seq + q) * D;
            for (int64_t d = 0; d < D; ++d) {
                qd[d] = bf16_bits_to_double(Q[d]);
                dod[d] = bf16_bits_to_double(dO[d]);
                dQ[d] = 0.0;
            }
            /* forward softmax of row q */
            double m = -INFINITY;
            for (int64_t k = 0; k <= q; ++k) {
                if (!visible(J, h, i, k / J->B, dense)) continue;
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d) dot += qd[d] * bf16_bits_to_double(K[k * D + d]);
                s[k] = J->scale * dot;
                if (s[k] > m) m = s[k];
            }
            if (m == -INFINITY) continue; /* no visible key: no gradient */
            double den = 0.0;
            for (int64_t k = 0; k <= q; ++k)
                if (visible(J, h, i, k / J->B, dense)) den += exp(s[k] - m);
            const double lse = m + log(den);
            /* P, dP and Dq */
            double Dq = 0.0;
            for (int64_t k = 0; k <= q; ++k) {
                if (!visible(J, h, i, k / J->B, dense)) continue;
                const double pk = exp(s[k] - lse);
                double dpk = 0.0;
                for (int64_t d = 0; d < D; ++d) dpk += dod[d] * bf16_bits_to_double(V[k * D + d]);
                p[k] = pk;
                s[k] = dpk; /* s now holds dP */
                Dq += pk * dpk;
            }
            /* dS, then the three products */
            for (int64_t k = 0; k <= q; ++k) {
                if (!visible(J, h, i, k / J->B, dense)) continue;
                const double ds = p[k] * (s[k] - Dq);
                for (int64_t d = 0; d < D; ++d) {
                    dV[k * D + d] += p[k] * dod[d];
                    dQ[d] += J->scale * ds * bf16_bits_to_double(K[k * D + d]);
                    dK[k * D + d] += J->scale * ds * qd[d];
                }
            }
        }
    }
}

/* Sampled backward, pass 1. Item t names (sampled plane p, query head hh of
 * its group, row q >= q_lo). The row's statistics by their definitions:
 * LSE = log sum_k exp(s_k) and D = sum_k P_k dP_k over the visible keys, with
 * s_k = scale Q.K_k, P_k = exp(s_k - LSE) and dP_k = dO.V_k. A row with no
 * visible key gets LSE = -inf and D = 0. */
static void row_stats(const job_t* J, int64_t t, double* s, double* qd, double* dod)
{
    const int64_t D = J->D, seq = J->seq, H = J->H, grp = H / J->Hkv, per = seq - J->q_lo;
    const int64_t p = t / (grp * per), hh = (t / per) % grp, q = J->q_lo + t % per;
    const int64_t e = J->planes[p], b = e / J->Hkv, h = (e % J->Hkv) * grp + hh;
    const int dense = J->dense ? J->dense[h] != 0 : 0;
    const int64_t i = q / J->B;
    const uint16_t* K = J->k + e * seq * D;
    const uint16_t* V = J->v + e * seq * D;
    const uint16_t* Q = J->q + ((b * H + h) * seq + q) * D;
    const uint16_t* dO = J->dout + ((b * H + h) * seq + q) * D;
    double* lse = J->st_lse + (p * grp + hh) * seq + q;
    double* Dq = J->st_D + (p * grp + hh) * seq + q;
    for (int64_t d = 0; d < D; ++d) {
        qd[d] = bf16_bits_to_double(Q[d]);
        dod[d] = bf16_bits_to_double(dO[d]);
    }
    double m = -INFINITY;
    for (int64_t k = 0; k <= q; ++k) {
        if (!visible(J, h, i, k / J->B, dense)) continue;
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qd[d] * bf16_bits_to_double(K[k * D + d]);
        s[k] = J->scale * dot;
        if (s[k] > m) m = s[k];
    }
    if (m == -INFINITY) {
        *lse = -INFINITY;
        *Dq = 0.0;
        return;
    }
    double den = 0.0;
    for (int64_t k = 0; k <= q; ++k)
        if (visible(J, h, i, k / J->B, dense)) den += exp(s[k] - m);
    *lse = m + log(den);
    double acc = 0.0;
    for (int64_t k = 0; k <= q; ++k) {
        if (!visible(J, h, i, k / J->B, dense)) continue;
        double dpk = 0.0;
        for (int64_t d = 0; d < D; ++d) dpk += dod[d] * bf16_bits_to_double(V[k * D + d]);
        acc += exp(s[k] - *lse) * dpk;
    }
    *Dq = acc;
}

/* Sampled backward, pass 2. Item t names (sampled plane p, entry r): for
 * r < nq the dQ row of query row qrows[r] (head hh = qrows[r] / seq of the
 * group), dQ = scale sum_k dS_k K_k; otherwise the dK and dV rows of key
 * position krows[r - nq], summed over the group's query heads and the rows
 * q >= k that see it: dV = sum_q P dO_q, dK = scale sum_q dS Q_q, with
 * dS = P (dP - D_q). */
static void sampled_grad(const job_t* J, int64_t t, double* qd, double* dod)
{
    const int64_t D = J->D, seq = J->seq, H = J->H, grp = H / J->Hkv, n = J->nq + J->nk;
    const int64_t p = t / n, r = t % n;
    const int64_t e = J->planes[p], b = e / J->Hkv, g = e % J->Hkv;
    const uint16_t* K = J->k + e * seq * D;
    const uint16_t* V = J->v + e * seq * D;
    if (r < J->nq) {
        const int64_t hh = J->qrows[r] / seq, q = J->qrows[r] % seq, h = g * grp + hh;
        const int dense = J->dense ? J->dense[h] != 0 : 0;
        const int64_t i = q / J->B;
        const uint16_t* Q = J->q + ((b * H + h) * seq + q) * D;
        const uint16_t* dO = J->dout + ((b * H + h) * seq + q) * D;
        const double lse = J->st_lse[(p * grp + hh) * seq + q];
        const double Dq = J->st_D[(p * grp + hh) * seq + q];
        double* dQ = J->dq + (p * J->nq + r) * D;
        for (int64_t d = 0; d < D; ++d) {
            qd[d] = bf16_bits_to_double(Q[d]);
            dod[d] = bf16_bits_to_double(dO[d]);
            dQ[d] = 0.0;
        }
        if (lse == -INFINITY) return; /* no visible key: no gradient */
        for (int64_t k = 0; k <= q; ++k) {
            if (!visible(J, h, i, k / J->B, dense)) continue;
            double dot = 0.0, dpk = 0.0;
            for (int64_t d = 0; d < D; ++d) {
                dot += qd[d] * bf16_bits_to_double(K[k * D + d]);
                dpk += dod[d] * bf16_bits_to_double(V[k * D + d]);
            }
            const double pk = exp(J->scale * dot - lse);
            const double ds = pk * (dpk - Dq);
            for (int64_t d = 0; d < D; ++d) dQ[d] += J->scale * ds * bf16_bits_to_double(K[k * D + d]);
        }
        return;
    }
    const int64_t kpos = J->krows[r - J->nq], j = kpos / J->B;
    double* dK = J->dk + (p * J->nk + r - J->nq) * D;
    double* dV = J->dv + (p * J->nk + r - J->nq) * D;
    double* kd = qd; /* K and V of the key row */
    double* vd = dod;
    for (int64_t d = 0; d < D; ++d) {
        kd[d] = bf16_bits_to_double(K[kpos * D + d]);
        vd[d] = bf16_bits_to_double(V[kpos * D + d]);
        dK[d] = dV[d] = 0.0;
    }
    for (int64_t hh = 0; hh < grp; ++hh) {
        const int64_t h = g * grp + hh;
        const int dense = J->dense ? J->dense[h] != 0 : 0;
        for (int64_t q = kpos; q < seq; ++q) {
            if (!visible(J, h, q / J->B, j, dense)) continue;
            const uint16_t* Q = J->q + ((b * H + h) * seq + q) * D;
            const uint16_t* dO = J->dout + ((b * H + h) * seq + q) * D;
            const double lse = J->st_lse[(p * grp + hh) * seq + q];
            const double Dq = J->st_D[(p * grp + hh) * seq + q];
            double dot = 0.0, dpk = 0.0;
            for (int64_t d = 0; d < D; ++d) {
                dot += bf16_bits_to_double(Q[d]) * kd[d];
                dpk += bf16_bits_to_double(dO[d]) * vd[d];
            }
            const double pk = exp(J->scale * dot - lse);
            const double ds = pk * (dpk - Dq);
            for (int64_t d = 0; d < D; ++d) {
                dV[d] += pk * bf16_bits_to_double(dO[d]);
                dK[d] += J->scale * ds * bf16_bits_to_double(Q[d]);
            }
        }
    }
}

static void* worker(void* arg)
{
    job_t* J = (job_t*)arg;
    const int64_t span = (J->kind == 1 || J->kind == 3) ? J->max_pages * J->page_size : J->seq;
    double* s = (double*)malloc(sizeof(double) * (size_t)(span > 0 ? span : 1));
    double* p = (double*)malloc(sizeof(double) * (size_t)(span > 0 ? span : 1));
    double* qd = (double*)malloc(sizeof(double) * (size_t)J->D);
    double* dod = (double*)malloc(sizeof(double) * (size_t)J->D);
    if (!s || !p || !qd || !dod) {
        pthread_mutex_lock(&J->lock);
        J->failed = 1;
        pthread_mutex_unlock(&J->lock);
        free(s);
        free(p);
        free(qd);
        free(dod);
        return NULL;
    }
    for (;;) {
        const int64_t t = take(J);
        if (t >= J->n_items) break;
        const int64_t id = J->items ? J->items[t] : t;
        if (J->kind == 2) {
            backward_plane(J, id, s, p, qd, dod);
            continue;
        }
        if (J->kind == 4) {
            row_stats(J, id, s, qd, dod);
            continue;
        }
        if (J->kind == 5) {
            sampled_grad(J, id, qd, dod);
            continue;
        }
        double* out = J->out + t * J->D;
        double* lse = J->lse + t;
        if (J->kind == 0) {
            prefill_row(J, id, s, qd, out, lse);
        } else if ((J->kind == 1 ? decode_item(J, id, s, qd, out, lse)
                                 : chunk_item(J, id, s, qd, out, lse)) != 0) {
            pthread_mutex_lock(&J->lock);
            J->failed = 1;
            pthread_mutex_unlock(&J->lock);
        }
    }
    free(s);
    free(p);
    free(qd);
    free(dod);
    return NULL;
}

static int run_job(job_t* J, int nthreads)
{
    if (nthreads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = n > 0 ? (int)n : 1;
    }
    if (nthreads > 1024) nthreads = 1024;
    pthread_mutex_init(&J->lock, NULL);
    J->next = 0;
    J->failed = 0;
    pthread_t tid[1024];
    int started = 0;
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&tid[started], NULL, worker, J) == 0) ++started;
    worker(J);
    for (int t = 0; t < started; ++t) pthread_join(tid[t], NULL);
    pthread_mutex_destroy(&J->lock);
    return J->failed ? -1 : 0;
}

/* Number of threads a call with nthreads <= 0 uses. */
int s2o_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Prefill oracle on selected rows.
 * q, k, v: bf16 bits, [batch][H][seq][D] contiguous.
 * rows: n_rows linear row ids (b * H + h) * seq + q, or NULL for all rows in
 *       order (then n_rows must be batch * H * seq).
 * out: [n_rows][D] fp64, lse: [n_rows] fp64. dense: [H] or NULL.
 * Returns 0, or -1 on a bad argument / allocation failure. */
int s2o_prefill_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                     int64_t batch, int64_t H, int64_t seq, int64_t D,
                     int64_t B, int64_t S, int64_t L, const uint8_t* dense,
                     double scale, int64_t n_rows, const int64_t* rows,
                     double* out, double* lse, int nthreads)
{
    if (!q || !k || !v || !out || !lse || batch < 1 || H < 1 || seq < 1 || D < 1 ||
        B < 1 || S < 1 || L < 1 || n_rows < 0)
        return -1;
    if (!rows && n_rows != batch * H * seq) return -1;
    if (rows)
        for (int64_t t = 0; t < n_rows; ++t)
            if (rows[t] < 0 || rows[t] >= batch * H * seq) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 0;
    J.q = q; J.k = k; J.v = v;
    J.batch = batch; J.H = H; J.seq = seq; J.D = D;
    J.B = B; J.S = S; J.L = L; J.dense = dense; J.scale = scale; J.Hkv = H;
    J.n_items = n_rows; J.items = rows; J.out = out; J.lse = lse;
    return run_job(&J, nthreads);
}

/* Prefill oracle under a given block mask [H][nbm][nbm] (nbm >= ceil(seq / B);
 * entries with j > i are ignored) and Hkv key/value heads: k, v are
 * [batch][Hkv][seq][D]. Other arguments as s2o_prefill_rows. */
int s2o_prefill_rows_mask(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          int64_t batch, int64_t H, int64_t Hkv, int64_t seq, int64_t D,
                          int64_t B, int64_t nbm, const uint8_t* bmask, double scale,
                          int64_t n_rows, const int64_t* rows, double* out, double* lse,
                          int nthreads)
{
    if (!q || !k || !v || !out || !lse || !bmask || batch < 1 || H < 1 || Hkv < 1 ||
        H % Hkv != 0 || seq < 1 || D < 1 || B < 1 || nbm < (seq + B - 1) / B || n_rows < 0)
        return -1;
    if (!rows && n_rows != batch * H * seq) return -1;
    if (rows)
        for (int64_t t = 0; t < n_rows; ++t)
            if (rows[t] < 0 || rows[t] >= batch * H * seq) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 0;
    J.q = q; J.k = k; J.v = v;
    J.batch = batch; J.H = H; J.seq = seq; J.D = D; J.B = B; J.Hkv = Hkv;
    J.bmask = bmask; J.nbm = nbm; J.scale = scale;
    J.n_items = n_rows; J.items = rows; J.out = out; J.lse = lse;
    return run_job(&J, nthreads);
}

/* Decode oracle on selected (sequence, head) items.
 * q: bf16 bits [batch][H][D]; k_cache, v_cache: [num_pages][H][page_size][D];
 * block_table: [batch][max_pages] physical page ids; ctx_lens: [batch], >= 1.
 * items: n_items ids s * H + h, or NULL for all in order (n_items = batch*H).
 * out: [n_items][D], lse: [n_items]. Returns 0, or -1 on a bad argument
 * (including a negative page id inside a context). */
int s2o_decode_items(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                     const int32_t* block_table, const int32_t* ctx_lens,
                     int64_t batch, int64_t H, int64_t D, int64_t page_size,
                     int64_t max_pages, int64_t B, int64_t S, int64_t L,
                     const uint8_t* dense, double scale, int64_t n_items,
                     const int64_t* items, double* out, double* lse, int nthreads)
{
    if (!q || !k_cache || !v_cache || !block_table || !ctx_lens || !out || !lse ||
        batch < 1 || H < 1 || D < 1 || page_size < 1 || max_pages < 1 || B < 1 ||
        S < 1 || L < 1 || n_items < 0)
        return -1;
    if (!items && n_items != batch * H) return -1;
    for (int64_t s = 0; s < batch; ++s)
        if (ctx_lens[s] < 1 || ctx_lens[s] > max_pages * page_size) return -1;
    if (items)
        for (int64_t t = 0; t < n_items; ++t)
            if (items[t] < 0 || items[t] >= batch * H) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 1;
    J.q = q; J.k = k_cache; J.v = v_cache;
    J.block_table = block_table; J.ctx_lens = ctx_lens;
    J.batch = batch; J.H = H; J.D = D; J.page_size = page_size; J.max_pages = max_pages;
    J.B = B; J.S = S; J.L = L; J.dense = dense; J.scale = scale; J.Hkv = H;
    J.n_items = n_items; J.items = items; J.out = out; J.lse = lse;
    return run_job(&J, nthreads);
}

/* Decode oracle under a given block mask [H][nbm][nbm] (nbm >= the block count
 * of the longest context) and Hkv key/value heads: the caches are
 * [num_pages][Hkv][page_size][D]. Other arguments as s2o_decode_items. */
int s2o_decode_items_mask(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                          const int32_t* block_table, const int32_t* ctx_lens,
                          int64_t batch, int64_t H, int64_t Hkv, int64_t D, int64_t page_size,
                          int64_t max_pages, int64_t B, int64_t nbm, const uint8_t* bmask,
                          double scale, int64_t n_items, const int64_t* items, double* out,
                          double* lse, int nthreads)
{
    if (!q || !k_cache || !v_cache || !block_table || !ctx_lens || !out || !lse || !bmask ||
        batch < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || D < 1 || page_size < 1 ||
        max_pages < 1 || B < 1 || nbm < 1 || n_items < 0)
        return -1;
    if (!items && n_items != batch * H) return -1;
    for (int64_t s = 0; s < batch; ++s)
        if (ctx_lens[s] < 1 || ctx_lens[s] > max_pages * page_size ||
            (ctx_lens[s] - 1) / B >= nbm)
            return -1;
    if (items)
        for (int64_t t = 0; t < n_items; ++t)
            if (items[t] < 0 || items[t] >= batch * H) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 1;
    J.q = q; J.k = k_cache; J.v = v_cache;
    J.block_table = block_table; J.ctx_lens = ctx_lens;
    J.batch = batch; J.H = H; J.Hkv = Hkv; J.D = D; J.page_size = page_size;
    J.max_pages = max_pages; J.B = B; J.bmask = bmask; J.nbm = nbm; J.scale = scale;
    J.n_items = n_items; J.items = items; J.out = out; J.lse = lse;
    return run_job(&J, nthreads);
}

/* Backward oracle (the gradients in the header) under the HHST rule
 * (bmask == NULL; S, L, dense as s2o_prefill_rows) or a block mask
 * [H][nbm][nbm] (nbm >= ceil(seq / B)). q, dout: [batch][H][seq][D];
 * k, v: [batch][Hkv][seq][D]. dq: [batch][H][seq][D]; dk, dv:
 * [batch][Hkv][seq][D], fp64. The softmax is recomputed here in fp64 (no
 * saved statistics are taken from the caller). Returns 0 or -1. */
int s2o_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                 int64_t batch, int64_t H, int64_t Hkv, int64_t seq, int64_t D, int64_t B,
                 int64_t S, int64_t L, const uint8_t* dense, int64_t nbm, const uint8_t* bmask,
                 double scale, double* dq, double* dk, double* dv, int nthreads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv || batch < 1 || H < 1 || Hkv < 1 ||
        H % Hkv != 0 || seq < 1 || D < 1 || B < 1)
        return -1;
    if (bmask ? nbm < (seq + B - 1) / B : (S < 1 || L < 1)) return -1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 2;
    J.q = q; J.k = k; J.v = v; J.dout = dout;
    J.dq = dq; J.dk = dk; J.dv = dv;
    J.batch = batch; J.H = H; J.Hkv = Hkv; J.seq = seq; J.D = D; J.B = B;
    J.S = S; J.L = L; J.dense = dense; J.bmask = bmask; J.nbm = nbm; J.scale = scale;
    J.n_items = batch * Hkv; J.items = NULL;
    return run_job(&J, nthreads);
}

/* Backward oracle on a sample: the gradients of s2o_backward for chosen rows.
 * planes[n_planes]: K/V planes b * Hkv + g. qrows[nq]: query rows of each
 * sampled plane's group, hh * seq + q (query head g * (H / Hkv) + hh).
 * krows[nk]: key positions. Outputs dq [n_planes][nq][D], dk and dv
 * [n_planes][nk][D], fp64. Each row's softmax statistics are computed by
 * their definitions from q_lo = the smallest sampled position on (a key is
 * seen only by rows at or after it), then each sampled gradient row sums its
 * terms one by one. Returns 0 or -1. */
int s2o_backward_sampled(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                         const uint16_t* dout, int64_t batch, int64_t H, int64_t Hkv, int64_t seq,
                         int64_t D, int64_t B, int64_t S, int64_t L, const uint8_t* dense,
                         int64_t nbm, const uint8_t* bmask, double scale, int64_t n_planes,
                         const int64_t* planes, int64_t nq, const int64_t* qrows, int64_t nk,
                         const int64_t* krows, double* dq, double* dk, double* dv, int nthreads)
{
    if (!q || !k || !v || !dout || batch < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || seq < 1 ||
        D < 1 || B < 1 || n_planes < 1 || !planes || nq < 0 || nk < 0 || nq + nk < 1 ||
        (nq && (!qrows || !dq)) || (nk && (!krows || !dk || !dv)))
        return -1;
    if (bmask ? nbm < (seq + B - 1) / B : (S < 1 || L < 1)) return -1;
    const int64_t grp = H / Hkv;
    int64_t q_lo = seq;
    for (int64_t p = 0; p < n_planes; ++p)
        if (planes[p] < 0 || planes[p] >= batch * Hkv) return -1;
    for (int64_t r = 0; r < nq; ++r) {
        if (qrows[r] < 0 || qrows[r] >= grp * seq) return -1;
        if (qrows[r] % seq < q_lo) q_lo = qrows[r] % seq;
    }
    for (int64_t r = 0; r < nk; ++r) {
        if (krows[r] < 0 || krows[r] >= seq) return -1;
        if (krows[r] < q_lo) q_lo = krows[r];
    }
    const size_t nst = (size_t)(n_planes * grp * seq);
    double* st_lse = (double*)malloc(sizeof(double) * nst);
    double* st_D = (double*)malloc(sizeof(double) * nst);
    if (!st_lse || !st_D) {
        free(st_lse);
        free(st_D);
        return -1;
    }
    job_t J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v; J.dout = dout;
    J.dq = dq; J.dk = dk; J.dv = dv;
    J.batch = batch; J.H = H; J.Hkv = Hkv; J.seq = seq; J.D = D; J.B = B;
    J.S = S; J.L = L; J.dense = dense; J.bmask = bmask; J.nbm = nbm; J.scale = scale;
    J.n_planes = n_planes; J.planes = planes; J.nq = nq; J.qrows = qrows; J.nk = nk;
    J.krows = krows; J.q_lo = q_lo; J.st_lse = st_lse; J.st_D = st_D;
    J.kind = 4;
    J.n_items = n_planes * grp * (seq - q_lo);
    int rc = run_job(&J, nthreads);
    if (rc == 0) {
        J.kind = 5;
        J.n_items = n_planes * (nq + nk);
        rc = run_job(&J, nthreads);
    }
    free(st_lse);
    free(st_D);
    return rc;
}

/* Chunked-prefill oracle: each sequence s appends a chunk of
 * q_start[s+1] - q_start[s] query tokens at the end of a paged context of
 * ctx_lens[s] tokens (the chunk's own keys and values already in the cache);
 * every chunk row attends to keys 0..its position under the HHST rule
 * (bmask == NULL; S, L, dense) or a block mask [H][nbm][nbm].
 * q: [total_q][H][D] packed rows (total_q = q_start[batch]); caches
 * [num_pages][Hkv][page_size][D]; out [total_q][H][D], lse [total_q][H].
 * Returns 0 or -1 (a chunk longer than its context, a bad page id, ...). */
int s2o_chunk_rows(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                   const int32_t* block_table, const int32_t* ctx_lens, const int32_t* q_start,
                   int64_t batch, int64_t H, int64_t Hkv, int64_t D, int64_t page_size,
                   int64_t max_pages, int64_t B, int64_t S, int64_t L, const uint8_t* dense,
                   int64_t nbm, const uint8_t* bmask, double scale, double* out, double* lse,
                   int nthreads)
{
    if (!q || !k_cache || !v_cache || !block_table || !ctx_lens || !q_start || !out || !lse ||
        batch < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || D < 1 || page_size < 1 ||
        max_pages < 1 || B < 1 || q_start[0] != 0)
        return -1;
    if (bmask ? nbm < 1 : (S < 1 || L < 1)) return -1;
    for (int64_t s = 0; s < batch; ++s) {
        const int64_t ql = q_start[s + 1] - q_start[s];
        if (ql < 0 || ctx_lens[s] < ql || ctx_lens[s] > max_pages * page_size) return -1;
        if (bmask && ctx_lens[s] > 0 && (ctx_lens[s] - 1) / B >= nbm) return -1;
    }
    job_t J;
    memset(&J, 0, sizeof J);
    J.kind = 3;
    J.q = q; J.k = k_cache; J.v = v_cache;
    J.block_table = block_table; J.ctx_lens = ctx_lens; J.q_start = q_start;
    J.batch = batch; J.H = H; J.Hkv = Hkv; J.D = D; J.page_size = page_size;
    J.max_pages = max_pages; J.B = B; J.S = S; J.L = L; J.dense = dense;
    J.bmask = bmask; J.nbm = nbm; J.scale = scale;
    J.n_items = q_start[batch] * H; J.items = NULL; J.out = out; J.lse = lse;
    return run_job(&J, nthreads);
}
