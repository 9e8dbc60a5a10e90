/*
 * attn_oracle.c -- fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY. The test-suite, the smoke check and the CPU-baseline leg of
 * the benchmark are the only code that may load this library. The product path (the CUDA
 * library and its Python binding) never calls it, and this file shares no code, header or
 * constant with that path.
 *
 * What is computed, and where it is defined:
 *
 *   "Resumen Tecnico: FlashMLA-ETAP" (gist.science, paper 2506.01969), section
 *   "Mecanismo Central": the standard flow S = Q.K^T, P = softmax(S), O = P.V, and the
 *   transposed flow S^T = K.Q^T, P^T = softmax(S^T), O = (V^T.P^T)^T that gives the same O.
 *
 *   "Activar Flash Attention con llama.cpp" (quellm.com), section "Que es Flash Attention":
 *   the tiled method changes only where the intermediates live (on-chip instead of HBM), not
 *   the result. So the oracle is the plain definition, materialising S and P.
 *
 *   Same page, FAQ "diferencia entre Flash Attention y GQA": key/value heads are shared by
 *   groups of query heads. Reading taken: contiguous groups, kv head = h / (Hq / Hkv).
 *
 *   FlashMLA-ETAP summary, sections "Planteamiento del Problema" and "Limitaciones": the MLA
 *   decode shape (16 heads, head dim 576, KV up to 64K, 1-2 query tokens). Reading taken:
 *   one latent KV head whose first 512 columns also serve as V, passed here as v == k with
 *   a row stride ldv = 576.
 *
 * Readings where the pages are silent (each one is listed in the design notes too):
 *   - scale multiplies Q.K^T before the softmax (s_ij = scale * q_i . k_j);
 *   - causal masking is bottom-right aligned: key j is visible to query row i iff
 *     j <= i + (Lk - Lq); the Lq new tokens are the last Lq positions of the sequence;
 *   - LSE is the natural log of sum_j exp(s_ij) over the visible keys, scale included;
 *   - an empty visible set gives O = 0 and LSE = -inf (this only occurs for split
 *     partials, never for a whole row, because causal calls need Lq <= Lk);
 *   - inputs are 16-bit bit patterns, all bf16 or all IEEE binary16 (fp16, the input type of
 *     the FlashMLA-ETAP summary's H20 figures, "Planteamiento del Problema"); each value is
 *     widened exactly to double.
 *
 *   MInference article (7minutos.es), on the sparse patterns of long-context prefill (A-shape,
 *   vertical bar, block-sparse): with a given sparse index the attention stays the exact
 *   softmax, restricted to the listed keys. Reading taken for the block form: query rows are
 *   cut into blocks of blk_q rows and keys into blocks of blk_k keys; query block qb of head
 *   (b, h) sees exactly the key blocks in its list (and the causal mask still applies). A row
 *   that sees no key gets O = 0 and LSE = -inf.
 *
 * Layouts (row-major, contiguous): q [B,Hq,Lq,d], k [B,Hkv,Lk,d], v [B,Hkv,Lk,ldv] with
 * the first dv columns used; outputs are double. Block lists: cnt [B,Hq,ceil(Lq/blk_q)] and
 * idx [B,Hq,ceil(Lq/blk_q),max_blk] (int32; the first cnt entries of each list are used).
 *
 * Build: gcc -O2 -shared -fPIC -pthread attn_oracle.c -o liboracle.so -lm
 * ORACLE_MUTANT (compile-time, default 0) plants one deliberate mistake; only the mutation
 * tests build it non-zero, to show that the pins catch each mistake.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

enum { ELEM_BF16 = 0, ELEM_F16 = 1 };

/* bf16 bit pattern -> double, exact (bf16 is the upper half of an IEEE binary32). */
static double widen_bf16(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * IEEE 754 binary16 bit pattern -> double, exact, from the format's definition: sign bit 15,
 * 5-bit biased exponent e (bias 15) in bits 10-14, 10-bit fraction f. e = 0 is zero or
 * subnormal, f * 2^-24; 1 <= e <= 30 is (1024 + f) * 2^(e - 25); e = 31 is +-inf (f = 0)
 * or NaN. Every binary16 value is a double, so ldexp is exact.
 */
static double widen_f16(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, f = h & 1023;
    double mag;
    if (e == 31) {
        mag = f == 0 ? INFINITY : NAN;
    } else if (e == 0) {
#if ORACLE_MUTANT == 9
        mag = ldexp((double)(1024 + f), -24); /* planted: implicit leading one on subnormals */
#else
        mag = ldexp((double)f, -24);
#endif
    } else {
        mag = ldexp((double)(1024 + f), e - 25);
    }
    return s ? -mag : mag;
}

static double widen(int elem, uint16_t h) {
    return elem == ELEM_F16 ? widen_f16(h) : widen_bf16(h);
}

typedef struct {
    const uint16_t *q, *k, *v;
    int64_t B, Hq, Hkv, Lq, Lk, d, dv, ldv;
    double scale;
    int causal;
    int64_t kv_begin, kv_end;
    int elem;
    const int32_t *blk_idx, *blk_cnt; /* NULL: dense */
    int64_t max_blk, blk_q, blk_k;
} problem;

static int check_problem(const problem *p) {
    if (!p->q || !p->k || !p->v) return 1;
    if (p->B < 1 || p->Hq < 1 || p->Hkv < 1 || p->Lq < 1 || p->Lk < 1) return 1;
    if (p->d < 1 || p->dv < 1 || p->ldv < p->dv) return 1;
    if (p->Hq % p->Hkv != 0) return 1;
    if (p->kv_begin < 0 || p->kv_end > p->Lk || p->kv_begin > p->kv_end) return 1;
    if (p->elem != ELEM_BF16 && p->elem != ELEM_F16) return 1;
    if (p->blk_cnt) {
        if (!p->blk_idx || p->blk_q < 1 || p->blk_k < 1 || p->max_blk < 0) return 1;
        const int64_t nqb = (p->Lq + p->blk_q - 1) / p->blk_q, nkb = (p->Lk + p->blk_k - 1) / p->blk_k;
        for (int64_t s = 0; s < p->B * p->Hq * nqb; ++s) {
            if (p->blk_cnt[s] < 0 || p->blk_cnt[s] > p->max_blk) return 1;
            for (int32_t t = 0; t < p->blk_cnt[s]; ++t) {
                const int32_t kb = p->blk_idx[s * p->max_blk + t];
                if (kb < 0 || kb >= nkb) return 1;
            }
        }
    }
    return 0;
}

/* kv head that serves query head h (GQA, contiguous groups). */
static int64_t kv_head_of(const problem *p, int64_t h) {
#if ORACLE_MUTANT == 3
    return h % p->Hkv; /* planted: interleaved instead of contiguous groups */
#else
    return h / (p->Hq / p->Hkv);
#endif
}

/* Is key j in one of the key blocks listed for the query block of row i of head (b, h)? */
static int listed(const problem *p, int64_t b, int64_t h, int64_t i, int64_t j) {
    if (!p->blk_cnt) return 1;
    const int64_t nqb = (p->Lq + p->blk_q - 1) / p->blk_q;
    const int64_t slot = (b * p->Hq + h) * nqb + i / p->blk_q;
    const int64_t kb = j / p->blk_k;
    const int32_t *lst = p->blk_idx + slot * p->max_blk;
    for (int32_t t = 0; t < p->blk_cnt[slot]; ++t) {
#if ORACLE_MUTANT == 10
        if (kb <= lst[t]) return 1; /* planted: the list read as an upper bound */
#else
        if (lst[t] == kb) return 1;
#endif
    }
    return 0;
}

/* Is key j visible to query row i of head (b, h)? */
static int visible(const problem *p, int64_t b, int64_t h, int64_t i, int64_t j) {
    if (j < p->kv_begin || j >= p->kv_end) return 0;
    if (!listed(p, b, h, i, j)) return 0;
#if ORACLE_MUTANT == 14
    if (p->blk_cnt) return 1; /* planted: a listed block bypasses the causal rule */
#endif
    if (!p->causal) return 1;
#if ORACLE_MUTANT == 4
    return j <= i; /* planted: top-left alignment */
#else
    return j <= i + (p->Lk - p->Lq);
#endif
}

static double dot_qk(const problem *p, int64_t b, int64_t h, int64_t i, int64_t j) {
    const uint16_t *qr = p->q + ((b * p->Hq + h) * p->Lq + i) * p->d;
    const uint16_t *kr = p->k + ((b * p->Hkv + kv_head_of(p, h)) * p->Lk + j) * p->d;
    /* four partial sums: a plain fp64 dot product, split only so the loop pipelines */
    double a0 = 0, a1 = 0, a2 = 0, a3 = 0;
    int64_t c = 0;
    for (; c + 4 <= p->d; c += 4) {
        a0 += widen(p->elem, qr[c + 0]) * widen(p->elem, kr[c + 0]);
        a1 += widen(p->elem, qr[c + 1]) * widen(p->elem, kr[c + 1]);
        a2 += widen(p->elem, qr[c + 2]) * widen(p->elem, kr[c + 2]);
        a3 += widen(p->elem, qr[c + 3]) * widen(p->elem, kr[c + 3]);
    }
    for (; c < p->d; ++c) a0 += widen(p->elem, qr[c]) * widen(p->elem, kr[c]);
    return (a0 + a1) + (a2 + a3);
}

static double v_at(const problem *p, int64_t b, int64_t hkv, int64_t j, int64_t c) {
#if ORACLE_MUTANT == 5
    /* planted: operand indexed transposed (column-major read of a row-major V) */
    int64_t flat = c * p->Lk + j;
    int64_t jj = flat / p->ldv % p->Lk, cc = flat % p->ldv;
    return widen(p->elem, p->v[((b * p->Hkv + hkv) * p->Lk + jj) * p->ldv + cc]);
#else
    return widen(p->elem, p->v[((b * p->Hkv + hkv) * p->Lk + j) * p->ldv + c]);
#endif
}

/*
 * One query row, standard flow: materialise the score row s_j = scale * q_i . k_j over the
 * visible set, the probability row P_j = exp(s_j - m) / sum_l exp(s_l - m), then
 * O = sum_j P_j v_j and LSE = m + ln sum_j exp(s_j - m).
 * s and pr are scratch rows of length Lk. If p_out is not NULL the full probability row
 * (zeros at masked keys) is copied there.
 */
static void one_row(const problem *p, int64_t row, double *s, double *pr, double *o,
                    double *lse, double *p_out) {
    int64_t i = row % p->Lq;
    int64_t h = (row / p->Lq) % p->Hq;
    int64_t b = row / (p->Lq * p->Hq);
    int64_t hkv = kv_head_of(p, h);

    double m = -INFINITY;
    int64_t n_vis = 0;
    for (int64_t j = 0; j < p->Lk; ++j) {
        if (!visible(p, b, h, i, j)) { s[j] = -INFINITY; continue; }
#if ORACLE_MUTANT == 7
        s[j] = dot_qk(p, b, h, i, j); /* planted: scale dropped */
#else
        s[j] = p->scale * dot_qk(p, b, h, i, j);
#endif
        if (s[j] > m) m = s[j];
        ++n_vis;
    }
    for (int64_t c = 0; c < p->dv; ++c) o[c] = 0.0;
    if (n_vis == 0) {
        *lse = -INFINITY;
        if (p_out) for (int64_t j = 0; j < p->Lk; ++j) p_out[j] = 0.0;
        return;
    }
    double l = 0.0;
    for (int64_t j = 0; j < p->Lk; ++j) {
        if (s[j] == -INFINITY) { pr[j] = 0.0; continue; }
#if ORACLE_MUTANT == 1
        pr[j] = exp(s[j]); /* planted: no max subtraction */
#elif ORACLE_MUTANT == 2
        pr[j] = exp(m - s[j]); /* planted: wrong sign */
#else
        pr[j] = exp(s[j] - m);
#endif
        l += pr[j];
    }
#if ORACLE_MUTANT != 8
    for (int64_t j = 0; j < p->Lk; ++j) pr[j] /= l; /* P = softmax(S) */
#endif
#if ORACLE_MUTANT == 1
    *lse = log(l);
#elif ORACLE_MUTANT == 6
    *lse = log(l); /* planted: max term dropped from LSE */
#else
    *lse = m + log(l);
#endif
    for (int64_t j = 0; j < p->Lk; ++j) {
        if (pr[j] == 0.0) continue;
        for (int64_t c = 0; c < p->dv; ++c) o[c] += pr[j] * v_at(p, b, hkv, j, c);
    }
    if (p_out) memcpy(p_out, pr, (size_t)p->Lk * sizeof(double));
}

typedef struct {
    const problem *p;
    const int64_t *rows;
    int64_t begin, end;
    double *o, *lse;
    int err;
} job;

static void *run_job(void *arg) {
    job *jb = (job *)arg;
    const problem *p = jb->p;
    double *s = (double *)malloc((size_t)p->Lk * sizeof(double));
    double *pr = (double *)malloc((size_t)p->Lk * sizeof(double));
    if (!s || !pr) { jb->err = 2; free(s); free(pr); return NULL; }
    for (int64_t r = jb->begin; r < jb->end; ++r)
        one_row(p, jb->rows[r], s, pr, jb->o + r * p->dv, jb->lse + r, NULL);
    free(s);
    free(pr);
    return NULL;
}

/*
 * Attention for a list of query rows. rows[r] is the flat row id (b*Hq + h)*Lq + i.
 * Only keys in [kv_begin, kv_end) take part (the whole row: 0, Lk); a sub-range gives the
 * split partial: O normalised by its own sum and the LSE of that range.
 * o: n_rows x dv, lse: n_rows. Returns 0 on success, 1 on bad arguments, 2 on no memory.
 */
static int run_rows(const problem *pp, const int64_t *rows, int64_t n_rows, double *o, double *lse,
                    int nthreads) {
    problem p = *pp;
    if (check_problem(&p) || (n_rows > 0 && (!rows || !o || !lse)) || n_rows < 0) return 1;
    int64_t total = p.B * p.Hq * p.Lq;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return 1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > n_rows) nthreads = (int)(n_rows > 0 ? n_rows : 1);
    pthread_t tid[256];
    job jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].p = &p;
        jobs[t].rows = rows;
        jobs[t].begin = n_rows * t / nthreads;
        jobs[t].end = n_rows * (t + 1) / nthreads;
        jobs[t].o = o;
        jobs[t].lse = lse;
        jobs[t].err = 0;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&tid[t], NULL, run_job, &jobs[t]);
    run_job(&jobs[0]);
    int err = jobs[0].err;
    for (int t = 1; t < nthreads; ++t) {
        pthread_join(tid[t], NULL);
        if (jobs[t].err) err = jobs[t].err;
    }
    return err;
}

/*
 * Attention for a list of query rows. rows[r] is the flat row id (b*Hq + h)*Lq + i.
 * Only keys in [kv_begin, kv_end) take part (the whole row: 0, Lk); a sub-range gives the
 * split partial: O normalised by its own sum and the LSE of that range.
 * o: n_rows x dv, lse: n_rows. Returns 0 on success, 1 on bad arguments, 2 on no memory.
 */
int oracle_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B,
                     int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk, int64_t d, int64_t dv,
                     int64_t ldv, double scale, int causal, int64_t kv_begin, int64_t kv_end,
                     const int64_t *rows, int64_t n_rows, double *o, double *lse, int elem,
                     int nthreads) {
    problem p = {q, k, v, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, kv_begin, kv_end, elem,
                 NULL, NULL, 0, 1, 1};
    return run_rows(&p, rows, n_rows, o, lse, nthreads);
}

/*
 * Block-sparse attention for a list of query rows: as oracle_attn_rows over all keys, with
 * key j visible to row i of head (b, h) only if block j / blk_k is in the list of query block
 * i / blk_q (lists: cnt [B,Hq,nqb], idx [B,Hq,nqb,max_blk], entries in [0, ceil(Lk/blk_k))).
 */
int oracle_attn_rows_sparse(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t B,
                            int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk, int64_t d,
                            int64_t dv, int64_t ldv, double scale, int causal, int64_t blk_q,
                            int64_t blk_k, const int32_t *blk_idx, const int32_t *blk_cnt,
                            int64_t max_blk, const int64_t *rows, int64_t n_rows, double *o,
                            double *lse, int elem, int nthreads) {
    if (!blk_cnt) return 1;
    problem p = {q, k, v, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, 0, Lk, elem,
                 blk_idx, blk_cnt, max_blk, blk_q, blk_k};
    return run_rows(&p, rows, n_rows, o, lse, nthreads);
}

/* The probability row P[i, :] (length Lk, zero at masked keys) of one flat row id. */
int oracle_softmax_row(const uint16_t *q, const uint16_t *k, int64_t B, int64_t Hq,
                       int64_t Hkv, int64_t Lq, int64_t Lk, int64_t d, double scale,
                       int causal, int64_t row, double *p_out, int elem) {
    problem p = {q, k, k, B, Hq, Hkv, Lq, Lk, d, 1, d, scale, causal, 0, Lk, elem, NULL, NULL, 0, 1, 1};
    if (check_problem(&p) || row < 0 || row >= B * Hq * Lq || !p_out) return 1;
    double *s = (double *)malloc((size_t)Lk * sizeof(double));
    double *pr = (double *)malloc((size_t)Lk * sizeof(double));
    double o1, l1;
    if (!s || !pr) { free(s); free(pr); return 2; }
    one_row(&p, row, s, pr, &o1, &l1, p_out);
    free(s);
    free(pr);
    return 0;
}

/*
 * Transposed flow of the FlashMLA-ETAP summary ("Mecanismo Central", item 1) for one
 * (batch, query head): St = K.Q^T (Lk x Lq, scaled), Pt = column-wise softmax of St
 * (over the key index, per query column), Ot = V^T.Pt (dv x Lq), then O = Ot^T.
 * All three matrices are materialised. o: Lq x dv, lse: Lq.
 */
int oracle_attn_transposed_head(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                int64_t B, int64_t Hq, int64_t Hkv, int64_t Lq, int64_t Lk,
                                int64_t d, int64_t dv, int64_t ldv, double scale, int causal,
                                int64_t b, int64_t h, double *o, double *lse, int elem) {
    problem p = {q, k, v, B, Hq, Hkv, Lq, Lk, d, dv, ldv, scale, causal, 0, Lk, elem, NULL, NULL, 0, 1, 1};
    if (check_problem(&p) || b < 0 || b >= B || h < 0 || h >= Hq || !o || !lse) return 1;
    int64_t hkv = kv_head_of(&p, h);
    double *St = (double *)malloc((size_t)(Lk * Lq) * sizeof(double));
    double *Ot = (double *)malloc((size_t)(dv * Lq) * sizeof(double));
    if (!St || !Ot) { free(St); free(Ot); return 2; }
    /* St[j][i] = scale * sum_c K[j][c] * Q[i][c] */
    for (int64_t j = 0; j < Lk; ++j) {
        const uint16_t *kr = k + ((b * Hkv + hkv) * Lk + j) * d;
        for (int64_t i = 0; i < Lq; ++i) {
            const uint16_t *qr = q + ((b * Hq + h) * Lq + i) * d;
            double acc = 0.0;
            for (int64_t c = 0; c < d; ++c) acc += widen(elem, kr[c]) * widen(elem, qr[c]);
            St[j * Lq + i] = visible(&p, b, h, i, j) ? scale * acc : -INFINITY;
        }
    }
    /* Pt = softmax over j of each column i (in place) */
    for (int64_t i = 0; i < Lq; ++i) {
        double m = -INFINITY, l = 0.0;
        for (int64_t j = 0; j < Lk; ++j) if (St[j * Lq + i] > m) m = St[j * Lq + i];
        if (m == -INFINITY) {
            for (int64_t j = 0; j < Lk; ++j) St[j * Lq + i] = 0.0;
            lse[i] = -INFINITY;
            continue;
        }
        for (int64_t j = 0; j < Lk; ++j) {
            double e = St[j * Lq + i] == -INFINITY ? 0.0 : exp(St[j * Lq + i] - m);
            St[j * Lq + i] = e;
            l += e;
        }
        for (int64_t j = 0; j < Lk; ++j) St[j * Lq + i] /= l;
        lse[i] = m + log(l);
    }
#if ORACLE_MUTANT == 12
    /* planted: each key's probabilities renormalised over the queries (the wrong axis of P^T) */
    for (int64_t j = 0; j < Lk; ++j) {
        double t = 0.0;
        for (int64_t i = 0; i < Lq; ++i) t += St[j * Lq + i];
        if (t > 0.0)
            for (int64_t i = 0; i < Lq; ++i) St[j * Lq + i] /= t;
    }
#endif
    /* Ot[c][i] = sum_j V[j][c] * Pt[j][i] */
    for (int64_t c = 0; c < dv; ++c)
        for (int64_t i = 0; i < Lq; ++i) {
            double acc = 0.0;
            for (int64_t j = 0; j < Lk; ++j)
                acc += widen(elem, v[((b * Hkv + hkv) * Lk + j) * ldv + c]) * St[j * Lq + i];
            Ot[c * Lq + i] = acc;
        }
    /* O = Ot^T */
    for (int64_t i = 0; i < Lq; ++i)
        for (int64_t c = 0; c < dv; ++c)
#if ORACLE_MUTANT == 13
            o[i * dv + c] = Ot[i * dv + c]; /* planted: the final transpose left out */
#else
            o[i * dv + c] = Ot[c * Lq + i];
#endif
    free(St);
    free(Ot);
    return 0;
}

/*
 * Merge of split partials over disjoint key ranges (the log-sum-exp combine):
 *   LSE = ln sum_s exp(lse_s),  O = sum_s exp(lse_s - LSE) * O_s.
 * Splits with lse_s = -inf hold no key and carry no weight.
 * o_parts: n_splits x n_rows x dv, lse_parts: n_splits x n_rows.
 */
int oracle_combine(const double *o_parts, const double *lse_parts, int64_t n_splits,
                   int64_t n_rows, int64_t dv, double *o, double *lse) {
    if (!o_parts || !lse_parts || !o || !lse || n_splits < 1 || n_rows < 0 || dv < 1)
        return 1;
    for (int64_t r = 0; r < n_rows; ++r) {
        double m = -INFINITY;
        for (int64_t s = 0; s < n_splits; ++s)
            if (lse_parts[s * n_rows + r] > m) m = lse_parts[s * n_rows + r];
        for (int64_t c = 0; c < dv; ++c) o[r * dv + c] = 0.0;
        if (m == -INFINITY) { lse[r] = -INFINITY; continue; }
        double sum = 0.0;
        for (int64_t s = 0; s < n_splits; ++s) {
            double ls = lse_parts[s * n_rows + r];
            if (ls == -INFINITY) continue;
            sum += exp(ls - m);
        }
        double L = m + log(sum);
        lse[r] = L;
        for (int64_t s = 0; s < n_splits; ++s) {
            double ls = lse_parts[s * n_rows + r];
            if (ls == -INFINITY) continue;
#if ORACLE_MUTANT == 11
            double w = exp(ls - m); /* planted: weights not divided by the sum over splits */
#else
            double w = exp(ls - L);
#endif
            for (int64_t c = 0; c < dv; ++c) o[r * dv + c] += w * o_parts[(s * n_rows + r) * dv + c];
        }
    }
    return 0;
}

/* The exact widening the oracle applies: out[i] = value of the 16-bit pattern in[i] read as
 * elem (0 = bf16, 1 = fp16). Returns 1 for an unknown elem. */
int oracle_widen(const uint16_t *in, int64_t n, int elem, double *out) {
    if ((elem != ELEM_BF16 && elem != ELEM_F16) || n < 0 || (n > 0 && (!in || !out))) return 1;
    for (int64_t i = 0; i < n; ++i) out[i] = widen(elem, in[i]);
    return 0;
}

int oracle_mutant_id(void) { return ORACLE_MUTANT; }
