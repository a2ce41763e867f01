/*
 * li_oracle.c -- plain fp64 CPU oracle for the LightningIndexer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * helper with the CUDA library; the two meet only in the seeded inputs.
 *
 * What it computes, for every query row (batch b, position i), following the
 * formula of the mindspore.ops.lightning_indexer page (section ".. math::"),
 * the three-step flow of the CANN LightningIndexerV2 guide (section
 * "三步计算流程") and, for the quantised variant, the formula of the
 * VllmQuantLightningIndexer README (section "功能说明"):
 *
 *   for every key t of batch b that the sparse mode leaves visible:
 *     logit_h(t) = sum_d q[b,i,h,d] * k[b,t,d]                    (Q_index @ K_index^T)
 *     quant:       logit_h(t) *= Scale_Q[b,i,h] * Scale_K[b,t]    (dequant before ReLU)
 *     s(t)       = sum_h W[b,i,h] * ReLU(logit_h(t))              ([1]_{1xg} @ (W (.) ReLU(.)))
 *   Top-k: order the visible keys by s descending (ties: lower key index
 *   first), keep min(k, visible) of them, pad the rest with index -1 and value
 *   -inf (CANN guide, "通用约束": invalid slots are -1 / -inf).
 *   Sink tokens and the local window (the open-sourcing issue's comparison of
 *   the MT lightning_indexer, which lists init_num -- sink tokens always
 *   selected -- and local_num -- the diagonal local window): the first
 *   init_num and the last local_num visible keys are always kept; the other
 *   min(k, visible) - |forced| slots take the best of the remaining visible
 *   keys; all kept keys are then ordered as above.
 *
 * Everything is evaluated in double precision from the exact values the
 * stored bits encode (bf16, fp16, fp8 e4m3 and int8 are decoded here from
 * their format definitions), so the oracle sees exactly the inputs a GPU sees.
 *
 * Readings taken where the pages are silent (each one is also listed in the
 * design notes of the repository):
 *   - right-down causal (sparse_mode 3): key t is visible to query i of batch
 *     b iff t <= i + Sk_b - Sq_b (the triangle anchored at the bottom-right);
 *   - the deterministic Top-k breaks ties toward the lower key index;
 *   - indices are positions inside the batch's own key sequence;
 *   - TND actual lengths are prefix sums (no leading 0), BSND/PA are counts;
 *   - BSND rows with i >= actual query length are pure padding;
 *   - compressed keys (CANN LightningIndexerV2 guide: cmp_ratio, with
 *     cmp_residual_k < cmp_ratio under mask_mode 3): compressed key t stands
 *     for the cmp_ratio original tokens [t*r, (t+1)*r); the batch's original
 *     key length is Sk*r + residual; under right-down causal masking t is
 *     visible once its last original token (t+1)*r - 1 is, i.e. when
 *     (t+1)*r - 1 <= i + Sk*r + residual - Sq.  Indices count compressed keys.
 *
 * Planted mistakes: the field `mutation` (0 in every real use) lets the tests
 * inject one deliberate error at a time into this oracle, to show that each
 * pin fails when the oracle is wrong.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_BF16 = 0, OR_FP16 = 1, OR_FP32 = 2, OR_E4M3 = 3, OR_INT8 = 4 };
enum { OR_BSND = 0, OR_TND = 1, OR_PA_BSND = 2 };

typedef struct {
    int32_t layout_q, layout_k;
    int32_t dtype_qk, dtype_w, dtype_scale;
    int32_t quant;
    int32_t B, S1, S2, T1, T2, N1, N2, D;
    int32_t num_blocks, block_size, max_blocks_per_seq;
    int64_t key_block_stride;      /* elements between PA blocks; 0 = block_size*N2*D */
    int32_t sparse_count, sparse_mode, return_value;
    int32_t mutation;              /* 0 = the real oracle; >0 plants one mistake */
    int32_t init_num, local_num;   /* forced sink tokens / local window (0 = none) */
    int32_t cmp_ratio;             /* original tokens per key (0 or 1 = none) */
    const int32_t *cmp_residual_k; /* [B] leftover original tokens (mode 3, cmp_ratio > 1) */
} or_problem;

/* ---- decoders, from the format definitions ------------------------------ */

/* bfloat16: the upper half of an IEEE binary32. */
static double dec_bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
static double dec_fp16(uint16_t h)
{
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);     /* (1 + m/2^10) * 2^(e-15) */
    return s ? -v : v;
}

/* OCP FP8 E4M3 ("fn"): bias 7, no infinities, S.1111.111 is NaN, max 448. */
static double dec_e4m3(uint8_t b)
{
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9);                  /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);        /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

static double load(const void *base, int64_t i, int dtype)
{
    switch (dtype) {
    case OR_BF16: return dec_bf16(((const uint16_t *)base)[i]);
    case OR_FP16: return dec_fp16(((const uint16_t *)base)[i]);
    case OR_FP32: return (double)((const float *)base)[i];
    case OR_E4M3: return dec_e4m3(((const uint8_t *)base)[i]);
    case OR_INT8: return (double)((const int8_t *)base)[i];
    }
    return NAN;
}

double li_oracle_decode(const void *base, int64_t i, int dtype) { return load(base, i, dtype); }

/* ---- sequence bookkeeping (mindspore page, "actual_seq_lengths_*") -------- */

typedef struct { int64_t q_off, k_off; int64_t Sq, Sk; int64_t res; } seq_info;

static seq_info seq_of(const or_problem *p, const int32_t *act_q, const int32_t *act_k, int b)
{
    seq_info s;
    if (p->layout_q == OR_TND) {                       /* prefix sums, no leading 0 */
        s.q_off = b ? act_q[b - 1] : 0;
        s.Sq = act_q[b] - s.q_off;
    } else {
        s.q_off = (int64_t)b * p->S1;
        s.Sq = act_q ? act_q[b] : p->S1;
    }
    if (p->layout_k == OR_TND) {
        s.k_off = b ? act_k[b - 1] : 0;
        s.Sk = act_k[b] - s.k_off;
    } else if (p->layout_k == OR_BSND) {
        s.k_off = (int64_t)b * p->S2;
        s.Sk = act_k ? act_k[b] : p->S2;
    } else {                                           /* PA: a count per batch */
        s.k_off = 0;
        s.Sk = act_k[b];
    }
    s.res = (p->cmp_ratio > 1 && p->sparse_mode == 3 && p->cmp_residual_k) ? p->cmp_residual_k[b] : 0;
    return s;
}

/* Element offset of key t, feature d, of batch b (head n2 = 0). */
static int64_t key_elem(const or_problem *p, const int32_t *block_table, seq_info s, int b,
                        int64_t t, int d)
{
    if (p->layout_k == OR_PA_BSND) {
        int64_t stride = p->key_block_stride ? p->key_block_stride
                                             : (int64_t)p->block_size * p->N2 * p->D;
        int64_t blk = block_table[(int64_t)b * p->max_blocks_per_seq + t / p->block_size];
        return blk * stride + ((t % p->block_size) * p->N2) * p->D + d;
    }
    return ((s.k_off + t) * p->N2) * p->D + d;
}

/* Dequant scale of key t (per token, head n2 = 0). */
static double key_scale(const or_problem *p, const void *k_scale, const int32_t *block_table,
                        seq_info s, int b, int64_t t)
{
    if (p->layout_k == OR_PA_BSND) {
        int64_t blk = block_table[(int64_t)b * p->max_blocks_per_seq + t / p->block_size];
        return load(k_scale, (blk * p->block_size + t % p->block_size) * p->N2, p->dtype_scale);
    }
    return load(k_scale, (s.k_off + t) * p->N2, p->dtype_scale);
}

/* Visibility of key t to query i (mindspore page, "sparse_mode"; CANN guide,
 * "mask_mode 参数解释").  Mode 0 shows every key inside the actual length;
 * mode 3 is the right-down causal triangle. */
static int visible(const or_problem *p, seq_info s, int64_t i, int64_t t)
{
    if (t >= s.Sk)
        return 0;
    if (p->sparse_mode == 0)
        return 1;
    const int64_t r = p->cmp_ratio > 1 ? p->cmp_ratio : 1;
    const int64_t last_tok = (t + 1) * r - 1;            /* last original token of key t */
    const int64_t diag = i + s.Sk * r + s.res - s.Sq;    /* right-down causal, original tokens */
    if (p->mutation == 4)                      /* planted: off-by-one diagonal */
        return last_tok < diag;
    return last_tok <= diag;
}

typedef struct { double s; int64_t t; } cand;

static int cmp_cand(const void *a, const void *b)
{
    const cand *x = (const cand *)a, *y = (const cand *)b;
    if (x->s > y->s) return -1;                 /* larger score first */
    if (x->s < y->s) return 1;
    return (x->t < y->t) ? -1 : (x->t > y->t);  /* tie: lower key index first */
}
static int cmp_cand_hi_tie(const void *a, const void *b)   /* planted: higher index first */
{
    const cand *x = (const cand *)a, *y = (const cand *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->t > y->t) ? -1 : (x->t < y->t);
}
static int cmp_cand_asc(const void *a, const void *b)      /* planted: smallest first */
{
    return -cmp_cand(a, b);
}

/* Map a query row to (b, i).  BSND rows are b*S1+i; TND rows are token ids. */
static int row_to_bi(const or_problem *p, const int32_t *act_q, int64_t row, int *b, int64_t *i)
{
    if (p->layout_q == OR_BSND) {
        *b = (int)(row / p->S1);
        *i = row % p->S1;
        return 1;
    }
    for (int bb = 0; bb < p->B; ++bb) {
        int64_t lo = bb ? act_q[bb - 1] : 0;
        if (row >= lo && row < act_q[bb]) {
            *b = bb;
            *i = row - lo;
            return 1;
        }
    }
    return 0;   /* a TND row past the last prefix sum has no batch: padding */
}

/*
 * Evaluate `n_rows` query rows (all rows when rows == NULL).
 *   out_idx  [n_rows, k] int32    selected key indices, -1 padded
 *   out_val  [n_rows, k] float    their scores rounded to fp32, -inf padded
 *   out_v64  [n_rows, k] double   the same in fp64 (optional)
 *   scores   [n_rows, ld] double  full score row, NaN where invisible (optional)
 *   nvis     [n_rows] int64       number of visible keys (optional)
 * Returns 0, or -1 on a bad argument.
 */
int li_oracle_rows(const or_problem *p, const void *query, const void *key, const void *weights,
                   const void *q_scale, const void *k_scale, const int32_t *act_q,
                   const int32_t *act_k, const int32_t *block_table, const int64_t *rows,
                   int64_t n_rows, int32_t *out_idx, float *out_val, double *out_v64,
                   double *scores, int64_t ld, int64_t *nvis, int nthreads)
{
    if (!p || !query || !key || !weights || !out_idx || !out_val || p->N1 <= 0 || p->D <= 0)
        return -1;
    if (p->quant && (!q_scale || !k_scale))
        return -1;
    const int kk = p->sparse_count;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t row = rows ? rows[r] : r;
        int32_t *oi = out_idx + r * kk;
        float *ov = out_val + r * kk;
        double *o64 = out_v64 ? out_v64 + r * kk : NULL;
        for (int j = 0; j < kk; ++j) {
            oi[j] = -1;
            ov[j] = -INFINITY;
            if (o64) o64[j] = -INFINITY;
        }
        if (nvis) nvis[r] = 0;
        if (scores)
            for (int64_t t = 0; t < ld; ++t) scores[r * ld + t] = NAN;
        int b;
        int64_t i;
        if (!row_to_bi(p, act_q, row, &b, &i))
            continue;
        seq_info s = seq_of(p, act_q, act_k, b);
        if (i >= s.Sq || s.Sk <= 0)
            continue;                            /* padding row */
        int64_t qrow = s.q_off + i;              /* token row of q / weights / q_scale */
        cand *c = (cand *)malloc(sizeof(cand) * (size_t)s.Sk);
        double *qv = (double *)malloc(sizeof(double) * (size_t)p->N1 * p->D);
        double *wv = (double *)malloc(sizeof(double) * (size_t)p->N1);
        double *sq = (double *)malloc(sizeof(double) * (size_t)p->N1);
        double *kv = (double *)malloc(sizeof(double) * (size_t)p->D);
        if (!c || !qv || !wv || !sq || !kv) {
            bad |= 1;
            free(c); free(qv); free(wv); free(sq); free(kv);
            continue;
        }
        for (int h = 0; h < p->N1; ++h) {
            for (int d = 0; d < p->D; ++d)
                qv[h * p->D + d] = load(query, (qrow * p->N1 + h) * p->D + d, p->dtype_qk);
            wv[h] = load(weights, qrow * p->N1 + h, p->dtype_w);
            sq[h] = p->quant ? load(q_scale, qrow * p->N1 + h, p->dtype_scale) : 1.0;
        }
        int64_t nc = 0;
        for (int64_t t = 0; t < s.Sk; ++t) {
            if (!visible(p, s, i, t))
                continue;
            for (int d = 0; d < p->D; ++d)
                kv[d] = load(key, key_elem(p, block_table, s, b, t, d), p->dtype_qk);
            double skt = p->quant ? key_scale(p, k_scale, block_table, s, b, t) : 1.0;
            double acc = 0.0;
            for (int h = 0; h < p->N1; ++h) {
                double logit = 0.0;
                for (int d = 0; d < p->D; ++d)
                    logit += qv[h * p->D + d] * kv[d];
                if (p->quant)
                    logit *= sq[h] * skt;                  /* dequant before ReLU */
                double term;
                if (p->mutation == 1)                      /* planted: ReLU dropped */
                    term = wv[h] * logit;
                else if (p->mutation == 2)                 /* planted: ReLU after weighting */
                    term = fmax(wv[h] * logit, 0.0);
                else
                    term = wv[h] * fmax(logit, 0.0);
                acc += term;
            }
            if (p->mutation == 6 && t == 0)                /* planted: key 0 dropped */
                continue;
            c[nc].s = acc;
            c[nc].t = t;
            ++nc;
            if (scores) scores[r * ld + t] = acc;
        }
        if (p->mutation == 3)
            qsort(c, (size_t)nc, sizeof(cand), cmp_cand_hi_tie);
        else if (p->mutation == 5)
            qsort(c, (size_t)nc, sizeof(cand), cmp_cand_asc);
        else
            qsort(c, (size_t)nc, sizeof(cand), cmp_cand);
        int64_t keep = nc < kk ? nc : kk;
        if (p->init_num > 0 || p->local_num > 0) {
            /* visible keys are t in [0, nv): force t < init_num and t >= nv - local_num */
            int64_t nv = 0;
            for (int64_t t = 0; t < s.Sk; ++t)
                if (visible(p, s, i, t)) ++nv;
            cand *f = (cand *)malloc(sizeof(cand) * (size_t)(nc ? nc : 1));
            cand *o = (cand *)malloc(sizeof(cand) * (size_t)(nc ? nc : 1));
            if (!f || !o) {
                bad |= 1;
                free(f); free(o); free(c); free(qv); free(wv); free(sq); free(kv);
                continue;
            }
            int64_t nf = 0, no = 0;
            /* planted mistake 7: the local window one key short */
            const int64_t lo_local = nv - p->local_num + (p->mutation == 7 ? 1 : 0);
            for (int64_t j = 0; j < nc; ++j) {
                const int forced = c[j].t < p->init_num || c[j].t >= lo_local;
                if (forced) f[nf++] = c[j]; else o[no++] = c[j];
            }
            qsort(o, (size_t)no, sizeof(cand), cmp_cand);          /* the best others */
            int64_t take = keep - nf;
            if (take < 0) take = 0;
            if (take > no) take = no;
            for (int64_t j = 0; j < take; ++j) f[nf++] = o[j];
            qsort(f, (size_t)nf, sizeof(cand), cmp_cand);          /* all kept, in order */
            if (nf > keep) nf = keep;
            memcpy(c, f, sizeof(cand) * (size_t)nf);
            keep = nf;
            free(f);
            free(o);
        }
        for (int64_t j = 0; j < keep; ++j) {
            oi[j] = (int32_t)c[j].t;
            ov[j] = (float)c[j].s;
            if (o64) o64[j] = c[j].s;
        }
        if (nvis) nvis[r] = nc;
        free(c); free(qv); free(wv); free(sq); free(kv);
    }
    return bad ? -1 : 0;
}

int li_oracle_abi_version(void) { return 3; }
