/*
 * attn_oracle.c -- fp64 CPU reference for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may call this file.  It shares no code, header or constant
 * with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes is the plain definition of attention, one query row at a
 * time, over the full score row (no tiling, no online softmax):
 *
 *   s_ij  = scale * <q_i, k_j>                    for every key j < Sk
 *   allowed(i, j) = !causal || j <= i + (Sk - Sq)  (causal mask, bottom-right aligned)
 *   M_i   = max_{allowed j} s_ij
 *   l_i   = sum_{allowed j} exp(s_ij - M_i)
 *   P_ij  = exp(s_ij - M_i) / l_i
 *   O_i   = sum_j P_ij v_j
 *   LSE_i = M_i + ln(l_i)
 *
 * ("FlashAttention 4: Snellere, Geheugenefficiente Aandacht voor LLM's",
 * introduction and "Slimmere Online Softmax-herwaardering": attention is
 * softmax(Q K^T) V, and the tiled method keeps a running max and sum per query
 * row so that it reaches this same result without storing the score matrix.)
 *
 * Backward, given dO (explicit chain rule of the definition above):
 *   dP_ij = <dO_i, v_j>
 *   D_i   = sum_j P_ij dP_ij          (from P and dP, not from O)
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_{h in group} sum_i dS_ij q_i
 *   dV_j  = sum_{h in group} sum_i P_ij dO_i
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - tensors are [batch, seq, heads, head_dim] ("h3-blackwell-runtime/FLASH4.md",
 *     section "API": the adapter calls the kernel in that native layout);
 *   - grouped-query heads are contiguous: query head h reads key/value head
 *     h / (Hq / Hkv);
 *   - LSE is the natural-log log-sum-exp of the scaled scores, [B, Hq, Sq];
 *   - a row with no allowed key (causal with Sq > Sk) has O = 0, LSE = -inf and
 *     zero gradients.
 *
 * Inputs are the 16-bit tensors handed to the GPU (bf16 or fp16), widened
 * exactly to double here (float64 inputs are also accepted, for the
 * finite-difference tests).  All arithmetic is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_BF16 = 0, ORACLE_FP16 = 1, ORACLE_F64 = 2 };

/* Exact widening of one 16-bit value to double. */
static double widen16(uint16_t bits, int dtype)
{
    if (dtype == ORACLE_BF16) {
        uint32_t w = (uint32_t)bits << 16;
        float f;
        memcpy(&f, &w, sizeof f);
        return (double)f;
    }
    /* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
    int sign = (bits >> 15) & 1;
    int e = (bits >> 10) & 0x1f;
    int m = bits & 0x3ff;
    double r;
    if (e == 0)
        r = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        r = m ? NAN : INFINITY;
    else
        r = ldexp((double)(m + 1024), e - 25);     /* (1 + m/1024) * 2^(e-15) */
    return sign ? -r : r;
}

typedef struct {
    const void *q, *k, *v, *dout;
    int dtype, B, Sq, Sk, Hq, Hkv, d, causal;
    double scale;
} problem;

/* Element `idx` of an input array, as double (16-bit inputs are widened exactly;
 * float64 inputs exist so that finite-difference tests can perturb them). */
static double elem(const void* base, int64_t idx, int dtype)
{
    if (dtype == ORACLE_F64) return ((const double*)base)[idx];
    return widen16(((const uint16_t*)base)[idx], dtype);
}
static double qv(const problem* p, int b, int i, int h, int c)
{
    return elem(p->q, (((int64_t)b * p->Sq + i) * p->Hq + h) * p->d + c, p->dtype);
}
static double kv_k(const problem* p, int b, int j, int g, int c)
{
    return elem(p->k, (((int64_t)b * p->Sk + j) * p->Hkv + g) * p->d + c, p->dtype);
}
static double kv_v(const problem* p, int b, int j, int g, int c)
{
    return elem(p->v, (((int64_t)b * p->Sk + j) * p->Hkv + g) * p->d + c, p->dtype);
}
static double dov(const problem* p, int b, int i, int h, int c)
{
    return elem(p->dout, (((int64_t)b * p->Sq + i) * p->Hq + h) * p->d + c, p->dtype);
}

static int allowed(const problem* p, int i, int j)
{
    return !p->causal || (int64_t)j <= (int64_t)i + (p->Sk - p->Sq);
}

static int kv_head(const problem* p, int h) { return h / (p->Hq / p->Hkv); }

/* s_ij for every key j of row (b, h, i); masked entries are -inf. */
static void score_row(const problem* p, int b, int h, int i, double* s)
{
    int g = kv_head(p, h);
    for (int j = 0; j < p->Sk; ++j) {
        if (!allowed(p, i, j)) {
            s[j] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int c = 0; c < p->d; ++c)
            acc += qv(p, b, i, h, c) * kv_k(p, b, j, g, c);
        s[j] = p->scale * acc;
    }
}

/* Row max M_i and row sum l_i of exp(s_ij - M_i); l = 0 when no key is allowed. */
static void row_max_sum(const problem* p, const double* s, double* M, double* l)
{
    double m = -INFINITY;
    for (int j = 0; j < p->Sk; ++j)
        if (s[j] > m) m = s[j];
    double sum = 0.0;
    if (m != -INFINITY)
        for (int j = 0; j < p->Sk; ++j)
            if (s[j] != -INFINITY) sum += exp(s[j] - m);
    *M = m;
    *l = sum;
}

/* P_ij for the whole row (0 for masked keys or an empty row). */
static void prob_row(const problem* p, const double* s, double M, double l, double* P)
{
    for (int j = 0; j < p->Sk; ++j)
        P[j] = (l > 0.0 && s[j] != -INFINITY) ? exp(s[j] - M) / l : 0.0;
}

/* dP_ij = <dO_i, v_j> for every key j. */
static void dp_row(const problem* p, int b, int h, int i, double* dP)
{
    int g = kv_head(p, h);
    for (int j = 0; j < p->Sk; ++j) {
        double acc = 0.0;
        for (int c = 0; c < p->d; ++c)
            acc += dov(p, b, i, h, c) * kv_v(p, b, j, g, c);
        dP[j] = acc;
    }
}

static int check_problem(const problem* p)
{
    if (p->B < 1 || p->Sq < 1 || p->Sk < 1 || p->Hq < 1 || p->Hkv < 1 || p->d < 1) return 1;
    if (p->Hq % p->Hkv) return 1;
    if (p->dtype != ORACLE_BF16 && p->dtype != ORACLE_FP16 && p->dtype != ORACLE_F64) return 1;
    return 0;
}

static int row_in_range(const problem* p, const int64_t* r, int nheads, int len)
{
    return r[0] >= 0 && r[0] < p->B && r[1] >= 0 && r[1] < nheads && r[2] >= 0 && r[2] < len;
}

/*
 * Forward for a list of query rows.  rows: nrows triples (b, h, i).
 * o: nrows x d, lse: nrows.  Returns 0 on success.
 */
int fa_oracle_fwd(const void* q, const void* k, const void* v, int dtype,
                  int B, int Sq, int Sk, int Hq, int Hkv, int d, int causal, double scale,
                  const int64_t* rows, int64_t nrows, double* o, double* lse)
{
    problem p = {q, k, v, NULL, dtype, B, Sq, Sk, Hq, Hkv, d, causal, scale};
    if (check_problem(&p)) return 1;
    for (int64_t r = 0; r < nrows; ++r)
        if (!row_in_range(&p, rows + 3 * r, Hq, Sq)) return 2;
    int bad = 0;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * Sk);
        double* P = (double*)malloc(sizeof(double) * Sk);
        {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                if (!s || !P) {
#pragma omp atomic write
                    bad = 3;
                    continue;
                }
                int b = (int)rows[3 * r], h = (int)rows[3 * r + 1], i = (int)rows[3 * r + 2];
                int g = kv_head(&p, h);
                double M, l;
                score_row(&p, b, h, i, s);
                row_max_sum(&p, s, &M, &l);
                prob_row(&p, s, M, l, P);
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < Sk; ++j)
                        if (P[j] != 0.0) acc += P[j] * kv_v(&p, b, j, g, c);
                    o[r * d + c] = acc;
                }
                lse[r] = (l > 0.0) ? M + log(l) : -INFINITY;
            }
        }
        free(s);
        free(P);
    }
    return bad;
}

/*
 * Backward.
 *   qrows  (nq triples b, h, i):      dq (nq x d) and D (nq) for those query rows.
 *   kvrows (nkv triples b, hkv, j):   dk, dv (nkv x d) for those key rows, each a full
 *                                     sum over every query row of every query head of
 *                                     the group.
 * Either list may be empty (pass n = 0).  Returns 0 on success.
 */
int fa_oracle_bwd(const void* q, const void* k, const void* v, const void* dout,
                  int dtype, int B, int Sq, int Sk, int Hq, int Hkv, int d, int causal,
                  double scale, const int64_t* qrows, int64_t nq, double* dq, double* Dout,
                  const int64_t* kvrows, int64_t nkv, double* dk, double* dv)
{
    problem p = {q, k, v, dout, dtype, B, Sq, Sk, Hq, Hkv, d, causal, scale};
    if (check_problem(&p)) return 1;
    for (int64_t r = 0; r < nq; ++r)
        if (!row_in_range(&p, qrows + 3 * r, Hq, Sq)) return 2;
    for (int64_t r = 0; r < nkv; ++r)
        if (!row_in_range(&p, kvrows + 3 * r, Hkv, Sk)) return 2;
    int bad = 0;

    /* dQ rows: everything they need is local to the row. */
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * Sk);
        double* P = (double*)malloc(sizeof(double) * Sk);
        double* dP = (double*)malloc(sizeof(double) * Sk);
        {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nq; ++r) {
                if (!s || !P || !dP) {
#pragma omp atomic write
                    bad = 3;
                    continue;
                }
                int b = (int)qrows[3 * r], h = (int)qrows[3 * r + 1], i = (int)qrows[3 * r + 2];
                int g = kv_head(&p, h);
                double M, l, D = 0.0;
                score_row(&p, b, h, i, s);
                row_max_sum(&p, s, &M, &l);
                prob_row(&p, s, M, l, P);
                dp_row(&p, b, h, i, dP);
                for (int j = 0; j < Sk; ++j) D += P[j] * dP[j];
                if (Dout) Dout[r] = D;
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < Sk; ++j)
                        if (P[j] != 0.0) acc += P[j] * (dP[j] - D) * kv_k(&p, b, j, g, c);
                    dq[r * d + c] = scale * acc;
                }
            }
        }
        free(s);
        free(P);
        free(dP);
    }
    if (bad || nkv == 0) return bad;

    /* dK / dV rows need M_i, l_i and D_i of every query row of the group's heads. */
    int G = Hq / Hkv;
    unsigned char* need = (unsigned char*)calloc((size_t)B * Hkv, 1);
    double* Ms = (double*)malloc(sizeof(double) * (size_t)B * Hq * Sq);
    double* Ls = (double*)malloc(sizeof(double) * (size_t)B * Hq * Sq);
    double* Ds = (double*)malloc(sizeof(double) * (size_t)B * Hq * Sq);
    if (!need || !Ms || !Ls || !Ds) {
        free(need); free(Ms); free(Ls); free(Ds);
        return 3;
    }
    for (int64_t r = 0; r < nkv; ++r) need[kvrows[3 * r] * Hkv + kvrows[3 * r + 1]] = 1;
    int64_t nstat = (int64_t)B * Hq * Sq;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * Sk);
        double* P = (double*)malloc(sizeof(double) * Sk);
        double* dP = (double*)malloc(sizeof(double) * Sk);
        {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = 0; t < nstat; ++t) {
                if (!s || !P || !dP) {
#pragma omp atomic write
                    bad = 3;
                    continue;
                }
                int b = (int)(t / ((int64_t)Hq * Sq));
                int h = (int)((t / Sq) % Hq);
                int i = (int)(t % Sq);
                if (!need[b * Hkv + kv_head(&p, h)]) continue;
                double M, l, D = 0.0;
                score_row(&p, b, h, i, s);
                row_max_sum(&p, s, &M, &l);
                prob_row(&p, s, M, l, P);
                dp_row(&p, b, h, i, dP);
                for (int j = 0; j < Sk; ++j) D += P[j] * dP[j];
                Ms[t] = M;
                Ls[t] = l;
                Ds[t] = D;
            }
        }
        free(s);
        free(P);
        free(dP);
    }
    if (!bad) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t r = 0; r < nkv; ++r) {
            int b = (int)kvrows[3 * r], g = (int)kvrows[3 * r + 1], j = (int)kvrows[3 * r + 2];
            double* dkr = dk + r * d;
            double* dvr = dv + r * d;
            for (int c = 0; c < d; ++c) dkr[c] = dvr[c] = 0.0;
            for (int hh = 0; hh < G; ++hh) {
                int h = g * G + hh;
                for (int i = 0; i < Sq; ++i) {
                    int64_t t = ((int64_t)b * Hq + h) * Sq + i;
                    if (!allowed(&p, i, j) || !(Ls[t] > 0.0)) continue;
                    double sij = 0.0, dpij = 0.0;
                    for (int c = 0; c < d; ++c) {
                        sij += qv(&p, b, i, h, c) * kv_k(&p, b, j, g, c);
                        dpij += dov(&p, b, i, h, c) * kv_v(&p, b, j, g, c);
                    }
                    double P = exp(scale * sij - Ms[t]) / Ls[t];
                    double dS = P * (dpij - Ds[t]);
                    for (int c = 0; c < d; ++c) {
                        dvr[c] += P * dov(&p, b, i, h, c);
                        dkr[c] += scale * dS * qv(&p, b, i, h, c);
                    }
                }
            }
        }
    }
    free(need);
    free(Ms);
    free(Ls);
    free(Ds);
    return bad;
}

/* Number of threads the OpenMP runtime will use (reported beside CPU timings). */
int fa_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
