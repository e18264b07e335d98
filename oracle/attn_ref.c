/*
 * CPU oracle for exact attention: TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline /
 * reference leg load this library. The product path (the CUDA library) never
 * calls it, links it or shares code with it.
 *
 * What it computes is the plain definition of scaled dot-product attention as
 * the FlashAttention pages state it ("FlashAttention (UR)", section "Problem
 * of standard attention": Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V),
 * with the mask added to the scores before the softmax (the fused operation
 * chain in section "Fusing operations into one CUDA kernel" lists masking
 * between Q K^T and the softmax). It is the "standard" implementation those
 * pages contrast with the fused one: every score of a query row is
 * materialised, then the softmax is taken in two passes (max, then sum of
 * exponentials) over the whole row. No tiling, no online rescaling.
 *
 * Grouped / multi-query attention (the FlashAttention-2 extension to MQA named
 * in "FlashAttention (UR)", section "FlashAttention-2 (2023)"): K and V may
 * have Hkv <= H heads, H a multiple of Hkv; query head h attends with K/V head
 * h / (H / Hkv). Hkv == H is ordinary multi-head attention.
 *
 * Fewer queries than keys (Nq <= Nk: the decode / key-value-cache case of
 * "FlashAttention (UR)", section "Specialised solutions"): query row i stands
 * at position i + (Nk - Nq) of the key sequence, so with Nq == Nk the mask is
 * the square one.
 *
 * Readings taken where the pages are silent:
 *   - scale is passed by the caller (1/sqrt(d) in every workload);
 *   - the mask is additive -inf; causal means key j is allowed iff
 *     j <= i + (Nk - Nq) (square when Nq == Nk); key padding masks keys
 *     j >= kv_len[b], and query rows are still computed against the valid keys;
 *   - a row with no allowed key gets O = 0 and lse = -inf;
 *   - lse_i = ln sum_j exp(s_ij), natural log, scale included.
 *
 * Arithmetic: IEEE fp64 throughout. bf16 inputs are widened exactly (a bf16
 * value is the top 16 bits of an fp32, and fp32 -> fp64 is exact).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

static double bf16_to_f64(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Is key j visible to query row i (which stands at key position i + off)? */
static int key_allowed(int i, int j, int causal, int kv_lim, int off)
{
    if (j >= kv_lim) return 0;
    if (causal && j > i + off) return 0;
    return 1;
}

/*
 * One query row against one head's K and V (row-major [N][d] fp64).
 * srow is caller scratch of N doubles: the materialised score row.
 */
static void attn_one_row(const double *qi, const double *K, const double *V,
                         int N, int d, double scale, int i, int causal,
                         int kv_lim, int off, double *srow, double *oi, double *lse_i)
{
    /* s_ij = scale * <q_i, k_j> + mask_ij, over the N keys */
    for (int j = 0; j < N; ++j) {
        if (!key_allowed(i, j, causal, kv_lim, off)) {
            srow[j] = -INFINITY;
            continue;
        }
        const double *kj = K + (size_t)j * d;
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += qi[t] * kj[t];
        srow[j] = scale * dot;
    }
    /* pass 1: row max */
    double m = -INFINITY;
    for (int j = 0; j < N; ++j)
        if (srow[j] > m) m = srow[j];
    for (int t = 0; t < d; ++t) oi[t] = 0.0;
    if (m == -INFINITY) { /* no visible key */
        *lse_i = -INFINITY;
        return;
    }
    /* pass 2: sum of exponentials, then the normaliser */
    double sum = 0.0;
    for (int j = 0; j < N; ++j)
        if (srow[j] != -INFINITY) sum += exp(srow[j] - m);
    double lse = m + log(sum);
    /* O_i = sum_j softmax_ij * v_j */
    for (int j = 0; j < N; ++j) {
        if (srow[j] == -INFINITY) continue;
        double p = exp(srow[j] - lse);
        const double *vj = V + (size_t)j * d;
        for (int t = 0; t < d; ++t) oi[t] += p * vj[t];
    }
    *lse_i = lse;
}

static int check_args(int B, int H, int N, int d, double scale, int causal)
{
    if (B < 0 || H < 0 || N < 0 || d <= 0) return ORACLE_EINVAL;
    if (!(scale == scale) || isinf(scale)) return ORACLE_EINVAL;
    if (causal != 0 && causal != 1) return ORACLE_EINVAL;
    return ORACLE_OK;
}

/*
 * Shared driver. Inputs are either fp64 (qd/kd/vd) or bf16 bit patterns
 * (qb/kb/vb); exactly one set is non-null. `rows` (nullable) selects which
 * query rows of every head to compute; outputs are then [B,H,nrows,d] and
 * [B,H,nrows]. With rows == NULL, nrows must equal N and all rows are done.
 */
static int attn_driver(const double *qd, const double *kd, const double *vd,
                       const uint16_t *qb, const uint16_t *kb, const uint16_t *vb,
                       double *o, double *lse, int B, int H, int Hkv, int Nq, int N, int d,
                       double scale, int causal, const int32_t *kv_len,
                       const int32_t *rows, int nrows, int nthreads)
{
    int rc = check_args(B, H, N, d, scale, causal);
    if (rc) return rc;
    if (Nq < 0 || Nq > N) return ORACLE_EINVAL;
    if (B == 0 || H == 0) return ORACLE_OK;
    if (Hkv <= 0 || Hkv > H || H % Hkv != 0) return ORACLE_EINVAL;
    if (nrows < 0 || (rows == NULL && nrows != Nq)) return ORACLE_EINVAL;
    if (rows)
        for (int r = 0; r < nrows; ++r)
            if (rows[r] < 0 || rows[r] >= Nq) return ORACLE_EINVAL;
    if (B == 0 || H == 0 || nrows == 0) return ORACLE_OK;
    if (N == 0) return ORACLE_EINVAL; /* rows must index into N */

    const size_t head = (size_t)N * d;      /* one K or V head */
    const size_t qhead = (size_t)Nq * d;    /* one Q head */
    const int off = N - Nq;                 /* key position of query row 0 */
    const int widen = (qb != NULL);
    double *Kh = NULL, *Vh = NULL, *Qh = NULL;
    if (widen) {
        Kh = (double *)malloc(head * sizeof(double));
        Vh = (double *)malloc(head * sizeof(double));
        Qh = (double *)malloc((qhead ? qhead : 1) * sizeof(double));
        if (!Kh || !Vh || !Qh) {
            free(Kh); free(Vh); free(Qh);
            return ORACLE_ENOMEM;
        }
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int err = ORACLE_OK;
    for (int b = 0; b < B; ++b) {
        int kv_lim = N;
        if (kv_len) {
            kv_lim = kv_len[b];
            if (kv_lim < 0) kv_lim = 0;
            if (kv_lim > N) kv_lim = N;
        }
        for (int h = 0; h < H; ++h) {
            const size_t base = ((size_t)b * H + h) * qhead;                 /* Q */
            const size_t kvbase = ((size_t)b * Hkv + h / (H / Hkv)) * head;  /* K, V */
            const double *Q, *K, *V;
            if (widen) {
                for (size_t e = 0; e < qhead; ++e) Qh[e] = bf16_to_f64(qb[base + e]);
                for (size_t e = 0; e < head; ++e) {
                    Kh[e] = bf16_to_f64(kb[kvbase + e]);
                    Vh[e] = bf16_to_f64(vb[kvbase + e]);
                }
                Q = Qh; K = Kh; V = Vh;
            } else {
                Q = qd + base; K = kd + kvbase; V = vd + kvbase;
            }
            double *o_bh = o + ((size_t)b * H + h) * (size_t)nrows * d;
            double *l_bh = lse + ((size_t)b * H + h) * (size_t)nrows;
#pragma omp parallel
            {
                double *srow = (double *)malloc((size_t)N * sizeof(double));
                if (!srow) {
#pragma omp atomic write
                    err = ORACLE_ENOMEM;
                } else {
#pragma omp for schedule(dynamic, 4)
                    for (int r = 0; r < nrows; ++r) {
                        int i = rows ? rows[r] : r;
                        attn_one_row(Q + (size_t)i * d, K, V, N, d, scale, i,
                                     causal, kv_lim, off, srow,
                                     o_bh + (size_t)r * d, l_bh + r);
                    }
                    free(srow);
                }
            }
        }
    }
    free(Kh); free(Vh); free(Qh);
    return err;
}

/* General form: q, o [B,H,Nq,d]; k, v [B,Hkv,Nk,d], Nq <= Nk (query row i at
 * key position i + Nk - Nq). Either fp64 inputs (qd/kd/vd) or bf16 bits
 * (qb/kb/vb); rows (nullable) as in attn_driver, indices into Nq. */
int oracle_attn_general(const double *qd, const double *kd, const double *vd,
                        const uint16_t *qb, const uint16_t *kb, const uint16_t *vb,
                        double *o, double *lse, int B, int H, int Hkv, int Nq, int Nk,
                        int d, double scale, int causal, const int32_t *kv_len,
                        const int32_t *rows, int nrows, int nthreads)
{
    const int fp64 = qd && kd && vd, bits = qb && kb && vb;
    if (fp64 == bits || !o || !lse) return ORACLE_EINVAL;
    return attn_driver(qd, kd, vd, qb, kb, vb, o, lse, B, H, Hkv, Nq, Nk, d, scale,
                       causal, kv_len, rows, nrows, nthreads);
}

/*
 * Backward pass: gradients of the attention above for a scalar loss L, given
 * dO = dL/dO. The pages report training speed-ups ("FlashAttention (UR)",
 * section "Experimental results"), which need these gradients, but state no
 * backward algorithm; this is the exact gradient of the forward definition by
 * the chain rule through the row softmax, evaluated one query row at a time:
 *   P_ij  = softmax_j(s_ij)                      (0 for hidden keys)
 *   dV_j += P_ij dO_i                            (dV = P^T dO)
 *   dP_ij = <dO_i, v_j>                          (dP = dO V^T)
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)                   (softmax Jacobian)
 *   dQ_i  = scale sum_j dS_ij k_j                (dQ = scale dS K)
 *   dK_j += scale dS_ij q_i                      (dK = scale dS^T Q)
 * A K/V head shared by a group of query heads collects the sum over the
 * group. A row with no visible key has P = 0 and contributes nothing.
 * q, dO, dq: [B,H,N,d]; k, v, dk, dv: [B,Hkv,N,d] (square: Nq == Nk == N).
 * Inputs fp64 (qd..dod) or bf16 bits (qb..dob), exactly one set non-null.
 */
/*
 * Row i's softmax weights P_ij (0 for hidden keys) into prow, dP_ij =
 * <dO_i, v_j> into dprow (0 where P_ij = 0), and D_i = sum_j P_ij dP_ij as the
 * return value. Returns 0 with prow and dprow all 0 if row i sees no key.
 */
static double bwd_row_p_dp(const double *qi, const double *doi, const double *K,
                           const double *V, int N, int d, double scale, int i, int causal,
                           int kv_lim, double *prow, double *dprow)
{
    double m = -INFINITY;
    for (int j = 0; j < N; ++j) {
        if (!key_allowed(i, j, causal, kv_lim, 0)) {
            prow[j] = -INFINITY;
            continue;
        }
        const double *krow = K + (size_t)j * d;
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += qi[t] * krow[t];
        prow[j] = scale * dot;
        if (prow[j] > m) m = prow[j];
    }
    if (m == -INFINITY) {
        for (int j = 0; j < N; ++j) prow[j] = dprow[j] = 0.0;
        return 0.0;
    }
    double sum = 0.0;
    for (int j = 0; j < N; ++j)
        if (prow[j] != -INFINITY) sum += exp(prow[j] - m);
    for (int j = 0; j < N; ++j)
        prow[j] = (prow[j] == -INFINITY) ? 0.0 : exp(prow[j] - m) / sum;
    double D = 0.0;
    for (int j = 0; j < N; ++j) {
        if (prow[j] == 0.0) {
            dprow[j] = 0.0;
            continue;
        }
        const double *vrow = V + (size_t)j * d;
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += doi[t] * vrow[t];
        dprow[j] = dot;
        D += prow[j] * dot;
    }
    return D;
}

static void bwd_one_row(const double *qi, const double *doi, const double *K, const double *V,
                        int N, int d, double scale, int i, int causal, int kv_lim,
                        double *prow, double *dprow, double *dqi, double *dK, double *dV)
{
    const double D = bwd_row_p_dp(qi, doi, K, V, N, d, scale, i, causal, kv_lim, prow, dprow);
    for (int t = 0; t < d; ++t) dqi[t] = 0.0;
    for (int j = 0; j < N; ++j) {
        const double pij = prow[j];
        if (pij == 0.0) continue;
        const double ds = pij * (dprow[j] - D);
        const double *krow = K + (size_t)j * d;
        double *dkj = dK + (size_t)j * d;
        double *dvj = dV + (size_t)j * d;
        for (int t = 0; t < d; ++t) {
            dqi[t] += scale * ds * krow[t];
            dkj[t] += scale * ds * qi[t];
            dvj[t] += pij * doi[t];
        }
    }
}

int oracle_attn_bwd(const double *qd, const double *kd, const double *vd, const double *dod,
                    const uint16_t *qb, const uint16_t *kb, const uint16_t *vb,
                    const uint16_t *dob, double *dq, double *dk, double *dv, int B, int H,
                    int Hkv, int N, int d, double scale, int causal, const int32_t *kv_len,
                    int nthreads)
{
    const int fp64 = qd && kd && vd && dod, bits = qb && kb && vb && dob;
    if (fp64 == bits || !dq || !dk || !dv) return ORACLE_EINVAL;
    int rc = check_args(B, H, N, d, scale, causal);
    if (rc) return rc;
    if (B == 0 || H == 0 || N == 0) return ORACLE_OK;
    if (Hkv <= 0 || Hkv > H || H % Hkv != 0) return ORACLE_EINVAL;
    const int G = H / Hkv;
    const size_t head = (size_t)N * d;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int err = ORACLE_OK;
    /* one (batch, K/V head) group per iteration: its dK, dV sums stay private */
#pragma omp parallel for schedule(dynamic, 1)
    for (int g = 0; g < B * Hkv; ++g) {
        const int b = g / Hkv, hk = g % Hkv;
        int kv_lim = N;
        if (kv_len) {
            kv_lim = kv_len[b];
            if (kv_lim < 0) kv_lim = 0;
            if (kv_lim > N) kv_lim = N;
        }
        double *buf = (double *)malloc((4 * head + 2 * (size_t)N) * sizeof(double));
        if (!buf) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
            continue;
        }
        double *K = buf, *V = buf + head, *Q = buf + 2 * head, *dO = buf + 3 * head;
        double *prow = buf + 4 * head, *dprow = prow + N;
        const size_t kvbase = (size_t)g * head;
        for (size_t e = 0; e < head; ++e) {
            K[e] = bits ? bf16_to_f64(kb[kvbase + e]) : kd[kvbase + e];
            V[e] = bits ? bf16_to_f64(vb[kvbase + e]) : vd[kvbase + e];
        }
        double *dK = dk + kvbase, *dV = dv + kvbase;
        for (size_t e = 0; e < head; ++e) dK[e] = dV[e] = 0.0;
        for (int hq = hk * G; hq < (hk + 1) * G; ++hq) {
            const size_t qbase = ((size_t)b * H + hq) * head;
            for (size_t e = 0; e < head; ++e) {
                Q[e] = bits ? bf16_to_f64(qb[qbase + e]) : qd[qbase + e];
                dO[e] = bits ? bf16_to_f64(dob[qbase + e]) : dod[qbase + e];
            }
            for (int i = 0; i < N; ++i)
                bwd_one_row(Q + (size_t)i * d, dO + (size_t)i * d, K, V, N, d, scale, i, causal,
                            kv_lim, prow, dprow, dq + qbase + (size_t)i * d, dK, dV);
        }
        free(buf);
    }
    return err;
}

/*
 * dQ of selected query rows only (same definition as oracle_attn_bwd, which
 * dQ row i depends on through row i alone: its P, dP and D). For checks at
 * sizes where the full backward is out of reach. dq_rows: [B,H,nrows,d].
 * bf16 inputs only.
 */
int oracle_attn_bwd_dq_rows(const uint16_t *qb, const uint16_t *kb, const uint16_t *vb,
                            const uint16_t *dob, double *dq_rows, int B, int H, int Hkv, int N,
                            int d, double scale, int causal, const int32_t *kv_len,
                            const int32_t *rows, int nrows, int nthreads)
{
    if (!qb || !kb || !vb || !dob || !dq_rows || !rows) return ORACLE_EINVAL;
    int rc = check_args(B, H, N, d, scale, causal);
    if (rc) return rc;
    if (B == 0 || H == 0 || N == 0 || nrows == 0) return ORACLE_OK;
    if (Hkv <= 0 || Hkv > H || H % Hkv != 0 || nrows < 0) return ORACLE_EINVAL;
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_EINVAL;
    const size_t head = (size_t)N * d;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    int err = ORACLE_OK;
#pragma omp parallel
    {
        /* per thread: one K/V head, and scratch for the dK/dV sums it discards */
        double *buf = (double *)malloc((4 * head + 4 * (size_t)d + 2 * (size_t)N) * sizeof(double));
        if (!buf) {
#pragma omp atomic write
            err = ORACLE_ENOMEM;
        } else {
            double *K = buf, *V = buf + head, *dKs = buf + 2 * head, *dVs = buf + 3 * head;
            double *qi = buf + 4 * head, *doi = qi + d;
            double *prow = doi + 2 * (size_t)d, *dprow = prow + N;
            int loaded = -1;
#pragma omp for schedule(dynamic, 1)
            for (int bh = 0; bh < B * H; ++bh) {
                const int b = bh / H, h = bh % H;
                const int g = b * Hkv + h / (H / Hkv);
                int kv_lim = N;
                if (kv_len) {
                    kv_lim = kv_len[b];
                    if (kv_lim < 0) kv_lim = 0;
                    if (kv_lim > N) kv_lim = N;
                }
                if (g != loaded) {
                    for (size_t e = 0; e < head; ++e) {
                        K[e] = bf16_to_f64(kb[(size_t)g * head + e]);
                        V[e] = bf16_to_f64(vb[(size_t)g * head + e]);
                    }
                    loaded = g;
                }
                for (int r = 0; r < nrows; ++r) {
                    const int i = rows[r];
                    const size_t qoff = ((size_t)bh * N + i) * d;
                    for (int t = 0; t < d; ++t) {
                        qi[t] = bf16_to_f64(qb[qoff + t]);
                        doi[t] = bf16_to_f64(dob[qoff + t]);
                    }
                    for (size_t e = 0; e < head; ++e) dKs[e] = dVs[e] = 0.0;
                    bwd_one_row(qi, doi, K, V, N, d, scale, i, causal, kv_lim, prow, dprow,
                                dq_rows + ((size_t)bh * nrows + r) * d, dKs, dVs);
                }
            }
            free(buf);
        }
    }
    return err;
}

/*
 * dK and dV of selected key rows only (same definition as oracle_attn_bwd:
 * dK_j = scale sum_i dS_ij q_i and dV_j = sum_i P_ij dO_i over every query
 * row i of every query head of the K/V head's group). Key row j needs P_ij,
 * dP_ij and D_i of every row i, so each row's softmax and D are still
 * computed in full; only the accumulation is restricted to the selected keys.
 * For checks at sizes where the full backward is out of reach. dk_rows,
 * dv_rows: [B,Hkv,nrows,d]. bf16 inputs only.
 */
int oracle_attn_bwd_kv_rows(const uint16_t *qb, const uint16_t *kb, const uint16_t *vb,
                            const uint16_t *dob, double *dk_rows, double *dv_rows, int B, int H,
                            int Hkv, int N, int d, double scale, int causal,
                            const int32_t *kv_len, const int32_t *rows, int nrows, int nthreads)
{
    if (!qb || !kb || !vb || !dob || !dk_rows || !dv_rows || !rows) return ORACLE_EINVAL;
    int rc = check_args(B, H, N, d, scale, causal);
    if (rc) return rc;
    if (B == 0 || H == 0 || N == 0 || nrows == 0) return ORACLE_OK;
    if (Hkv <= 0 || Hkv > H || H % Hkv != 0 || nrows < 0) return ORACLE_EINVAL;
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_EINVAL;
    const int G = H / Hkv;
    const size_t head = (size_t)N * d, sel = (size_t)nrows * d;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    double *K = (double *)malloc(4 * head * sizeof(double));
    if (!K) return ORACLE_ENOMEM;
    double *V = K + head, *Q = K + 2 * head, *dO = K + 3 * head;
    int err = ORACLE_OK;
    for (int g = 0; g < B * Hkv && err == ORACLE_OK; ++g) {
        const int b = g / Hkv, hk = g % Hkv;
        int kv_lim = N;
        if (kv_len) {
            kv_lim = kv_len[b];
            if (kv_lim < 0) kv_lim = 0;
            if (kv_lim > N) kv_lim = N;
        }
        for (size_t e = 0; e < head; ++e) {
            K[e] = bf16_to_f64(kb[(size_t)g * head + e]);
            V[e] = bf16_to_f64(vb[(size_t)g * head + e]);
        }
        double *dKr = dk_rows + (size_t)g * sel, *dVr = dv_rows + (size_t)g * sel;
        for (size_t e = 0; e < sel; ++e) dKr[e] = dVr[e] = 0.0;
        for (int hq = hk * G; hq < (hk + 1) * G; ++hq) {
            const size_t qbase = ((size_t)b * H + hq) * head;
            for (size_t e = 0; e < head; ++e) {
                Q[e] = bf16_to_f64(qb[qbase + e]);
                dO[e] = bf16_to_f64(dob[qbase + e]);
            }
#pragma omp parallel
            {
                /* per thread: one row's P and dP, and private sums for the selected keys */
                double *buf = (double *)malloc((2 * (size_t)N + 2 * sel) * sizeof(double));
                if (!buf) {
#pragma omp atomic write
                    err = ORACLE_ENOMEM;
                } else {
                    double *prow = buf, *dprow = buf + N, *aK = buf + 2 * (size_t)N, *aV = aK + sel;
                    for (size_t e = 0; e < 2 * sel; ++e) aK[e] = 0.0;
#pragma omp for schedule(dynamic, 16)
                    for (int i = 0; i < N; ++i) {
                        const double *qi = Q + (size_t)i * d, *doi = dO + (size_t)i * d;
                        const double D = bwd_row_p_dp(qi, doi, K, V, N, d, scale, i, causal,
                                                      kv_lim, prow, dprow);
                        for (int r = 0; r < nrows; ++r) {
                            const double pij = prow[rows[r]];
                            if (pij == 0.0) continue;
                            const double ds = pij * (dprow[rows[r]] - D);
                            for (int t = 0; t < d; ++t) {
                                aK[(size_t)r * d + t] += scale * ds * qi[t];
                                aV[(size_t)r * d + t] += pij * doi[t];
                            }
                        }
                    }
#pragma omp critical
                    for (size_t e = 0; e < sel; ++e) {
                        dKr[e] += aK[e];
                        dVr[e] += aV[e];
                    }
                    free(buf);
                }
            }
        }
    }
    free(K);
    return err;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
