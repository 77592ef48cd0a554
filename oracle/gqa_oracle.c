/*
 * fp64 CPU oracle for causal grouped-query softmax attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
 * CPU-baseline / reference arm may load this code. The product path (the
 * CUDA library) never calls it and shares no code with it.
 *
 * What it computes, written out from the definition with no tiling, no
 * online softmax and no reordering:
 *
 *   o_a = softmax( Q_a K_{g(a)}^T / sqrt(d_h) + M ) V_{g(a)}
 *     -- "注意力家族" (wineandchord.com, attention variants), section 统一记号,
 *        the o_a equation.
 *   g(a) = floor(a / (H_q / H_kv)): consecutive query heads share a KV head
 *     -- "Attention Architecture Evolution", section GQA, group(i) formula;
 *        "注意力家族", section 最小语义实现 (repeat_interleave mapping).
 *   M: causal mask with the suffix offset. Query row i sits at absolute
 *      position (T_k - T_q) + i and sees keys j <= (T_k - T_q) + i; the key at
 *      the query's own position is visible.
 *     -- "注意力家族", section 最小语义实现 (query_pos / key_pos / future) and
 *        section Mask 与增量位置; "A Visual Guide to Attention", section
 *        "Which positions are visible?".
 *   Scale 1/sqrt(D) with D the head dimension (the ABI allows an override).
 *   Optional sliding window w > 0: the query at position p sees only its w most
 *   recent positions, keys j with p - w < j <= p (itself included)
 *     -- "A Visual Guide to Attention", section "Which positions are visible?"
 *        (sliding-window attention keeps the most recent w positions directly
 *        visible); w <= 0 means plain causal attention.
 *
 * Precision: every input is a bf16 value, widened exactly to double; all
 * arithmetic is double; nothing is rounded to a lower precision. Subtracting
 * the row maximum before exp() does not change the mathematical result; it
 * only keeps exp() finite in double. The natural-log LSE (m + ln l) is also
 * returned, for the split-KV merge checks.
 *
 * Layout: q element (b,a,i,d) at b*q_sb + a*q_sh + i*D + d; k and v element
 * (b,h,t,d) at b*k_sb + h*k_sh + t*D + d (likewise v_*). A row id is the flat
 * index (b*H_q + a)*T_q + i. Rows are independent, so any subset can be
 * computed exactly.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline double bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

typedef struct {
    const uint16_t *q, *k, *v;
    int B, Hq, Hkv, Tq, Tk, D;
    long long q_sb, q_sh, k_sb, k_sh, v_sb, v_sh;
    double scale;
    int window; /* <= 0: causal only */
    const long long* rows;
    long long n_rows;
    double* out;
    double* lse;
    long long next; /* shared work counter */
} oracle_job;

/* One output row: o[b,a,i,:] and its log-sum-exp. s holds T_k doubles. */
static void oracle_row(const oracle_job* J, long long row, double* s, double* qd,
                       double* o, double* lse_out) {
    const int D = J->D;
    const long long i = row % J->Tq;
    const long long a = (row / J->Tq) % J->Hq;
    const long long b = row / ((long long)J->Tq * J->Hq);
    const long long group = J->Hq / J->Hkv;       /* H_q / H_kv query heads per KV head */
    const long long g = a / group;                 /* g(a) */
    const long long pos = (long long)(J->Tk - J->Tq) + i; /* absolute query position */

    const uint16_t* qrow = J->q + b * J->q_sb + a * J->q_sh + i * D;
    const uint16_t* kplane = J->k + b * J->k_sb + g * J->k_sh;
    const uint16_t* vplane = J->v + b * J->v_sb + g * J->v_sh;

    for (int d = 0; d < D; ++d) qd[d] = bf16_to_double(qrow[d]);

    /* first visible key: 0 for causal attention, pos - w + 1 inside a window of w */
    const long long first = (J->window > 0 && pos - J->window + 1 > 0) ? pos - J->window + 1 : 0;

    /* scores s_j = scale * <q_i, k_j> for visible keys j = first..pos */
    double m = -INFINITY;
    for (long long j = first; j <= pos; ++j) {
        const uint16_t* krow = kplane + j * D;
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qd[d] * bf16_to_double(krow[d]);
        s[j] = J->scale * acc;
        if (s[j] > m) m = s[j];
    }
    /* softmax weights and normaliser */
    double l = 0.0;
    for (long long j = first; j <= pos; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    /* weighted sum of value rows */
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (long long j = first; j <= pos; ++j) {
        const uint16_t* vrow = vplane + j * D;
        const double w = s[j];
        for (int d = 0; d < D; ++d) o[d] += w * bf16_to_double(vrow[d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    if (lse_out) *lse_out = m + log(l);
}

static void* oracle_worker(void* arg) {
    oracle_job* J = (oracle_job*)arg;
    double* s = (double*)malloc(sizeof(double) * (size_t)J->Tk);
    double* qd = (double*)malloc(sizeof(double) * (size_t)J->D);
    if (!s || !qd) {
        free(s);
        free(qd);
        return (void*)1;
    }
    const long long chunk = 4;
    for (;;) {
        long long r0 = __atomic_fetch_add(&J->next, chunk, __ATOMIC_RELAXED);
        if (r0 >= J->n_rows) break;
        long long r1 = r0 + chunk < J->n_rows ? r0 + chunk : J->n_rows;
        for (long long r = r0; r < r1; ++r)
            oracle_row(J, J->rows[r], s, qd, J->out + r * J->D, J->lse ? J->lse + r : NULL);
    }
    free(s);
    free(qd);
    return NULL;
}

/*
 * Compute n_rows output rows. rows[r] is a flat row id (b*H_q + a)*T_q + i.
 * out is [n_rows][D] doubles; lse is [n_rows] doubles or NULL.
 * scale <= 0 selects 1/sqrt(D). n_threads <= 0 selects one thread.
 * Returns 0 on success, 1 on invalid arguments, 2 on allocation failure.
 */
int gqa_oracle_rows_window(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                           int Hkv, int Tq, int Tk, int D, long long q_sb, long long q_sh,
                           long long k_sb, long long k_sh, long long v_sb, long long v_sh,
                           double scale, int window, const long long* rows, long long n_rows,
                           double* out, double* lse, int n_threads) {
    if (!q || !k || !v || !out || (!rows && n_rows > 0)) return 1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tk <= 0 || D <= 0) return 1;
    if (Hq % Hkv != 0 || Tq > Tk) return 1; /* the pages' asserted preconditions */
    const long long total = (long long)B * Hq * Tq;
    for (long long r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= total) return 1;

    oracle_job J;
    J.q = q; J.k = k; J.v = v;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Tq = Tq; J.Tk = Tk; J.D = D;
    J.q_sb = q_sb; J.q_sh = q_sh; J.k_sb = k_sb; J.k_sh = k_sh; J.v_sb = v_sb; J.v_sh = v_sh;
    J.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)D);
    J.window = window;
    J.rows = rows; J.n_rows = n_rows; J.out = out; J.lse = lse; J.next = 0;

    if (n_threads <= 1) return oracle_worker(&J) ? 2 : 0;
    if (n_threads > 512) n_threads = 512;
    pthread_t th[512];
    int started[512];
    int rc = 0;
    for (int t = 0; t < n_threads; ++t) started[t] = pthread_create(&th[t], NULL, oracle_worker, &J) == 0;
    for (int t = 0; t < n_threads; ++t) {
        if (!started[t]) continue;
        void* ret = NULL;
        pthread_join(th[t], &ret);
        if (ret) rc = 2;
    }
    /* if no thread could start, do the work here */
    int any = 0;
    for (int t = 0; t < n_threads; ++t) any |= started[t];
    if (!any) rc = oracle_worker(&J) ? 2 : 0;
    return rc;
}

/* Plain causal attention (no window). */
int gqa_oracle_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                    int Hkv, int Tq, int Tk, int D, long long q_sb, long long q_sh,
                    long long k_sb, long long k_sh, long long v_sb, long long v_sh, double scale,
                    const long long* rows, long long n_rows, double* out, double* lse,
                    int n_threads) {
    return gqa_oracle_rows_window(q, k, v, B, Hq, Hkv, Tq, Tk, D, q_sb, q_sh, k_sb, k_sh, v_sb, v_sh,
                                  scale, 0, rows, n_rows, out, lse, n_threads);
}

/*
 * Gradients of the same attention, for the training side (fp64, test infrastructure).
 *
 * The pages only say that FlashAttention's backward recomputes the scores, which adds
 * FLOPs ("长上下文与高效注意力：研究账本", section FlashAttention). What it computes is
 * the derivative of the o_a definition above. With P_ij the softmax weights of row i over its
 * visible keys j, s_ij = scale <q_i, k_j>, and dO = dL/dO for a scalar loss L:
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   dS_ij = P_ij (dP_ij - sum_l P_il dP_il)         (softmax Jacobian applied to dP)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 * A KV head's dK and dV sum over every query head a with g(a) = g, and over every row.
 * One (b, g) plane per work item, rows in order, so the fp64 sums are deterministic.
 */
typedef struct {
    const uint16_t *q, *k, *v, *dout;
    int B, Hq, Hkv, Tq, Tk, D;
    long long q_sb, q_sh, k_sb, k_sh, v_sb, v_sh; /* dout uses q's strides */
    double scale;
    int window;
    double *dq, *dk, *dv; /* [B,Hq,Tq,D], [B,Hkv,Tk,D], [B,Hkv,Tk,D], contiguous */
    long long next;
} oracle_bwd_job;

static void oracle_bwd_plane(const oracle_bwd_job* J, long long bg, double* p, double* dp, double* qd,
                             double* dod) {
    const int D = J->D;
    const long long Tk = J->Tk, Tq = J->Tq;
    const long long b = bg / J->Hkv, g = bg % J->Hkv;
    const long long group = J->Hq / J->Hkv;
    const uint16_t* kplane = J->k + b * J->k_sb + g * J->k_sh;
    const uint16_t* vplane = J->v + b * J->v_sb + g * J->v_sh;
    double* dk = J->dk + bg * Tk * D;
    double* dv = J->dv + bg * Tk * D;
    for (long long e = 0; e < Tk * D; ++e) dk[e] = dv[e] = 0.0;
    for (long long a = g * group; a < (g + 1) * group; ++a) {
        for (long long i = 0; i < Tq; ++i) {
            const long long pos = (Tk - Tq) + i;
            const long long first = (J->window > 0 && pos - J->window + 1 > 0) ? pos - J->window + 1 : 0;
            const uint16_t* qrow = J->q + b * J->q_sb + a * J->q_sh + i * D;
            const uint16_t* dorow = J->dout + b * J->q_sb + a * J->q_sh + i * D;
            for (int d = 0; d < D; ++d) {
                qd[d] = bf16_to_double(qrow[d]);
                dod[d] = bf16_to_double(dorow[d]);
            }
            /* P: softmax of the scaled scores over the visible keys */
            double m = -INFINITY;
            for (long long j = first; j <= pos; ++j) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qd[d] * bf16_to_double(kplane[j * D + d]);
                p[j] = J->scale * acc;
                if (p[j] > m) m = p[j];
            }
            double l = 0.0;
            for (long long j = first; j <= pos; ++j) {
                p[j] = exp(p[j] - m);
                l += p[j];
            }
            for (long long j = first; j <= pos; ++j) p[j] /= l;
            /* dP and the row term sum_l P_il dP_il */
            double rowterm = 0.0;
            for (long long j = first; j <= pos; ++j) {
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += dod[d] * bf16_to_double(vplane[j * D + d]);
                dp[j] = acc;
                rowterm += p[j] * dp[j];
            }
            double* dqrow = J->dq + ((b * J->Hq + a) * Tq + i) * D;
            for (int d = 0; d < D; ++d) dqrow[d] = 0.0;
            for (long long j = first; j <= pos; ++j) {
                const double ds = p[j] * (dp[j] - rowterm);
                for (int d = 0; d < D; ++d) {
                    dqrow[d] += J->scale * ds * bf16_to_double(kplane[j * D + d]);
                    dk[j * D + d] += J->scale * ds * qd[d];
                    dv[j * D + d] += p[j] * dod[d];
                }
            }
        }
    }
}

static void* oracle_bwd_worker(void* arg) {
    oracle_bwd_job* J = (oracle_bwd_job*)arg;
    double* p = (double*)malloc(sizeof(double) * (size_t)J->Tk);
    double* dp = (double*)malloc(sizeof(double) * (size_t)J->Tk);
    double* qd = (double*)malloc(sizeof(double) * (size_t)J->D);
    double* dod = (double*)malloc(sizeof(double) * (size_t)J->D);
    void* ret = NULL;
    if (!p || !dp || !qd || !dod) {
        ret = (void*)1;
    } else {
        for (;;) {
            const long long bg = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
            if (bg >= (long long)J->B * J->Hkv) break;
            oracle_bwd_plane(J, bg, p, dp, qd, dod);
        }
    }
    free(p);
    free(dp);
    free(qd);
    free(dod);
    return ret;
}

/*
 * dq [B,Hq,Tq,D], dk and dv [B,Hkv,Tk,D] (doubles, contiguous) of the attention of q over the
 * first Tk keys of k/v, for the output gradient dout (bf16 bits, q's layout).
 * scale <= 0 selects 1/sqrt(D); window as for gqa_oracle_rows_window.
 * Returns 0 on success, 1 on invalid arguments, 2 on allocation failure.
 */
int gqa_oracle_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout, int B,
                   int Hq, int Hkv, int Tq, int Tk, int D, long long q_sb, long long q_sh, long long k_sb,
                   long long k_sh, long long v_sb, long long v_sh, double scale, int window, double* dq,
                   double* dk, double* dv, int n_threads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return 1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Tq <= 0 || Tk <= 0 || D <= 0) return 1;
    if (Hq % Hkv != 0 || Tq > Tk) return 1;
    oracle_bwd_job J;
    J.q = q; J.k = k; J.v = v; J.dout = dout;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Tq = Tq; J.Tk = Tk; J.D = D;
    J.q_sb = q_sb; J.q_sh = q_sh; J.k_sb = k_sb; J.k_sh = k_sh; J.v_sb = v_sb; J.v_sh = v_sh;
    J.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)D);
    J.window = window;
    J.dq = dq; J.dk = dk; J.dv = dv; J.next = 0;
    if (n_threads <= 1) return oracle_bwd_worker(&J) ? 2 : 0;
    if (n_threads > 512) n_threads = 512;
    pthread_t th[512];
    int started[512], any = 0, rc = 0;
    for (int t = 0; t < n_threads; ++t) {
        started[t] = pthread_create(&th[t], NULL, oracle_bwd_worker, &J) == 0;
        any |= started[t];
    }
    for (int t = 0; t < n_threads; ++t) {
        if (!started[t]) continue;
        void* ret = NULL;
        pthread_join(th[t], &ret);
        if (ret) rc = 2;
    }
    if (!any) rc = oracle_bwd_worker(&J) ? 2 : 0;
    return rc;
}
