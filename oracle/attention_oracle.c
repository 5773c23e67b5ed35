/*
 * Plain fp64 CPU oracle for exact scaled-dot-product attention and its gradient.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file; only the test-suite, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (written out from the definition, not from any blocked algorithm):
 *
 *   The method is exact: "FlashAttention1" Q&A page, question "key algorithmic
 *   innovations" (it keeps mathematical equivalence with standard attention), and the
 *   "flash attention ... deep dive" page, section "Algorithm behind the article" (the
 *   blocked result is the real answer, not an approximation).  So the oracle is the
 *   standard attention of that deep-dive page, Steps 1-3 (S = Q K', row softmax,
 *   output = softmax(S) V), evaluated one query row at a time in fp64:
 *
 *     g      = Hq / Hkv, kv(h) = floor(h / g)          (grouped-query heads share K/V)
 *     J(i)   = {0..N-1}, or {0..i} when causal          (top-left causal mask), or, for
 *              local attention with a key window, {j : i - left <= j <= i + right}
 *     s_ij   = scale * <q_i, k_j>,  j in J(i)
 *     m_i    = max_j s_ij,  l_i = sum_j exp(s_ij - m_i)
 *     LSE_i  = m_i + ln l_i                              (natural log)
 *     P_ij   = exp(s_ij - LSE_i)
 *     O_i    = sum_j P_ij v_j
 *
 *   The pages never write the backward pass; they only require it to recompute the
 *   score tiles instead of storing them (next-generation page, "Recomputation").  The
 *   oracle therefore takes the plain calculus gradient of L = <O, dO>:
 *
 *     dP_ij  = <do_i, v_j>
 *     Delta_i = sum_j P_ij dP_ij
 *     dS_ij  = P_ij (dP_ij - Delta_i)
 *     dQ_i   = scale * sum_j dS_ij k_j
 *     dK_j   = scale * sum_{h: kv(h)=kv} sum_{i: j in J(i)} dS_ij q_i
 *     dV_j   =         sum_{h: kv(h)=kv} sum_{i: j in J(i)} P_ij do_i
 *
 * Layout: every tensor is [B, H, N, d] contiguous (LSE and Delta are [B, Hq, N]).
 * Every output element is written by exactly one loop iteration with a fixed summation
 * order, so results do not depend on the OpenMP thread count.
 *
 * Return codes: 0 on success, -1 for an invalid argument (nothing written),
 * -2 when scratch memory cannot be obtained.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <stddef.h>

static int check_args(int B, int Hq, int Hkv, int N, int d)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    return 0;
}

static double dotd(const double *a, const double *b, int d)
{
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += a[c] * b[c];
    return acc;
}

/*
 * Keys visible to query row i: J(i) = {j : lo <= j < hi} with
 *   lo = max(0, i - left)      (left  < 0: no lower limit)
 *   hi = min(N, i + right + 1) (right < 0: no upper limit)
 * Causal attention is right = 0; full attention is left = right = -1.
 */
static void row_range(int i, int N, int left, int right, int *lo, int *hi)
{
    *lo = (left < 0 || i - left < 0) ? 0 : i - left;
    *hi = (right < 0 || i + right + 1 > N) ? N : i + right + 1;
}

/* s_ij for j in J(i) into s[j - lo], and the natural-log logsumexp of that row. */
static double scores_and_lse(const double *qi, const double *kh, int lo, int hi, int d,
                             double scale, double *s)
{
    double m = -INFINITY;
    for (int j = lo; j < hi; ++j) {
        s[j - lo] = scale * dotd(qi, kh + (size_t)j * d, d);
        if (s[j - lo] > m) m = s[j - lo];
    }
    double l = 0.0;
    for (int j = lo; j < hi; ++j) l += exp(s[j - lo] - m);
    return m + log(l);
}

/* Forward with a key window: O [B,Hq,N,d] and LSE [B,Hq,N].  Every row must see at least
 * one key (always true when left >= 0 or right >= 0 admits j = i, or for full rows). */
int oracle_fwd_window(const double *q, const double *k, const double *v, double *o, double *lse,
                      int B, int Hq, int Hkv, int N, int d, int left, int right, double scale)
{
    if (check_args(B, Hq, Hkv, N, d) || !q || !k || !v || !o || !lse) return -1;
    const int g = Hq / Hkv;
    const long long rows = (long long)B * Hq * N;
    int fail = 0;
#pragma omp parallel reduction(|: fail)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        if (!s) {
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < rows; ++r) {
                const int i = (int)(r % N);
                const long long bh = r / N;
                const int h = (int)(bh % Hq), b = (int)(bh / Hq);
                const int kvh = h / g;
                const double *qi = q + (size_t)r * d;
                const double *kh = k + ((size_t)b * Hkv + kvh) * (size_t)N * d;
                const double *vh = v + ((size_t)b * Hkv + kvh) * (size_t)N * d;
                int lo, hi;
                row_range(i, N, left, right, &lo, &hi);
                const double L = scores_and_lse(qi, kh, lo, hi, d, scale, s);
                double *oi = o + (size_t)r * d;
                for (int c = 0; c < d; ++c) oi[c] = 0.0;
                for (int j = lo; j < hi; ++j) {
                    const double p = exp(s[j - lo] - L);
                    const double *vj = vh + (size_t)j * d;
                    for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
                }
                lse[r] = L;
            }
            free(s);
        }
    }
    return fail ? -2 : 0;
}

/* Forward: O [B,Hq,N,d] and LSE [B,Hq,N]; causal keeps keys j <= i. */
int oracle_fwd(const double *q, const double *k, const double *v, double *o, double *lse,
               int B, int Hq, int Hkv, int N, int d, int causal, double scale)
{
    return oracle_fwd_window(q, k, v, o, lse, B, Hq, Hkv, N, d, -1, causal ? 0 : -1, scale);
}

/*
 * Backward: dQ [B,Hq,N,d], dK and dV [B,Hkv,N,d].  lse_out and delta_out ([B,Hq,N])
 * may be NULL; when given they receive LSE_i and Delta_i.
 *
 * Pass 1 runs over query rows (LSE_i, Delta_i, dQ_i); pass 2 runs over key rows and
 * recomputes s_ij, P_ij and dP_ij for every query row that attends to that key.
 */
int oracle_bwd_window(const double *q, const double *k, const double *v, const double *dout,
                      double *dq, double *dk, double *dv, double *lse_out, double *delta_out,
                      int B, int Hq, int Hkv, int N, int d, int left, int right, double scale)
{
    if (check_args(B, Hq, Hkv, N, d) || !q || !k || !v || !dout || !dq || !dk || !dv)
        return -1;
    const int g = Hq / Hkv;
    const long long qrows = (long long)B * Hq * N;
    double *L = (double *)malloc(sizeof(double) * (size_t)qrows);
    double *D = (double *)malloc(sizeof(double) * (size_t)qrows);
    if (!L || !D) { free(L); free(D); return -2; }
    int fail = 0;

    /* Pass 1: per query row. */
#pragma omp parallel reduction(|: fail)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)N);
        if (!s || !dp) {
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < qrows; ++r) {
                const int i = (int)(r % N);
                const long long bh = r / N;
                const int h = (int)(bh % Hq), b = (int)(bh / Hq);
                const int kvh = h / g;
                const double *qi = q + (size_t)r * d;
                const double *doi = dout + (size_t)r * d;
                const double *kh = k + ((size_t)b * Hkv + kvh) * (size_t)N * d;
                const double *vh = v + ((size_t)b * Hkv + kvh) * (size_t)N * d;
                int lo, hi;
                row_range(i, N, left, right, &lo, &hi);
                const double Li = scores_and_lse(qi, kh, lo, hi, d, scale, s);
                double Di = 0.0;
                for (int j = lo; j < hi; ++j) {
                    dp[j - lo] = dotd(doi, vh + (size_t)j * d, d);
                    Di += exp(s[j - lo] - Li) * dp[j - lo];
                }
                double *dqi = dq + (size_t)r * d;
                for (int c = 0; c < d; ++c) dqi[c] = 0.0;
                for (int j = lo; j < hi; ++j) {
                    const double dS = exp(s[j - lo] - Li) * (dp[j - lo] - Di);
                    const double *kj = kh + (size_t)j * d;
                    for (int c = 0; c < d; ++c) dqi[c] += dS * kj[c];
                }
                for (int c = 0; c < d; ++c) dqi[c] *= scale;
                L[r] = Li;
                D[r] = Di;
            }
        }
        free(s);
        free(dp);
    }
    if (fail) { free(L); free(D); return -2; }

    /* Pass 2: per key row of each K/V head. */
    const long long krows = (long long)B * Hkv * N;
#pragma omp parallel for schedule(dynamic, 16)
    for (long long r = 0; r < krows; ++r) {
        const int j = (int)(r % N);
        const long long bk = r / N;
        const int kvh = (int)(bk % Hkv), b = (int)(bk / Hkv);
        const double *kj = k + (size_t)r * d;
        const double *vj = v + (size_t)r * d;
        double *dkj = dk + (size_t)r * d;
        double *dvj = dv + (size_t)r * d;
        for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
        for (int h = kvh * g; h < (kvh + 1) * g; ++h) {
            const size_t head = ((size_t)b * Hq + h) * (size_t)N;
            /* queries that see key j: j - right <= i <= j + left */
            const int i0 = (right < 0 || j - right < 0) ? 0 : j - right;
            const int i1 = (left < 0 || j + left + 1 > N) ? N : j + left + 1;
            for (int i = i0; i < i1; ++i) {
                const double *qi = q + (head + i) * d;
                const double *doi = dout + (head + i) * d;
                const double s = scale * dotd(qi, kj, d);
                const double P = exp(s - L[head + i]);
                const double dP = dotd(doi, vj, d);
                const double dS = P * (dP - D[head + i]);
                for (int c = 0; c < d; ++c) {
                    dvj[c] += P * doi[c];
                    dkj[c] += dS * qi[c];
                }
            }
        }
        for (int c = 0; c < d; ++c) dkj[c] *= scale;
    }

    if (lse_out)
        for (long long r = 0; r < qrows; ++r) lse_out[r] = L[r];
    if (delta_out)
        for (long long r = 0; r < qrows; ++r) delta_out[r] = D[r];
    free(L);
    free(D);
    return 0;
}

int oracle_bwd(const double *q, const double *k, const double *v, const double *dout,
               double *dq, double *dk, double *dv, double *lse_out, double *delta_out,
               int B, int Hq, int Hkv, int N, int d, int causal, double scale)
{
    return oracle_bwd_window(q, k, v, dout, dq, dk, dv, lse_out, delta_out, B, Hq, Hkv, N, d,
                             -1, causal ? 0 : -1, scale);
}

/*
 * The online-softmax recurrence of the "FlashAttention1" Q&A page, question
 * "computation of the softmax function", over one row of scores split into blocks of
 * `block` entries: for block t with local maximum lm_t and local sum
 * ls_t = sum exp(s - lm_t),
 *     m_t = max(m_{t-1}, lm_t)
 *     l_t = l_{t-1} exp(m_{t-1} - m_t) + ls_t exp(lm_t - m_t)
 * Returns m and l after the last block through the out-pointers (LSE = m + ln l).
 * Used by the tests to check that the blocked statistics equal the two-pass ones.
 */
int oracle_online_softmax_stats(const double *s, int n, int block, double *m_out,
                                double *l_out)
{
    if (!s || n < 1 || block < 1 || !m_out || !l_out) return -1;
    double m = -INFINITY, l = 0.0;
    for (int t0 = 0; t0 < n; t0 += block) {
        const int t1 = t0 + block < n ? t0 + block : n;
        double lm = -INFINITY;
        for (int j = t0; j < t1; ++j)
            if (s[j] > lm) lm = s[j];
        double ls = 0.0;
        for (int j = t0; j < t1; ++j) ls += exp(s[j] - lm);
        const double mn = lm > m ? lm : m;
        l = (m == -INFINITY ? 0.0 : l * exp(m - mn)) + ls * exp(lm - mn);
        m = mn;
    }
    *m_out = m;
    *l_out = l;
    return 0;
}

/*
 * Attention of Nq query rows against a cache of Nk key rows, of which the first lens[b]
 * are valid in batch b (lens == NULL: all Nk).  This is the incremental case of the
 * "FlashAttention1" Q&A page (question on scaling to long sequences, item 8: incremental
 * attention updates for streaming inference): the newest Nq tokens attend to everything
 * cached so far.  With `causal` the queries are the LAST Nq positions of the sequence
 * (bottom-right alignment): query t sits at position lens[b] - Nq + t and sees keys
 * j <= lens[b] - Nq + t.  A query that sees no key gets O = 0 and LSE = -inf.
 * q, o: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d]; lse: [B, Hq, Nq].
 */
int oracle_decode(const double *q, const double *k, const double *v, const int *lens,
                  double *o, double *lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                  int causal, double scale)
{
    if (check_args(B, Hq, Hkv, Nq, d) || Nk < 1 || !q || !k || !v || !o || !lse) return -1;
    if (lens)
        for (int b = 0; b < B; ++b)
            if (lens[b] < 0 || lens[b] > Nk) return -1;
    const int g = Hq / Hkv;
    const long long rows = (long long)B * Hq * Nq;
    int fail = 0;
#pragma omp parallel reduction(|: fail)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Nk);
        if (!s) {
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (long long r = 0; r < rows; ++r) {
                const int t = (int)(r % Nq);
                const long long bh = r / Nq;
                const int h = (int)(bh % Hq), b = (int)(bh / Hq);
                const int len = lens ? lens[b] : Nk;
                int hi = len;
                if (causal && len - Nq + t + 1 < hi) hi = len - Nq + t + 1;
                double *oi = o + (size_t)r * d;
                for (int c = 0; c < d; ++c) oi[c] = 0.0;
                if (hi <= 0) {
                    lse[r] = -INFINITY;
                    continue;
                }
                const double *kh = k + ((size_t)b * Hkv + h / g) * (size_t)Nk * d;
                const double *vh = v + ((size_t)b * Hkv + h / g) * (size_t)Nk * d;
                const double L = scores_and_lse(q + (size_t)r * d, kh, 0, hi, d, scale, s);
                for (int j = 0; j < hi; ++j) {
                    const double p = exp(s[j] - L);
                    const double *vj = vh + (size_t)j * d;
                    for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
                }
                lse[r] = L;
            }
            free(s);
        }
    }
    return fail ? -2 : 0;
}

/*
 * Merge of S partial attention results over disjoint key sets: the "efficient reduction"
 * that combines partial results of different blocks ("FlashAttention1" Q&A, question on
 * the key algorithmic innovations, item 3), in the log-sum-exp form of the softmax
 * recurrence on the same page (question on computing the softmax):
 *     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s
 * where O_s is part s's normalised output.  Parts with LSE_s = -inf (no visible key)
 * contribute nothing; when every part is -inf, O = 0 and LSE = -inf.
 * o_parts: [S, rows, d]; lse_parts: [S, rows]; o: [rows, d]; lse: [rows].
 */
int oracle_merge(const double *o_parts, const double *lse_parts, int S, long long rows, int d,
                 double *o, double *lse)
{
    if (!o_parts || !lse_parts || !o || !lse || S < 1 || rows < 1 || d < 1) return -1;
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < rows; ++r) {
        double m = -INFINITY;
        for (int s = 0; s < S; ++s)
            if (lse_parts[(size_t)s * rows + r] > m) m = lse_parts[(size_t)s * rows + r];
        double *orow = o + (size_t)r * d;
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double l = 0.0;
        for (int s = 0; s < S; ++s) l += exp(lse_parts[(size_t)s * rows + r] - m);
        const double L = m + log(l);
        for (int s = 0; s < S; ++s) {
            const double w = exp(lse_parts[(size_t)s * rows + r] - L);
            const double *op = o_parts + ((size_t)s * rows + r) * d;
            for (int c = 0; c < d; ++c) orow[c] += w * op[c];
        }
        lse[r] = L;
    }
    return 0;
}

/*
 * Variable-length batches: B sequences packed along the token axis.
 *   q, o: [total_q, Hq, d];  k, v: [total_k, Hkv, d];  lse: [total_q, Hq]
 *   sequence b owns query rows cu_q[b] .. cu_q[b+1]-1 and key rows cu_k[b] .. cu_k[b+1]-1.
 * Lengths may differ (Lq = cu_q[b+1] - cu_q[b], Lk likewise); the key band is aligned to
 * the END of both (bottom-right): with dlt = Lk - Lq, query i sees keys j with
 *     i + dlt - left <= j <= i + dlt + right,  0 <= j < Lk
 * (a negative bound is unlimited; causal is left < 0, right = 0).  Variable sequence
 * lengths are named on the "FlashAttention1" Q&A page (question on scaling, item 2).  A
 * query row that sees no key gets O = 0 and LSE = -inf.
 */
static void varlen_range(int i, int Lq, int Lk, int left, int right, int *lo, int *hi)
{
    const int c = i + (Lk - Lq);
    *lo = (left < 0 || c - left < 0) ? 0 : c - left;
    *hi = (right < 0 || c + right + 1 > Lk) ? Lk : c + right + 1;
    if (*hi < *lo) *hi = *lo;
}

static int check_cu(const int *cu, int B, int total)
{
    if (!cu || cu[0] < 0) return -1;
    for (int b = 0; b < B; ++b)
        if (cu[b + 1] < cu[b]) return -1;
    return cu[B] > total ? -1 : 0;
}

int oracle_fwd_varlen(const double *q, const double *k, const double *v, const int *cu_q,
                      const int *cu_k, double *o, double *lse, int B, int Hq, int Hkv,
                      int total_q, int total_k, int d, int left, int right, double scale)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv || !q || !k || !v || !o || !lse)
        return -1;
    if (check_cu(cu_q, B, total_q) || check_cu(cu_k, B, total_k)) return -1;
    const int g = Hq / Hkv;
    for (long long r = 0; r < (long long)total_q * Hq; ++r) lse[r] = -INFINITY;
    for (long long r = 0; r < (long long)total_q * Hq * d; ++r) o[r] = 0.0;
    int fail = 0;
    for (int b = 0; b < B; ++b) {
        const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
        const long long rows = (long long)Lq * Hq;
#pragma omp parallel reduction(|: fail)
        {
            double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
            if (!s) {
                fail = 1;
            } else {
#pragma omp for schedule(dynamic, 8)
                for (long long r = 0; r < rows; ++r) {
                    const int i = (int)(r / Hq), h = (int)(r % Hq);
                    int lo, hi;
                    varlen_range(i, Lq, Lk, left, right, &lo, &hi);
                    if (hi <= lo) continue;               /* no key: O = 0, LSE = -inf */
                    const size_t qrow = (size_t)(cu_q[b] + i) * Hq + h;
                    /* key row j of this head: k + ((cu_k[b] + j) * Hkv + h / g) * d */
                    double m = -INFINITY;
                    for (int j = lo; j < hi; ++j) {
                        const double *kj = k + ((size_t)(cu_k[b] + j) * Hkv + h / g) * d;
                        s[j - lo] = scale * dotd(q + qrow * d, kj, d);
                        if (s[j - lo] > m) m = s[j - lo];
                    }
                    double l = 0.0;
                    for (int j = lo; j < hi; ++j) l += exp(s[j - lo] - m);
                    const double L = m + log(l);
                    double *oi = o + qrow * d;
                    for (int j = lo; j < hi; ++j) {
                        const double p = exp(s[j - lo] - L);
                        const double *vj = v + ((size_t)(cu_k[b] + j) * Hkv + h / g) * d;
                        for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
                    }
                    lse[qrow] = L;
                }
                free(s);
            }
        }
    }
    return fail ? -2 : 0;
}

/*
 * Gradient of <O, dO> for variable-length batches (layouts as oracle_fwd_varlen; dq like q,
 * dk and dv like k).  Pass 1 runs over query rows (LSE, Delta, dQ); pass 2 over key rows,
 * visiting every query row whose band contains the key.
 */
int oracle_bwd_varlen(const double *q, const double *k, const double *v, const double *dout,
                      const int *cu_q, const int *cu_k, double *dq, double *dk, double *dv,
                      int B, int Hq, int Hkv, int total_q, int total_k, int d, int left,
                      int right, double scale)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || d < 1 || Hq % Hkv || !q || !k || !v || !dout || !dq ||
        !dk || !dv)
        return -1;
    if (check_cu(cu_q, B, total_q) || check_cu(cu_k, B, total_k)) return -1;
    const int g = Hq / Hkv;
    const long long nq = (long long)total_q * Hq;
    double *L = (double *)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1));
    double *D = (double *)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1));
    if (!L || !D) { free(L); free(D); return -2; }
    for (long long r = 0; r < nq * d; ++r) dq[r] = 0.0;
    for (long long r = 0; r < (long long)total_k * Hkv * d; ++r) { dk[r] = 0.0; dv[r] = 0.0; }
    for (long long r = 0; r < nq; ++r) { L[r] = -INFINITY; D[r] = 0.0; }
    int fail = 0;
    for (int b = 0; b < B && !fail; ++b) {
        const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
        const long long rows = (long long)Lq * Hq;
        /* Pass 1: per query row. */
#pragma omp parallel reduction(|: fail)
        {
            double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
            double *dp = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
            if (!s || !dp) {
                fail = 1;
            } else {
#pragma omp for schedule(dynamic, 8)
                for (long long r = 0; r < rows; ++r) {
                    const int i = (int)(r / Hq), h = (int)(r % Hq);
                    int lo, hi;
                    varlen_range(i, Lq, Lk, left, right, &lo, &hi);
                    if (hi <= lo) continue;
                    const size_t qrow = (size_t)(cu_q[b] + i) * Hq + h;
                    double m = -INFINITY;
                    for (int j = lo; j < hi; ++j) {
                        const double *kj = k + ((size_t)(cu_k[b] + j) * Hkv + h / g) * d;
                        s[j - lo] = scale * dotd(q + qrow * d, kj, d);
                        if (s[j - lo] > m) m = s[j - lo];
                    }
                    double l = 0.0;
                    for (int j = lo; j < hi; ++j) l += exp(s[j - lo] - m);
                    const double Li = m + log(l);
                    double Di = 0.0;
                    for (int j = lo; j < hi; ++j) {
                        const double *vj = v + ((size_t)(cu_k[b] + j) * Hkv + h / g) * d;
                        dp[j - lo] = dotd(dout + qrow * d, vj, d);
                        Di += exp(s[j - lo] - Li) * dp[j - lo];
                    }
                    double *dqi = dq + qrow * d;
                    for (int j = lo; j < hi; ++j) {
                        const double dS = exp(s[j - lo] - Li) * (dp[j - lo] - Di);
                        const double *kj = k + ((size_t)(cu_k[b] + j) * Hkv + h / g) * d;
                        for (int c = 0; c < d; ++c) dqi[c] += dS * kj[c];
                    }
                    for (int c = 0; c < d; ++c) dqi[c] *= scale;
                    L[qrow] = Li;
                    D[qrow] = Di;
                }
            }
            free(s);
            free(dp);
        }
        if (fail) break;
        /* Pass 2: per key row of each K/V head. */
        const long long krows = (long long)Lk * Hkv;
#pragma omp parallel for schedule(dynamic, 8)
        for (long long r = 0; r < krows; ++r) {
            const int j = (int)(r / Hkv), kvh = (int)(r % Hkv);
            const size_t krow = (size_t)(cu_k[b] + j) * Hkv + kvh;
            const double *kj = k + krow * d, *vj = v + krow * d;
            double *dkj = dk + krow * d, *dvj = dv + krow * d;
            for (int h = kvh * g; h < (kvh + 1) * g; ++h) {
                for (int i = 0; i < Lq; ++i) {
                    int lo, hi;
                    varlen_range(i, Lq, Lk, left, right, &lo, &hi);
                    if (j < lo || j >= hi) continue;
                    const size_t qrow = (size_t)(cu_q[b] + i) * Hq + h;
                    const double *qi = q + qrow * d, *doi = dout + qrow * d;
                    const double P = exp(scale * dotd(qi, kj, d) - L[qrow]);
                    const double dS = P * (dotd(doi, vj, d) - D[qrow]);
                    for (int c = 0; c < d; ++c) {
                        dvj[c] += P * doi[c];
                        dkj[c] += dS * qi[c];
                    }
                }
            }
            for (int c = 0; c < d; ++c) dkj[c] *= scale;
        }
    }
    free(L);
    free(D);
    return fail ? -2 : 0;
}

/*
 * Attention dropout.  The deep-dive page names dropout among the memory-bound steps of
 * standard attention ("Quantitative Evidence") but gives no generator; the reading here:
 * every probability P_ij of query head bh is kept with probability 1 - p and kept values
 * are scaled by 1 / (1 - p), so
 *     O_i = sum_j P_ij Z_ij / (1 - p) v_j,   Z_ij in {0, 1},
 * while LSE_i is the logsumexp of the scores (dropout does not enter the normaliser).
 * Z comes from the counter-based generator Philox4x32-10 (Salmon, Moraes, Dror and Shaw,
 * "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011), written from its published
 * definition: key (seed low 32 bits, seed high 32 bits), counter (j / 8, i, bh, 0).  The
 * four 32-bit output words hold eight 16-bit values, value j % 8 being the low (even) or
 * high (odd) half of word (j % 8) / 2; the element is kept iff that value is >= thr =
 * min(floor(p 2^16), 2^16 - 1), so the keep probability is exactly 1 - thr / 2^16 and the
 * kept values are scaled by its inverse, 2^16 / (2^16 - thr) (unbiased; within 2^-16 of
 * 1 / (1 - p)).  The decision is integer-only, so any implementation of the same
 * definition reproduces it bit for bit.
 */
static void philox4x32_10(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3, uint32_t k0,
                          uint32_t k1, uint32_t out[4])
{
    for (int round = 0; round < 10; ++round) {
        /* one Philox round: two 32x32 -> 64-bit products, then mix with the key */
        const uint64_t prod0 = (uint64_t)0xD2511F53u * x0;
        const uint64_t prod1 = (uint64_t)0xCD9E8D57u * x2;
        const uint32_t y0 = (uint32_t)(prod1 >> 32) ^ x1 ^ k0;
        const uint32_t y1 = (uint32_t)prod1;
        const uint32_t y2 = (uint32_t)(prod0 >> 32) ^ x3 ^ k1;
        const uint32_t y3 = (uint32_t)prod0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
        k0 += 0x9E3779B9u;  /* key schedule: Weyl sequence */
        k1 += 0xBB67AE85u;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The generator itself, exported so that tests can compare it word for word with an
 * independent implementation: out = Philox4x32-10(counter ctr[0..3], key key[0..1]). */
int oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    if (!ctr || !key || !out) return -1;
    philox4x32_10(ctr[0], ctr[1], ctr[2], ctr[3], key[0], key[1], out);
    return 0;
}

static uint32_t drop_threshold(double p)
{
    const double t = floor(p * 65536.0);
    return t >= 65535.0 ? 65535u : (uint32_t)t;
}

/* 1 when element (bh, i, j) is kept, 0 when dropped. */
static int drop_keep(uint64_t seed, uint32_t thr, uint32_t bh, int i, int j)
{
    uint32_t w[4];
    philox4x32_10((uint32_t)j >> 3, (uint32_t)i, bh, 0u, (uint32_t)seed, (uint32_t)(seed >> 32), w);
    const uint32_t word = w[(j & 7) >> 1];
    const uint32_t value = (j & 1) ? (word >> 16) : (word & 0xFFFFu);
    return value >= thr;
}

/* keep[bh][i][j] for BH query heads of N rows and N keys (uint8). */
int oracle_dropout_mask(unsigned char *keep, int BH, int N, double p, uint64_t seed)
{
    if (!keep || BH < 1 || N < 1 || !(p >= 0.0 && p < 1.0)) return -1;
    const uint32_t thr = drop_threshold(p);
#pragma omp parallel for schedule(static)
    for (long long r = 0; r < (long long)BH * N; ++r)
        for (int j = 0; j < N; ++j)
            keep[(size_t)r * N + j] = (unsigned char)drop_keep(seed, thr, (uint32_t)(r / N), (int)(r % N), j);
    return 0;
}

int oracle_fwd_dropout(const double *q, const double *k, const double *v, double *o, double *lse,
                       int B, int Hq, int Hkv, int N, int d, int causal, double scale, double p,
                       uint64_t seed)
{
    if (check_args(B, Hq, Hkv, N, d) || !q || !k || !v || !o || !lse || !(p >= 0.0 && p < 1.0))
        return -1;
    const int g = Hq / Hkv;
    const uint32_t thr = drop_threshold(p);
    const double inv_keep = 65536.0 / (65536.0 - (double)thr);
    const long long rows = (long long)B * Hq * N;
    int fail = 0;
#pragma omp parallel reduction(|: fail)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        if (!s) {
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < rows; ++r) {
                const int i = (int)(r % N);
                const long long bh = r / N;
                const int b = (int)(bh / Hq), h = (int)(bh % Hq);
                const double *kh = k + ((size_t)b * Hkv + h / g) * (size_t)N * d;
                const double *vh = v + ((size_t)b * Hkv + h / g) * (size_t)N * d;
                const int hi = causal ? i + 1 : N;
                const double L = scores_and_lse(q + (size_t)r * d, kh, 0, hi, d, scale, s);
                double *oi = o + (size_t)r * d;
                for (int c = 0; c < d; ++c) oi[c] = 0.0;
                for (int j = 0; j < hi; ++j) {
                    if (!drop_keep(seed, thr, (uint32_t)bh, i, j)) continue;
                    const double pz = exp(s[j] - L) * inv_keep;
                    const double *vj = vh + (size_t)j * d;
                    for (int c = 0; c < d; ++c) oi[c] += pz * vj[c];
                }
                lse[r] = L;
            }
            free(s);
        }
    }
    return fail ? -2 : 0;
}

/*
 * Gradient of <O, dO> for the dropout forward above (the mask is a fixed function of the
 * seed): with Zs_ij = Z_ij / keep probability,
 *     dP_ij = Zs_ij <do_i, v_j>,  Delta_i = sum_j P_ij dP_ij (= <do_i, o_i>),
 *     dS_ij = P_ij (dP_ij - Delta_i),
 *     dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i,  dV_j = sum_i P_ij Zs_ij do_i.
 */
int oracle_bwd_dropout(const double *q, const double *k, const double *v, const double *dout,
                       double *dq, double *dk, double *dv, int B, int Hq, int Hkv, int N, int d,
                       int causal, double scale, double p, uint64_t seed)
{
    if (check_args(B, Hq, Hkv, N, d) || !q || !k || !v || !dout || !dq || !dk || !dv ||
        !(p >= 0.0 && p < 1.0))
        return -1;
    const int g = Hq / Hkv;
    const uint32_t thr = drop_threshold(p);
    const double inv_keep = 65536.0 / (65536.0 - (double)thr);
    const long long qrows = (long long)B * Hq * N;
    double *Lv = (double *)malloc(sizeof(double) * (size_t)qrows);
    double *Dv = (double *)malloc(sizeof(double) * (size_t)qrows);
    if (!Lv || !Dv) { free(Lv); free(Dv); return -2; }
    int fail = 0;
#pragma omp parallel reduction(|: fail)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)N);
        if (!s || !dp) {
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < qrows; ++r) {
                const int i = (int)(r % N);
                const long long bh = r / N;
                const int b = (int)(bh / Hq), h = (int)(bh % Hq);
                const double *kh = k + ((size_t)b * Hkv + h / g) * (size_t)N * d;
                const double *vh = v + ((size_t)b * Hkv + h / g) * (size_t)N * d;
                const int hi = causal ? i + 1 : N;
                const double Li = scores_and_lse(q + (size_t)r * d, kh, 0, hi, d, scale, s);
                double Di = 0.0;
                for (int j = 0; j < hi; ++j) {
                    const double zs = drop_keep(seed, thr, (uint32_t)bh, i, j) ? inv_keep : 0.0;
                    dp[j] = zs * dotd(dout + (size_t)r * d, vh + (size_t)j * d, d);
                    Di += exp(s[j] - Li) * dp[j];
                }
                double *dqi = dq + (size_t)r * d;
                for (int c = 0; c < d; ++c) dqi[c] = 0.0;
                for (int j = 0; j < hi; ++j) {
                    const double dS = exp(s[j] - Li) * (dp[j] - Di);
                    const double *kj = kh + (size_t)j * d;
                    for (int c = 0; c < d; ++c) dqi[c] += dS * kj[c];
                }
                for (int c = 0; c < d; ++c) dqi[c] *= scale;
                Lv[r] = Li;
                Dv[r] = Di;
            }
        }
        free(s);
        free(dp);
    }
    if (fail) { free(Lv); free(Dv); return -2; }
    const long long krows = (long long)B * Hkv * N;
#pragma omp parallel for schedule(dynamic, 16)
    for (long long r = 0; r < krows; ++r) {
        const int j = (int)(r % N);
        const long long bk = r / N;
        const int kvh = (int)(bk % Hkv), b = (int)(bk / Hkv);
        const double *kj = k + (size_t)r * d, *vj = v + (size_t)r * d;
        double *dkj = dk + (size_t)r * d, *dvj = dv + (size_t)r * d;
        for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
        for (int h = kvh * g; h < (kvh + 1) * g; ++h) {
            const long long bh = (long long)b * Hq + h;
            for (int i = causal ? j : 0; i < N; ++i) {
                const size_t qr = (size_t)bh * N + i;
                const double *qi = q + qr * d, *doi = dout + qr * d;
                const double P = exp(scale * dotd(qi, kj, d) - Lv[qr]);
                const double zs = drop_keep(seed, thr, (uint32_t)bh, i, j) ? inv_keep : 0.0;
                const double dS = P * (zs * dotd(doi, vj, d) - Dv[qr]);
                for (int c = 0; c < d; ++c) {
                    dvj[c] += P * zs * doi[c];
                    dkj[c] += dS * qi[c];
                }
            }
        }
        for (int c = 0; c < d; ++c) dkj[c] *= scale;
    }
    free(Lv);
    free(Dv);
    return 0;
}

/*
 * Block-sparse attention: the deep-dive page closes by naming block-sparse FlashAttention
 * without defining it.  The reading here: a 0/1 mask over 128 x 128 blocks of the score
 * matrix of each query head, bmask[b][h][i / 128][j / 128] (nb = ceil(N / 128) blocks per
 * side), so key j is visible to query i iff its block is enabled (and, with `causal`,
 * j <= i).  A row that sees no key gets O = 0 and LSE = -inf.
 */
static int block_visible(const unsigned char *bmask, int nb, long long bh, int i, int j, int causal)
{
    if (causal && j > i) return 0;
    return bmask[((size_t)bh * nb + (size_t)(i / 128)) * nb + (size_t)(j / 128)] != 0;
}

int oracle_fwd_blocksparse(const double *q, const double *k, const double *v,
                           const unsigned char *bmask, double *o, double *lse, int B, int Hq,
                           int Hkv, int N, int d, int causal, double scale)
{
    if (check_args(B, Hq, Hkv, N, d) || !q || !k || !v || !bmask || !o || !lse) return -1;
    const int g = Hq / Hkv, nb = (N + 127) / 128;
    const long long rows = (long long)B * Hq * N;
    int fail = 0;
#pragma omp parallel reduction(|: fail)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        int *idx = (int *)malloc(sizeof(int) * (size_t)N);
        if (!s || !idx) {
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long long r = 0; r < rows; ++r) {
                const int i = (int)(r % N);
                const long long bh = r / N;
                const int b = (int)(bh / Hq), h = (int)(bh % Hq);
                const double *kh = k + ((size_t)b * Hkv + h / g) * (size_t)N * d;
                const double *vh = v + ((size_t)b * Hkv + h / g) * (size_t)N * d;
                double *oi = o + (size_t)r * d;
                for (int c = 0; c < d; ++c) oi[c] = 0.0;
                int n = 0;
                double m = -INFINITY;
                for (int j = 0; j < N; ++j) {
                    if (!block_visible(bmask, nb, bh, i, j, causal)) continue;
                    idx[n] = j;
                    s[n] = scale * dotd(q + (size_t)r * d, kh + (size_t)j * d, d);
                    if (s[n] > m) m = s[n];
                    ++n;
                }
                if (n == 0) {
                    lse[r] = -INFINITY;
                    continue;
                }
                double l = 0.0;
                for (int t = 0; t < n; ++t) l += exp(s[t] - m);
                const double L = m + log(l);
                for (int t = 0; t < n; ++t) {
                    const double p = exp(s[t] - L);
                    const double *vj = vh + (size_t)idx[t] * d;
                    for (int c = 0; c < d; ++c) oi[c] += p * vj[c];
                }
                lse[r] = L;
            }
        }
        free(s);
        free(idx);
    }
    return fail ? -2 : 0;
}

/* Gradient of <O, dO> for block-sparse attention (same mask and causal flag). */
int oracle_bwd_blocksparse(const double *q, const double *k, const double *v, const double *dout,
                           const unsigned char *bmask, double *dq, double *dk, double *dv, int B,
                           int Hq, int Hkv, int N, int d, int causal, double scale)
{
    if (check_args(B, Hq, Hkv, N, d) || !q || !k || !v || !dout || !bmask || !dq || !dk || !dv)
        return -1;
    const int g = Hq / Hkv, nb = (N + 127) / 128;
    const long long qrows = (long long)B * Hq * N;
    double *Lv = (double *)malloc(sizeof(double) * (size_t)qrows);
    double *Dv = (double *)malloc(sizeof(double) * (size_t)qrows);
    double *o = (double *)malloc(sizeof(double) * (size_t)qrows * d);
    if (!Lv || !Dv || !o) { free(Lv); free(Dv); free(o); return -2; }
    int rc = oracle_fwd_blocksparse(q, k, v, bmask, o, Lv, B, Hq, Hkv, N, d, causal, scale);
    if (rc) { free(Lv); free(Dv); free(o); return rc; }
    /* Delta_i = <dO_i, O_i>; rows without keys have O = 0, so Delta = 0. */
    for (long long r = 0; r < qrows; ++r) Dv[r] = dotd(dout + (size_t)r * d, o + (size_t)r * d, d);
    free(o);
#pragma omp parallel for schedule(dynamic, 16)
    for (long long r = 0; r < qrows; ++r) {
        const int i = (int)(r % N);
        const long long bh = r / N;
        const int b = (int)(bh / Hq), h = (int)(bh % Hq);
        const double *kh = k + ((size_t)b * Hkv + h / g) * (size_t)N * d;
        const double *vh = v + ((size_t)b * Hkv + h / g) * (size_t)N * d;
        double *dqi = dq + (size_t)r * d;
        for (int c = 0; c < d; ++c) dqi[c] = 0.0;
        for (int j = 0; j < N; ++j) {
            if (!block_visible(bmask, nb, bh, i, j, causal)) continue;
            const double P = exp(scale * dotd(q + (size_t)r * d, kh + (size_t)j * d, d) - Lv[r]);
            const double dS = P * (dotd(dout + (size_t)r * d, vh + (size_t)j * d, d) - Dv[r]);
            for (int c = 0; c < d; ++c) dqi[c] += dS * kh[(size_t)j * d + c];
        }
        for (int c = 0; c < d; ++c) dqi[c] *= scale;
    }
    const long long krows = (long long)B * Hkv * N;
#pragma omp parallel for schedule(dynamic, 16)
    for (long long r = 0; r < krows; ++r) {
        const int j = (int)(r % N);
        const long long bk = r / N;
        const int kvh = (int)(bk % Hkv), b = (int)(bk / Hkv);
        const double *kj = k + (size_t)r * d, *vj = v + (size_t)r * d;
        double *dkj = dk + (size_t)r * d, *dvj = dv + (size_t)r * d;
        for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
        for (int h = kvh * g; h < (kvh + 1) * g; ++h) {
            const long long bh = (long long)b * Hq + h;
            for (int i = 0; i < N; ++i) {
                if (!block_visible(bmask, nb, bh, i, j, causal)) continue;
                const size_t qr = (size_t)bh * N + i;
                const double *qi = q + qr * d, *doi = dout + qr * d;
                const double P = exp(scale * dotd(qi, kj, d) - Lv[qr]);
                const double dS = P * (dotd(doi, vj, d) - Dv[qr]);
                for (int c = 0; c < d; ++c) {
                    dvj[c] += P * doi[c];
                    dkj[c] += dS * qi[c];
                }
            }
        }
        for (int c = 0; c < d; ++c) dkj[c] *= scale;
    }
    free(Lv);
    free(Dv);
    return 0;
}
