/*
 * Scalar fp64 brute force of softmax attention and its gradient, one
 * (batch, head) slice per call.
 *
 * TEST INFRASTRUCTURE ONLY: a second, independent implementation used on tiny
 * shapes to check the NumPy oracle.  It shares no code with the NumPy oracle or
 * with the CUDA library, and the CUDA library never links it.
 *
 * Definitions (plainest reading of O = softmax(Q K^T * scale [+ causal mask]) V,
 * which "Flash Attention spiegata: una guida completa", section "Attention
 * standard vs Flash attention", says the tiled method reproduces exactly):
 *   S_ij  = scale * sum_c q_ic k_jc, for j <= i when causal, every j otherwise
 *   lse_i = m_i + log(sum_j exp(S_ij - m_i)),   m_i = max_j S_ij
 *   P_ij  = exp(S_ij - lse_i)
 *   o_ic  = sum_j P_ij v_jc
 * and for L = sum o * dO:
 *   dv_jc = sum_i P_ij do_ic
 *   dP_ij = sum_c do_ic v_jc
 *   dS_ij = P_ij (dP_ij - sum_l P_il dP_il)
 *   dq_ic = scale sum_j dS_ij k_jc,  dk_jc = scale sum_i dS_ij q_ic
 * With a sliding window W (causal only; "Flash Attention 2: attivarla", section
 * "Modelli con attenzione a finestra scorrevole non standard") row i sees only
 * keys i-W+1..i; brute_set_window(0) turns it off.
 * All arrays are row-major [n][d] doubles.
 */
#include <math.h>
#include <stdlib.h>

/* window <= 0: no sliding window; otherwise (causal) row i sees keys i-window+1..i */
static int g_window = 0;
static int visible(int i, int j, int causal) {
    if (causal && j > i) return 0;
    if (causal && g_window > 0 && j < i - g_window + 1) return 0;
    return 1;
}

static double score(const double *q, const double *k, int i, int j, int d,
                    double scale) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += q[(size_t)i * d + c] * k[(size_t)j * d + c];
    return scale * acc;
}

/* Row log-sum-exp of the scaled scores of query row i. */
static double row_lse(const double *q, const double *k, int i, int n, int d,
                      double scale, int causal) {
    double m = -INFINITY;
    for (int j = 0; j < n; ++j)
        if (visible(i, j, causal)) {
            double s = score(q, k, i, j, d, scale);
            if (s > m) m = s;
        }
    double z = 0.0;
    for (int j = 0; j < n; ++j)
        if (visible(i, j, causal)) z += exp(score(q, k, i, j, d, scale) - m);
    return m + log(z);
}

void brute_set_window(int window) { g_window = window; }

void brute_attn_fwd(const double *q, const double *k, const double *v,
                    double *o, double *lse, int n, int d, double scale,
                    int causal) {
    for (int i = 0; i < n; ++i) {
        double l = row_lse(q, k, i, n, d, scale, causal);
        lse[i] = l;
        for (int c = 0; c < d; ++c) o[(size_t)i * d + c] = 0.0;
        for (int j = 0; j < n; ++j) {
            if (!visible(i, j, causal)) continue;
            double p = exp(score(q, k, i, j, d, scale) - l);
            for (int c = 0; c < d; ++c)
                o[(size_t)i * d + c] += p * v[(size_t)j * d + c];
        }
    }
}

void brute_attn_bwd(const double *q, const double *k, const double *v,
                    const double *dout, double *dq, double *dk, double *dv,
                    int n, int d, double scale, int causal) {
    double *p = (double *)calloc((size_t)n * n, sizeof(double));
    double *dp = (double *)calloc((size_t)n * n, sizeof(double));
    for (size_t t = 0; t < (size_t)n * d; ++t) dq[t] = dk[t] = dv[t] = 0.0;
    for (int i = 0; i < n; ++i) {
        double l = row_lse(q, k, i, n, d, scale, causal);
        for (int j = 0; j < n; ++j) {
            if (!visible(i, j, causal)) continue;
            p[(size_t)i * n + j] = exp(score(q, k, i, j, d, scale) - l);
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += dout[(size_t)i * d + c] * v[(size_t)j * d + c];
            dp[(size_t)i * n + j] = acc;
        }
    }
    for (int i = 0; i < n; ++i) {
        double rowdot = 0.0;
        for (int j = 0; j < n; ++j) rowdot += p[(size_t)i * n + j] * dp[(size_t)i * n + j];
        for (int j = 0; j < n; ++j) {
            double pij = p[(size_t)i * n + j];
            double ds = pij * (dp[(size_t)i * n + j] - rowdot);
            for (int c = 0; c < d; ++c) {
                dv[(size_t)j * d + c] += pij * dout[(size_t)i * d + c];
                dq[(size_t)i * d + c] += scale * ds * k[(size_t)j * d + c];
                dk[(size_t)j * d + c] += scale * ds * q[(size_t)i * d + c];
            }
        }
    }
    free(p);
    free(dp);
}
