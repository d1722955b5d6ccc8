/*
 * Plain fp64 CPU oracle of the gated-retention (gRet) mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct statement
 * of what the GPU library computes.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the GPU product path never does,
 * and this file shares no code, header or table with the CUDA library.
 *
 * Sources (web pages on the YOCO decoder-decoder family):
 *  - "YOCO 深度技术分析" (liuhc.cn), section 2.2 "Gated Retention (gRet)":
 *    gate gamma = sigmoid(X W_gamma)^(1/tau); parallel form (Q K^T (.) D) V;
 *    recurrent form S_n = gamma_n S_{n-1} + K_n^T V_n, output Q_n S_n;
 *    multi-head output: GroupNorm per head, then a swish gate.
 *  - same page, section 5.3.2: chunkwise form (parallel inside a block of B
 *    tokens, recurrent between blocks); the three forms are exactly equivalent.
 *  - "YOCO" (zdszero.github.io), section "Self-Decoder": S_t = gamma_t S_{t-1}
 *    + K_t^T V_t, y_t = Q_t S_t.
 *  - Medium-article translation (xingfushuangcheng.com), "分段递归表示": the
 *    chunk state R_i and a "beta" that summarises the data-controlled decay
 *    (its formulas were lost; beta is read here as the chunk-local cumulative
 *    log-decay b_t).
 *
 * Readings where the pages are silent: no 1/sqrt(d_k) scale; D[n][m] is the
 * product of gamma_{m+1..n} (so D[n][n] = 1); one gate scalar per token and
 * head; GroupNorm over the d_v channels of one head and token, biased variance,
 * explicit eps, no affine; swish(g) = g * sigmoid(g); prefill starts from the
 * given S0 (zero when none is given).
 *
 * Layouts (row-major, contiguous):
 *   Q, K [B][N][H][dk]   V, G, Y, O [B][N][H][dv]   log-gamma, z [B][N][H]
 *   S0, S_final [B][H][dk][dv]
 * A "unit" is one (b, h) pair, u = b * H + h.  Functions that take [u0, u1)
 * process only those units, so callers may split units across threads.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define IDX4(b, n, h, c, N, H, D) ((((size_t)(b) * (N) + (n)) * (H) + (h)) * (D) + (c))

/* log gamma = log(sigmoid(z)^(1/tau)) = -softplus(-z) / tau, with
 * softplus(x) = max(x, 0) + log1p(exp(-|x|)) (section 2.2 gate). */
void oracle_log_gamma(const double* z, long n, double tau, double* lg) {
    for (long i = 0; i < n; ++i) {
        double x = -z[i];
        double sp = (x > 0 ? x : 0.0) + log1p(exp(-fabs(x)));
        lg[i] = -sp / tau;
    }
}

/* Recurrent form (section 2.2, item 2; "YOCO" Self-Decoder):
 *   S <- gamma_n S + K_n^T V_n ;  Y_n = Q_n S.
 * gamma_n = exp(lg_n); lg = -inf gives gamma = 0 exactly. */
void oracle_recurrent(const double* Q, const double* K, const double* V, const double* lg,
                      const double* S0, int B, int H, int N, int dk, int dv, int u0, int u1,
                      double* Y, double* S_final) {
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    for (int u = u0; u < u1; ++u) {
        int b = u / H, h = u % H;
        if (S0) memcpy(S, S0 + (size_t)u * dk * dv, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int n = 0; n < N; ++n) {
            double g = exp(lg[IDX4(b, n, h, 0, N, H, 1)]);
            const double* k = K + IDX4(b, n, h, 0, N, H, dk);
            const double* v = V + IDX4(b, n, h, 0, N, H, dv);
            const double* q = Q + IDX4(b, n, h, 0, N, H, dk);
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j] + k[i] * v[j];
            double* y = Y + IDX4(b, n, h, 0, N, H, dv);
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += q[i] * S[(size_t)i * dv + j];
                y[j] = acc;
            }
        }
        if (S_final) memcpy(S_final + (size_t)u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
    }
    free(S);
}

/* Parallel form (section 2.2, item 1): Y = (Q K^T (.) D) V with
 *   D[n][m] = prod_{i=m+1..n} gamma_i  (n >= m),  0 otherwise,
 * plus, for a non-zero initial state, (prod_{i=1..n} gamma_i) Q_n S0.
 * The products are taken of gamma values directly (not of log sums) so that
 * this form shares no step with the recurrent or chunkwise forms.
 * Costs O(N^2 (dk + dv)) per unit: small N only. */
void oracle_parallel(const double* Q, const double* K, const double* V, const double* lg,
                     const double* S0, int B, int H, int N, int dk, int dv, int u0, int u1,
                     double* Y) {
    double* gam = (double*)malloc(sizeof(double) * (size_t)N);
    double* D = (double*)malloc(sizeof(double) * (size_t)N * N);
    for (int u = u0; u < u1; ++u) {
        int b = u / H, h = u % H;
        for (int n = 0; n < N; ++n) gam[n] = exp(lg[IDX4(b, n, h, 0, N, H, 1)]);
        for (int n = 0; n < N; ++n)
            for (int m = 0; m < N; ++m) {
                if (m > n) { D[(size_t)n * N + m] = 0.0; continue; }
                double p = 1.0;
                for (int i = m + 1; i <= n; ++i) p *= gam[i];
                D[(size_t)n * N + m] = p;
            }
        for (int n = 0; n < N; ++n) {
            const double* q = Q + IDX4(b, n, h, 0, N, H, dk);
            double* y = Y + IDX4(b, n, h, 0, N, H, dv);
            for (int j = 0; j < dv; ++j) y[j] = 0.0;
            for (int m = 0; m <= n; ++m) {
                const double* k = K + IDX4(b, m, h, 0, N, H, dk);
                const double* v = V + IDX4(b, m, h, 0, N, H, dv);
                double a = 0.0;
                for (int i = 0; i < dk; ++i) a += q[i] * k[i];
                a *= D[(size_t)n * N + m];
                for (int j = 0; j < dv; ++j) y[j] += a * v[j];
            }
            if (S0) {
                double p = 1.0;
                for (int i = 0; i <= n; ++i) p *= gam[i];
                const double* s0 = S0 + (size_t)u * dk * dv;
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += q[i] * s0[(size_t)i * dv + j];
                    y[j] += p * acc;
                }
            }
        }
    }
    free(D);
    free(gam);
}

/* Chunkwise form (section 5.3.2; "分段递归表示"): blocks of C tokens, the last
 * one partial when C does not divide N.  With t, s local indices in a block and
 * b_t = sum_{j<=t} lg_j (chunk-local cumulative log-decay, the pages' "beta"):
 *   Y_t    = sum_{s<=t} (Q_t . K_s) e^{b_t - b_s} V_s + e^{b_t} Q_t S_prev
 *   S_next = e^{b_last} S_prev + sum_s e^{b_last - b_s} K_s^T V_s            */
void oracle_chunkwise(const double* Q, const double* K, const double* V, const double* lg,
                      const double* S0, int B, int H, int N, int dk, int dv, int C,
                      int u0, int u1, double* Y, double* S_final) {
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* Sn = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* bc = (double*)malloc(sizeof(double) * (size_t)C);
    for (int u = u0; u < u1; ++u) {
        int b = u / H, h = u % H;
        if (S0) memcpy(S, S0 + (size_t)u * dk * dv, sizeof(double) * (size_t)dk * dv);
        else memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int c0 = 0; c0 < N; c0 += C) {
            int L = (N - c0 < C) ? N - c0 : C;
            double run = 0.0;
            for (int t = 0; t < L; ++t) {
                run += lg[IDX4(b, c0 + t, h, 0, N, H, 1)];
                bc[t] = run;
            }
            for (int t = 0; t < L; ++t) {
                const double* q = Q + IDX4(b, c0 + t, h, 0, N, H, dk);
                double* y = Y + IDX4(b, c0 + t, h, 0, N, H, dv);
                double et = exp(bc[t]);
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += q[i] * S[(size_t)i * dv + j];
                    y[j] = et * acc;
                }
                for (int s = 0; s <= t; ++s) {
                    const double* k = K + IDX4(b, c0 + s, h, 0, N, H, dk);
                    const double* v = V + IDX4(b, c0 + s, h, 0, N, H, dv);
                    double a = 0.0;
                    for (int i = 0; i < dk; ++i) a += q[i] * k[i];
                    a *= exp(bc[t] - bc[s]);
                    for (int j = 0; j < dv; ++j) y[j] += a * v[j];
                }
            }
            double eL = exp(bc[L - 1]);
            for (size_t e = 0; e < (size_t)dk * dv; ++e) Sn[e] = eL * S[e];
            for (int s = 0; s < L; ++s) {
                const double* k = K + IDX4(b, c0 + s, h, 0, N, H, dk);
                const double* v = V + IDX4(b, c0 + s, h, 0, N, H, dv);
                double w = exp(bc[L - 1] - bc[s]);
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) Sn[(size_t)i * dv + j] += w * k[i] * v[j];
            }
            double* tmp = S; S = Sn; Sn = tmp;
        }
        if (S_final) memcpy(S_final + (size_t)u * dk * dv, S, sizeof(double) * (size_t)dk * dv);
    }
    free(bc);
    free(Sn);
    free(S);
}

/* Multi-head output (section 2.2, "GroupNorm per head + swish gate"):
 * for each row (one token of one head) of dv values,
 *   mu = mean(y), var = mean((y - mu)^2),
 *   O = (y - mu) / sqrt(var + eps) * g * sigmoid(g).                      */
void oracle_groupnorm_swish(const double* Y, const double* G, long rows, int dv, double eps,
                            double* O) {
    for (long r = 0; r < rows; ++r) {
        const double* y = Y + (size_t)r * dv;
        const double* g = G + (size_t)r * dv;
        double* o = O + (size_t)r * dv;
        double mu = 0.0;
        for (int j = 0; j < dv; ++j) mu += y[j];
        mu /= dv;
        double var = 0.0;
        for (int j = 0; j < dv; ++j) var += (y[j] - mu) * (y[j] - mu);
        var /= dv;
        double rs = 1.0 / sqrt(var + eps);
        for (int j = 0; j < dv; ++j) {
            double sg = 1.0 / (1.0 + exp(-g[j]));
            o[j] = (y[j] - mu) * rs * g[j] * sg;
        }
    }
}

/* One recurrent decode step (section 5.3.7 and "YOCO" Decode): for every
 * (sequence, head) unit, S <- gamma S + k^T v ; y = q S ; o = GN(y) (.) swish(g).
 * q, k [S][H][dk]; v, g, y, o [S][H][dv]; lg [S][H]; S_inout [S][H][dk][dv]. */
void oracle_decode_step(const double* q, const double* k, const double* v, const double* lg,
                        const double* g, double* S_inout, int num_seqs, int H, int dk, int dv,
                        double eps, int u0, int u1, double* y, double* o) {
    (void)num_seqs;
    for (int u = u0; u < u1; ++u) {
        double gm = exp(lg[u]);
        double* S = S_inout + (size_t)u * dk * dv;
        const double* ku = k + (size_t)u * dk;
        const double* qu = q + (size_t)u * dk;
        const double* vu = v + (size_t)u * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = gm * S[(size_t)i * dv + j] + ku[i] * vu[j];
        double* yu = y + (size_t)u * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += qu[i] * S[(size_t)i * dv + j];
            yu[j] = acc;
        }
        oracle_groupnorm_swish(yu, g + (size_t)u * dv, 1, dv, eps, o + (size_t)u * dv);
    }
}

/* Gate projection ("YOCO 深度技术分析", section 2.2: gamma = sigmoid(X W_gamma)^(1/tau),
 * with W_gamma in R^{d x 1} per head -- the Medium-article translation's
 * "门控保留率" paragraph gives the same shape): the gate logit of token n and
 * head h is z[n][h] = sum_i X[n][i] W[i][h].
 *   X [rows][d_model] (rows = B * N tokens), W [d_model][H], z [rows][H]. */
void oracle_gate_project(const double* X, const double* W, long rows, int d_model, int H, double* z) {
    for (long r = 0; r < rows; ++r)
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int i = 0; i < d_model; ++i) acc += X[(size_t)r * d_model + i] * W[(size_t)i * H + h];
            z[(size_t)r * H + h] = acc;
        }
}

/* The rotation Theta of Q and K ("YOCO 深度技术分析" section 2.2:
 * Q = (X W_Q) (.) Theta, K = (X W_K) (.) Theta; the "通用YOCO" page's notes on
 * reproduction: the self-decoder's position encoding is RoPE; section 5.3.6 of
 * the first page: the RoPE base grows 640K -> 5M -> 80M with context).  Theta_n
 * is read as e^{i n theta_j} acting on consecutive pairs of channels taken as
 * complex numbers x_{2j} + i x_{2j+1}, with theta_j = base^(-2j/d):
 *   x'_{2j}   = x_{2j} cos(n theta_j) - x_{2j+1} sin(n theta_j)
 *   x'_{2j+1} = x_{2j} sin(n theta_j) + x_{2j+1} cos(n theta_j)
 * n is the token's position in its sequence (pos0 + index).
 *   X, Xr [B][N][H][d] (d even). */
void oracle_rotate(const double* X, int B, int N, int H, int d, double base, long pos0, double* Xr) {
    for (int b = 0; b < B; ++b)
        for (int n = 0; n < N; ++n)
            for (int h = 0; h < H; ++h) {
                const double* x = X + IDX4(b, n, h, 0, N, H, d);
                double* y = Xr + IDX4(b, n, h, 0, N, H, d);
                for (int j = 0; j < d / 2; ++j) {
                    double theta = pow(base, -2.0 * j / d);
                    double ang = (double)(pos0 + n) * theta;
                    double c = cos(ang), s = sin(ang);
                    y[2 * j] = x[2 * j] * c - x[2 * j + 1] * s;
                    y[2 * j + 1] = x[2 * j] * s + x[2 * j + 1] * c;
                }
            }
}
