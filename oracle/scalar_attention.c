/*
 * Second, independent fp64 oracle: scalar loops in plain C.
 *
 * TEST INFRASTRUCTURE. It is compiled into oracle/_scalar_attention.so and
 * called only by the test suite, to pin the numpy oracle on small inputs. It
 * shares no code with the numpy oracle or with the CUDA library.
 *
 * It evaluates the attention definition of "Flash Attention V2核心网络算子解析"
 * §二.1 (softmax(Q Kᵀ · scale) V) with the causal / (left, right) window masks of
 * "FlashAttention技术解析：加速GPT训练的核心优化" §2.2, one query row at a time,
 * and the gradients of L = sum(dO * O) by the chain rule written out per element.
 *
 * Layout: q, k, v, dout, o, dq, dk, dv are (B, N, H, d) row-major doubles;
 * lse is (B, H, N). Window bounds are inclusive; -1 means unbounded; causal
 * forces the right bound to 0. Returns 0, or -1 on invalid sizes.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static long idx4(int b, int n, int h, int c, int N, int H, int d) {
    return (((long)b * N + n) * H + h) * (long)d + c;
}

static int key_visible(int i, int j, int causal, int win_l, int win_r) {
    int right = causal ? 0 : win_r;
    if (win_l >= 0 && j < i - win_l) return 0;
    if (right >= 0 && j > i + right) return 0;
    return 1;
}

/* Scores of row i (scaled, -inf where masked) and their max; returns the max. */
static double row_scores(const double* q, const double* k, int b, int h, int i, int N, int H, int d,
                         double scale, int causal, int win_l, int win_r, double* s) {
    double mx = -INFINITY;
    for (int j = 0; j < N; ++j) {
        if (!key_visible(i, j, causal, win_l, win_r)) { s[j] = -INFINITY; continue; }
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += q[idx4(b, i, h, c, N, H, d)] * k[idx4(b, j, h, c, N, H, d)];
        s[j] = scale * acc;
        if (s[j] > mx) mx = s[j];
    }
    return mx;
}

/* Softmax probabilities of row i into p; returns the natural-log LSE. */
static double row_probs(const double* q, const double* k, int b, int h, int i, int N, int H, int d,
                        double scale, int causal, int win_l, int win_r, double* p) {
    double mx = row_scores(q, k, b, h, i, N, H, d, scale, causal, win_l, win_r, p);
    if (mx == -INFINITY) {
        for (int j = 0; j < N; ++j) p[j] = 0.0;
        return -INFINITY;
    }
    double sum = 0.0;
    for (int j = 0; j < N; ++j) { p[j] = exp(p[j] - mx); sum += p[j]; }
    for (int j = 0; j < N; ++j) p[j] /= sum;
    return mx + log(sum);
}

int scalar_attention_fwd(const double* q, const double* k, const double* v, double* o, double* lse,
                         int B, int N, int H, int d, double scale, int causal, int win_l, int win_r) {
    if (B <= 0 || N <= 0 || H <= 0 || d <= 0) return -1;
    double* p = (double*)malloc(sizeof(double) * (size_t)N);
    if (!p) return -1;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < N; ++i) {
                lse[((long)b * H + h) * N + i] = row_probs(q, k, b, h, i, N, H, d, scale, causal, win_l, win_r, p);
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < N; ++j) acc += p[j] * v[idx4(b, j, h, c, N, H, d)];
                    o[idx4(b, i, h, c, N, H, d)] = acc;
                }
            }
    free(p);
    return 0;
}

/*
 * Per row i: dP_ij = sum_c dO_ic V_jc; D_i = sum_j P_ij dP_ij; dS_ij = P_ij (dP_ij - D_i);
 * dQ_i += scale * sum_j dS_ij K_j; dK_j += scale * dS_ij Q_i; dV_j += P_ij dO_i.
 */
int scalar_attention_bwd(const double* q, const double* k, const double* v, const double* dout,
                         double* dq, double* dk, double* dv,
                         int B, int N, int H, int d, double scale, int causal, int win_l, int win_r) {
    if (B <= 0 || N <= 0 || H <= 0 || d <= 0) return -1;
    size_t total = (size_t)B * N * H * d;
    memset(dq, 0, sizeof(double) * total);
    memset(dk, 0, sizeof(double) * total);
    memset(dv, 0, sizeof(double) * total);
    double* p = (double*)malloc(sizeof(double) * (size_t)N);
    double* dp = (double*)malloc(sizeof(double) * (size_t)N);
    if (!p || !dp) { free(p); free(dp); return -1; }
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int i = 0; i < N; ++i) {
                row_probs(q, k, b, h, i, N, H, d, scale, causal, win_l, win_r, p);
                double D = 0.0;
                for (int j = 0; j < N; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += dout[idx4(b, i, h, c, N, H, d)] * v[idx4(b, j, h, c, N, H, d)];
                    dp[j] = acc;
                    D += p[j] * acc;
                }
                for (int j = 0; j < N; ++j) {
                    if (p[j] == 0.0) continue;
                    double ds = p[j] * (dp[j] - D);
                    for (int c = 0; c < d; ++c) {
                        dq[idx4(b, i, h, c, N, H, d)] += scale * ds * k[idx4(b, j, h, c, N, H, d)];
                        dk[idx4(b, j, h, c, N, H, d)] += scale * ds * q[idx4(b, i, h, c, N, H, d)];
                        dv[idx4(b, j, h, c, N, H, d)] += p[j] * dout[idx4(b, i, h, c, N, H, d)];
                    }
                }
            }
    free(p);
    free(dp);
    return 0;
}
