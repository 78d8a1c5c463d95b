/*
 * ssd_oracle.c -- fp64 CPU oracle for the Mamba-2 SSD selective scan.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct definition
 * that the CUDA library is checked against.  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark may load it.  It shares no code,
 * header or constant with the CUDA library (mamba_ssd_b200/csrc).
 *
 * Sources (page title, then section):
 *   [abstract] "Compiler-First State Space Duality and Portable O(1) Autoregressive
 *              Caching for Inference" (Santoni), abstract: diagonal per-head
 *              dynamics, Mamba-2 checkpoint parity.
 *   [blog §x.y] the article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn news 991632)
 *              that walks through the same paper, section x.y:
 *              §1.1 diagonal state, discretisation, chunking, decay mask;
 *              §2.1 constant-size state and the sliding-window conv cache;
 *              §2.2 the cache update (conv window roll+set, ssm = ssm*A_bar + B_bar*x);
 *              §3.2 / §4.1 the decay and state update in float32 (here: float64).
 *
 * Readings where the pages are silent or garbled:
 *   - A = -exp(A_log) per head and the softplus applies to dt, not to A_log: the blog's
 *     printed exp(softplus(A_log)*dt) has lost its sign (a positive exponent would make
 *     the state grow without bound) and the abstract claims checkpoint parity with
 *     Mamba-2, whose discretisation is dA = dt * (-exp(A_log)).
 *   - dt = clip(softplus(dt_raw + dt_bias), dt_min, dt_max); the clipped dt is used
 *     both in the decay exp(dt*A) and in B_bar = dt*B (Euler form of the blog §2.2
 *     "B_bar").
 *   - y_t reads the state after the update at step t (inclusive diagonal), plus the
 *     per-head skip D[h]*x_t.
 *   - heads map to groups in contiguous blocks: g = h / (H/G).
 *   - decode conv: the cache holds the K-1 most recent raw inputs, oldest first; the
 *     weight tap K-1 multiplies the newest input; bias, then SiLU; the xBC channel
 *     order is [x | B | C].
 *
 * Every routine is plain loops in double precision.  OpenMP only splits independent
 * (batch, head) recurrences across threads; the arithmetic per recurrence is the
 * sequential definition, in order.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Thread control, so that a timed run can state how many host threads it used. */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* softplus(z) = log(1 + e^z).  For z > 30 the identity z + log1p(e^-z) avoids
 * overflow of e^z; it is the same real number. */
static double sp(double z) { return z > 30.0 ? z + log1p(exp(-z)) : log1p(exp(z)); }

static double clip(double v, double lo, double hi) { return v < lo ? lo : (v > hi ? hi : v); }

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Discretised step size of [blog §1.1]/[blog §4.1] with the sign reading above. */
double oracle_dt(double dt_raw, double bias, double dt_min, double dt_max)
{
    return clip(sp(dt_raw + bias), dt_min, dt_max);
}

/*
 * Sequential recurrence, token by token ([blog §1.1] diagonal state, [blog §2.2] the
 * update ssm = ssm*A_bar + B_bar*x):
 *     dt_t = clip(softplus(dt_raw[b,t,h] + dt_bias[h]), dt_min, dt_max)
 *     a_t  = exp(dt_t * (-exp(A_log[h])))
 *     h    = a_t * h + dt_t * x[b,t,h,:] (outer) B[b,t,g,:]        (P x N)
 *     y[b,t,h,p] = sum_n h[p,n] * C[b,t,g,n] + D[h] * x[b,t,h,p]
 * Layouts (row-major): x,y [B,L,H,P]; dt_raw [B,L,H]; Bm,Cm [B,L,G,N];
 * h0,h_final [B,H,P,N].  D, dt_bias, h0 may be NULL (zeros); h_final may be NULL.
 */
void oracle_ssd_scan_seq(int B, int L, int H, int P, int G, int N,
                         const double *x, const double *dt_raw, const double *A_log,
                         const double *Bm, const double *Cm, const double *D,
                         const double *dt_bias, double dt_min, double dt_max,
                         const double *h0, double *y, double *h_final)
{
    const int heads_per_group = H / G;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const int g = h / heads_per_group;
            const double A = -exp(A_log[h]);
            const double bias = dt_bias ? dt_bias[h] : 0.0;
            const double skip = D ? D[h] : 0.0;
            double *st = (double *)malloc(sizeof(double) * (size_t)P * N);
            for (int i = 0; i < P * N; ++i)
                st[i] = h0 ? h0[((size_t)b * H + h) * P * N + i] : 0.0;
            for (int t = 0; t < L; ++t) {
                const size_t bt = (size_t)b * L + t;
                const double dt = oracle_dt(dt_raw[bt * H + h], bias, dt_min, dt_max);
                const double a = exp(dt * A);
                const double *xt = x + (bt * H + h) * P;
                const double *Bt = Bm + (bt * G + g) * N;
                const double *Ct = Cm + (bt * G + g) * N;
                double *yt = y + (bt * H + h) * P;
                for (int p = 0; p < P; ++p) {
                    double *row = st + (size_t)p * N;
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) {
                        row[n] = a * row[n] + dt * xt[p] * Bt[n];
                        acc += row[n] * Ct[n];
                    }
                    yt[p] = acc + skip * xt[p];
                }
            }
            if (h_final)
                memcpy(h_final + ((size_t)b * H + h) * P * N, st, sizeof(double) * (size_t)P * N);
            free(st);
        }
    }
}

/*
 * Causal depthwise conv1d + bias + SiLU over a whole sequence ([blog §2.1] sliding
 * window conv), zero left padding:
 *     out[b,t,c] = SiLU( sum_k w[c,k] * xBC[b, t-(K-1)+k, c] + bias[c] )
 * and the cache left behind, conv_state[b,c,j] = xBC[b, L-(K-1)+j, c] (0 if before
 * the start), oldest first.  xBC,out [B,L,Cc]; w [Cc,K]; bias [Cc] or NULL;
 * conv_state [B,Cc,K-1] or NULL.
 */
void oracle_causal_conv1d(int B, int L, int Cc, int K, const double *xBC, const double *w,
                          const double *bias, double *out, double *conv_state)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int c = 0; c < Cc; ++c) {
            for (int t = 0; t < L; ++t) {
                double acc = bias ? bias[c] : 0.0;
                for (int k = 0; k < K; ++k) {
                    const int s = t - (K - 1) + k;
                    if (s >= 0) acc += w[(size_t)c * K + k] * xBC[((size_t)b * L + s) * Cc + c];
                }
                out[((size_t)b * L + t) * Cc + c] = silu(acc);
            }
            if (conv_state) {
                for (int j = 0; j < K - 1; ++j) {
                    const int s = L - (K - 1) + j;
                    conv_state[((size_t)b * Cc + c) * (K - 1) + j] =
                        s >= 0 ? xBC[((size_t)b * L + s) * Cc + c] : 0.0;
                }
            }
        }
    }
}

/*
 * One cached decode step ([blog §2.1] O(1) state, [blog §2.2] Mamba2Cache.update):
 *   window = [conv_state[b,c,0..K-2], xBC_t[b,c]]          (oldest .. newest)
 *   u[c]   = SiLU( sum_k w[c,k] * window[k] + bias[c] )
 *   conv_state[b,c,:] = window[1..K-1]                       (roll, then set newest)
 *   split u into x [H*P] | B [G*N] | C [G*N]
 *   dt = clip(softplus(dt_t[b,h] + dt_bias[h])), a = exp(dt * (-exp(A_log[h])))
 *   ssm[b,h] = a * ssm[b,h] + dt * x_h (outer) B_g
 *   y_t[b,h,p] = sum_n ssm[b,h,p,n] * C_g[n] + D[h] * x_h[p]
 * Cc = H*P + 2*G*N.  ssm_state [B,H,P,N] and conv_state [B,Cc,K-1] are updated in
 * place.  conv_b, D, dt_bias may be NULL.
 */
void oracle_decode_step(int B, int H, int P, int G, int N, int K,
                        double *ssm_state, double *conv_state,
                        const double *xBC_t, const double *dt_t, const double *A_log,
                        const double *D, const double *dt_bias, double dt_min, double dt_max,
                        const double *conv_w, const double *conv_b, double *y_t)
{
    const int Cc = H * P + 2 * G * N;
    const int heads_per_group = H / G;
    for (int b = 0; b < B; ++b) {
        double *u = (double *)malloc(sizeof(double) * (size_t)Cc);
        for (int c = 0; c < Cc; ++c) {
            double *cs = conv_state + ((size_t)b * Cc + c) * (K - 1);
            const double newest = xBC_t[(size_t)b * Cc + c];
            double acc = conv_b ? conv_b[c] : 0.0;
            for (int k = 0; k < K; ++k) {
                const double v = (k < K - 1) ? cs[k] : newest;
                acc += conv_w[(size_t)c * K + k] * v;
            }
            u[c] = silu(acc);
            for (int j = 0; j + 1 < K - 1; ++j) cs[j] = cs[j + 1];
            if (K > 1) cs[K - 2] = newest;
        }
        const double *xs = u;
        const double *Bs = u + H * P;
        const double *Cs = u + H * P + G * N;
        for (int h = 0; h < H; ++h) {
            const int g = h / heads_per_group;
            const double dt = oracle_dt(dt_t[(size_t)b * H + h], dt_bias ? dt_bias[h] : 0.0,
                                        dt_min, dt_max);
            const double a = exp(dt * (-exp(A_log[h])));
            for (int p = 0; p < P; ++p) {
                double *row = ssm_state + (((size_t)b * H + h) * P + p) * N;
                const double xp = xs[h * P + p];
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    row[n] = a * row[n] + dt * xp * Bs[g * N + n];
                    acc += row[n] * Cs[g * N + n];
                }
                y_t[((size_t)b * H + h) * P + p] = acc + (D ? D[h] : 0.0) * xp;
            }
        }
        free(u);
    }
}
