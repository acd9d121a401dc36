/*
 * Gated DeltaNet token mixer: plain CPU oracle in double precision.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) includes, links or calls this file; only the tests, the
 * smoke check and the benchmark's CPU-baseline leg do.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * What it computes (one sequence, one value head, token by token, in the
 * order the method states it):
 *
 *   Qwen3.8 27B model card (Nestmodels for Linnet), "Gated DeltaNet" bullet:
 *     one projection gives q (16 heads), k (16 heads) and v (48 heads), each
 *     128 wide; a depthwise causal conv of width 4 followed by silu runs over
 *     them; q and k are L2-normalised; each value head keeps a [128,128]
 *     state that the gated delta rule decays by exp(-exp(A_log)*softplus(a +
 *     dt_bias)) and writes at rate sigmoid(b); the heads' outputs are
 *     RMS-normalised and gated by silu(z).
 *   Same card, "Norms" bullet: RMS norms scale by (1 + w), in f32 (here f64).
 *   Same card, cache paragraph: each row keeps its conv history and its
 *     recurrent state between calls.
 *   Qwen/Qwen3.8-27B architecture page, header table: norm eps 1e-06.
 *
 * Readings where the pages are silent (each one is also listed in the design
 * notes):
 *   - channel order of the fused projection is [q | k | v], heads contiguous;
 *   - value head h reads q/k head h / (Vh / Kh) (contiguous groups);
 *   - conv is a cross-correlation: tap W-1 multiplies the current token, tap 0
 *     the token W-1 steps back; missing history is zero; no conv bias (the
 *     module tree lists 10240x1x4 = 40,960 conv parameters, 41.0K);
 *   - L2 norm is x / sqrt(sum x^2 + eps) with the same eps;
 *   - the read-out uses the updated state and q / sqrt(Dk);
 *   - the gated norm is o * rsqrt(mean(o^2) + eps) * (1 + w) * silu(z), one
 *     weight vector of length Dv shared by all heads.
 *
 * Recurrence (per token, state S is [Dv rows][Dk cols], row i belongs to
 * value channel i):
 *   alpha = exp(g),  r = S k,  u = beta * (v - alpha * r),
 *   S <- alpha * S + u k^T,    o = S q.
 *
 * Build: gcc -O3 -fopenmp -shared -fPIC gdn_oracle.c -o libgdn_oracle.so -lm
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- scalar pieces ------------------------------------------------------ */

double oracle_silu(double x) { return x / (1.0 + exp(-x)); }

double oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* softplus(x) = log(1 + e^x), written without overflow and without a cut-off. */
double oracle_softplus(double x) { return fmax(x, 0.0) + log1p(exp(-fabs(x))); }

/* Gates of one token and one value head (model card, "Gated DeltaNet" bullet):
 *   g    = -exp(A_log) * softplus(a + dt_bias)   (log of the decay factor)
 *   beta = sigmoid(b)                             (write rate)            */
void oracle_gates(double A_log, double dt_bias, double a, double b, double* g, double* beta)
{
    *g = -exp(A_log) * oracle_softplus(a + dt_bias);
    *beta = oracle_sigmoid(b);
}

/* Depthwise causal conv of one channel at one position: taps xw[0..W-1] run
 * from the oldest (W-1 tokens back) to the current token; result before silu. */
double oracle_conv_tap(int W, const double* xw, const double* w)
{
    double acc = 0.0;
    for (int j = 0; j < W; ++j) acc += w[j] * xw[j];
    return acc;
}

/* One channel over a whole sequence: xbar holds the W-1 history values
 * (oldest first) followed by the L inputs; c[s] = sum_j w[j] * xbar[s + j]. */
void oracle_causal_conv(int L, int W, const double* xbar, const double* w, double* c)
{
    for (int s = 0; s < L; ++s) c[s] = oracle_conv_tap(W, xbar + s, w);
}

/* y = x / sqrt(sum x^2 + eps) */
void oracle_l2norm(int n, const double* x, double eps, double* y)
{
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < n; ++i) y[i] = x[i] * r;
}

/* One token of the gated delta rule on state S [Dv][Dk]; writes o [Dv]. */
void oracle_delta_rule_step(int Dk, int Dv, const double* q, const double* k, const double* v,
                            double g, double beta, double* S, double* o)
{
    double alpha = exp(g);
    for (int i = 0; i < Dv; ++i) {
        double* Si = S + (size_t)i * Dk;
        double r = 0.0;
        for (int j = 0; j < Dk; ++j) r += Si[j] * k[j];
        double u = beta * (v[i] - alpha * r);
        double oi = 0.0;
        for (int j = 0; j < Dk; ++j) {
            Si[j] = alpha * Si[j] + u * k[j];
            oi += Si[j] * q[j];
        }
        o[i] = oi;
    }
}

/* The recurrence over T tokens on prepared inputs: q,k [T][Dk], v [T][Dv],
 * g, beta [T]; S [Dv][Dk] in/out; o [T][Dv]. */
void oracle_delta_rule(int T, int Dk, int Dv, const double* q, const double* k, const double* v,
                       const double* g, const double* beta, double* S, double* o)
{
    for (int t = 0; t < T; ++t)
        oracle_delta_rule_step(Dk, Dv, q + (size_t)t * Dk, k + (size_t)t * Dk, v + (size_t)t * Dv,
                               g[t], beta[t], S, o + (size_t)t * Dv);
}

/* Zero-centred gated RMSNorm of one head: y = o * rsqrt(mean(o^2)+eps) * (1+w) * silu(z). */
void oracle_gated_rmsnorm(int D, const double* o, const double* z, const double* w, double eps, double* y)
{
    double ms = 0.0;
    for (int i = 0; i < D; ++i) ms += o[i] * o[i];
    ms /= (double)D;
    double r = 1.0 / sqrt(ms + eps);
    for (int i = 0; i < D; ++i) y[i] = o[i] * r * (1.0 + w[i]) * oracle_silu(z[i]);
}

/* ---- the whole mixer ---------------------------------------------------- */

/*
 * Packed (varlen) prefill over N rows; row n owns tokens [cu[n], cu[n+1]).
 * Decode is the special case of rows of length 1.
 *
 *   qkv  [total][C]       C = (2*Kh + Vh) * D, channel order [q | k | v]
 *   z    [total][Vh*D]
 *   a, b [total][Vh]
 *   conv_w [C][W];  A_log, dt_bias [Vh];  norm_w [D]
 *   init_state [N][Vh][D][D] or NULL (zeros);  init_conv [N][W-1][C] or NULL
 *   Value heads [h_lo, h_hi) are computed; outputs are indexed by h - h_lo:
 *   out [total][(h_hi-h_lo)*D] (may be NULL), final_state [N][h_hi-h_lo][D][D]
 *   (may be NULL), final_conv [N][W-1][C] (may be NULL; covers all channels).
 * Returns 0, or -1 on inconsistent arguments.
 */
int oracle_mixer(int Kh, int Vh, int D, int W, int N, const int64_t* cu,
                 const double* qkv, const double* z, const double* a, const double* b,
                 const double* conv_w, const double* A_log, const double* dt_bias, const double* norm_w,
                 const double* init_state, const double* init_conv,
                 int h_lo, int h_hi, double eps,
                 double* out, double* final_state, double* final_conv, int nthreads)
{
    if (Kh <= 0 || Vh <= 0 || D <= 0 || W <= 0 || N < 0 || Vh % Kh != 0) return -1;
    if (h_lo < 0 || h_hi > Vh || h_lo > h_hi) return -1;
    for (int n = 0; n < N; ++n)
        if (cu[n + 1] < cu[n]) return -1;
    const int C = (2 * Kh + Vh) * D;
    const int H = h_hi - h_lo;
    const int group = Vh / Kh;
    const int Hm = W - 1;
    const double qscale = 1.0 / sqrt((double)D);

    /* Final conv history of every row: the last W-1 rows of [history; inputs]. */
    if (final_conv) {
        for (int n = 0; n < N; ++n) {
            int64_t L = cu[n + 1] - cu[n];
            for (int r = 0; r < Hm; ++r) {
                int64_t e = L + r; /* index into xbar = [history (W-1 rows); inputs] */
                double* dst = final_conv + ((size_t)n * Hm + r) * C;
                for (int ch = 0; ch < C; ++ch) {
                    double x;
                    if (e < Hm) x = init_conv ? init_conv[((size_t)n * Hm + e) * C + ch] : 0.0;
                    else x = qkv[(size_t)(cu[n] + e - Hm) * C + ch];
                    dst[ch] = x;
                }
            }
        }
    }

    const long long jobs = (long long)N * H;
    int err = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (long long job = 0; job < jobs; ++job) {
        const int n = (int)(job / H);
        const int h = h_lo + (int)(job % H);
        const int kap = h / group;
        const int chq = kap * D, chk = Kh * D + kap * D, chv = 2 * Kh * D + h * D;
        const int64_t t0 = cu[n];
        const int64_t L = cu[n + 1] - cu[n];

        double* S = (double*)malloc(sizeof(double) * (size_t)D * D);
        double* buf = (double*)malloc(sizeof(double) * (size_t)(8 * D + 2 * W));
        if (!S || !buf) { free(S); free(buf); err = 1; continue; }
        double *q = buf, *k = buf + D, *v = buf + 2 * D, *o = buf + 3 * D, *y = buf + 4 * D;
        double *zz = buf + 5 * D, *pre = buf + 6 * D, *xw = buf + 8 * D;

        if (init_state) memcpy(S, init_state + ((size_t)n * Vh + h) * D * D, sizeof(double) * D * D);
        else memset(S, 0, sizeof(double) * D * D);

        for (int64_t s = 0; s < L; ++s) {
            const int64_t tok = t0 + s;
            /* conv + silu over the head's q, k and v channels */
            const int bases[3] = {chq, chk, chv};
            double* dsts[3] = {q, k, v};
            for (int grp = 0; grp < 3; ++grp) {
                for (int c = 0; c < D; ++c) {
                    const int ch = bases[grp] + c;
                    for (int j = 0; j < W; ++j) {
                        int64_t e = s + j;
                        if (e < Hm) xw[j] = init_conv ? init_conv[((size_t)n * Hm + e) * C + ch] : 0.0;
                        else xw[j] = qkv[(size_t)(t0 + e - Hm) * C + ch];
                    }
                    dsts[grp][c] = oracle_silu(oracle_conv_tap(W, xw, conv_w + (size_t)ch * W));
                }
            }
            /* L2 norm of q and k; q then scaled by 1/sqrt(D) */
            oracle_l2norm(D, q, eps, pre);
            for (int c = 0; c < D; ++c) q[c] = pre[c] * qscale;
            oracle_l2norm(D, k, eps, pre);
            for (int c = 0; c < D; ++c) k[c] = pre[c];
            /* gates */
            double g, beta;
            oracle_gates(A_log[h], dt_bias[h], a[(size_t)tok * Vh + h], b[(size_t)tok * Vh + h], &g, &beta);
            /* recurrence and read-out */
            oracle_delta_rule_step(D, D, q, k, v, g, beta, S, o);
            /* gated RMSNorm */
            if (out) {
                for (int c = 0; c < D; ++c) zz[c] = z[(size_t)tok * Vh * D + (size_t)h * D + c];
                oracle_gated_rmsnorm(D, o, zz, norm_w, eps, y);
                memcpy(out + (size_t)tok * H * D + (size_t)(h - h_lo) * D, y, sizeof(double) * D);
            }
        }
        if (final_state) memcpy(final_state + ((size_t)n * H + (h - h_lo)) * D * D, S, sizeof(double) * D * D);
        free(S);
        free(buf);
    }
    return err ? -2 : 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
