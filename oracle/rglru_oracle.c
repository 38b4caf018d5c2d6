/*
 * rglru_oracle.c -- float64 CPU oracle of the RG-LRU recurrent-block core.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the GPU path computes.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg may build, load or call it; the
 * product path never does.  It shares no code, header or constant with the
 * CUDA library.
 *
 * What it computes (one recurrent temporal block's core, conv input to the
 * product with the GELU branch):
 *
 *   Structure -- "Gemma explained: RecurrentGemma architecture"
 *   (gemma.gh.miniasp.com), section "Residual block with recurrent block" and
 *   the RecurrentGemmaRecurrentBlock module printout:
 *     branch B: Conv1d(D, D, kernel_size=4, padding=3, groups=D) then RG-LRU;
 *     branch A: GELU, tanh form (PytorchGELUTanh);
 *     output  : elementwise product of the two branches.
 *   The pages name the RG-LRU module (RecurrentGemmaRglru) but do not print
 *   its equations; they are those of Griffin / RecurrentGemma
 *   ("RecurrentGemma: Moving Past Transformers for Efficient Open Language
 *   Models", arXiv 2404.07839), stated here in full:
 *
 *   1. causal depthwise conv, tap k (0..3) multiplies the input 3-k steps
 *      back; taps that would reach before the current document are dropped:
 *        xc[t,d] = conv_b[d] + sum_k conv_w[k,d] * X[t-3+k,d] * [3-k <= segpos[t]]
 *      X[t] = x[t] for t >= 0 and the carried conv state for t in {-3,-2,-1}.
 *   2. gates, block-diagonal over heads of 256 channels (W[h][out][in]):
 *        r = sigmoid(W_a[h] xc_h + b_a),  i = sigmoid(W_x[h] xc_h + b_x)
 *   3. decay  a = sigmoid(Lambda)^(c*r)  = exp(c * r * log sigmoid(Lambda))
 *   4. scan   h_t = a_t h_{t-1} + sqrt(1 - a_t^2) * (i_t * xc_t),
 *      except where segpos == 0 (document start): h_t = i_t * xc_t.
 *   5. y = GELU_tanh(g) * h,
 *        GELU_tanh(g) = 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3))).
 *   6. carried state out: h at the last token, conv state = the last three
 *      raw inputs X[T-3], X[T-2], X[T-1] (oldest first).
 *
 * Layouts (row-major, channel fastest): x, g, y [B,T,D]; conv_w [4,D];
 * conv_b, b_a, b_x, lambda [D]; W_a, W_x [H,256,256]; segpos [B,T];
 * conv_state [B,3,D]; h_state [B,D].  D must be a multiple of 256.
 *
 * Optional trace arrays (each [B,T,D], NULL to skip) record xc, r, i, a and
 * h per element so that the tests can pin each step separately.
 *
 * gate_bf16 = 1 evaluates step 2 on the conv output rounded to bf16 (the
 * operand precision of the tensor-core gate projections in bf16 I/O mode);
 * 0, the default everywhere else, keeps it exact.
 *
 * Independent units are the (batch row, head) pairs: heads never mix
 * (depthwise conv, block-diagonal gates, per-channel scan).  OpenMP runs the
 * units in parallel; inside a unit tokens run strictly in order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define HEAD 256

/* log sigmoid(v) = -softplus(-v), written in the branch that cannot overflow. */
static double log_sigmoid(double v)
{
    if (v >= 0.0)
        return -log1p(exp(-v));
    return v - log1p(exp(v));
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* Nearest bf16 value (8 significant bits, ties to even) of v.  Used only
 * when the caller asks for the gate projections in the precision of bf16
 * I/O mode, where the tensor-core gate GEMM takes bf16 operands: the
 * conv output enters the dot products rounded to bf16 (the scan and every
 * other step keep it exact). */
static double round_bf16(double v)
{
    if (v == 0.0 || !isfinite(v))
        return v;
    int e;
    const double m = frexp(v, &e);        /* v = m 2^e, 0.5 <= |m| < 1 */
    return ldexp(nearbyint(ldexp(m, 8)), e - 8);
}

static double gelu_tanh(double g)
{
    const double k = sqrt(2.0 / M_PI);
    return 0.5 * g * (1.0 + tanh(k * (g + 0.044715 * g * g * g)));
}

int rglru_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Returns 0 on success, -1 on a bad argument. */
int rglru_oracle_prefill(int B, int T, int D, double c,
                         const double *x, const double *g,
                         const double *conv_w, const double *conv_b,
                         const double *W_a, const double *b_a,
                         const double *W_x, const double *b_x,
                         const double *lambda, const int32_t *segpos,
                         double *conv_state, double *h_state, double *y,
                         double *tr_xc, double *tr_r, double *tr_i,
                         double *tr_a, double *tr_h, int nthreads, int gate_bf16)
{
    if (B < 1 || T < 1 || D < HEAD || D % HEAD != 0)
        return -1;
    const int H = D / HEAD;
    const int64_t TD = (int64_t)T * D;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        for (int hd = 0; hd < H; ++hd) {
            const int d0 = hd * HEAD;
            const double *xb = x + b * TD;
            const double *gb = g + b * TD;
            const int32_t *sp = segpos + (int64_t)b * T;
            double *cs = conv_state + (int64_t)b * 3 * D;
            double xc[HEAD], xg[HEAD], h[HEAD], newcs[3][HEAD];

            for (int j = 0; j < HEAD; ++j)
                h[j] = h_state[(int64_t)b * D + d0 + j];

            for (int t = 0; t < T; ++t) {
                const int pos = sp[t];
                /* step 1: causal depthwise conv with the document mask */
                for (int j = 0; j < HEAD; ++j) {
                    const int d = d0 + j;
                    double acc = conv_b[d];
                    for (int k = 0; k < 4; ++k) {
                        const int lag = 3 - k;
                        if (lag > pos)
                            continue;
                        const int ts = t - lag;
                        const double xv = ts >= 0 ? xb[(int64_t)ts * D + d]
                                                  : cs[(3 + ts) * D + d];
                        acc += conv_w[k * D + d] * xv;
                    }
                    xc[j] = acc;
                    xg[j] = gate_bf16 ? round_bf16(acc) : acc;
                }
                /* steps 2-5 per output channel j of this head */
                for (int j = 0; j < HEAD; ++j) {
                    const int d = d0 + j;
                    const double *wa = W_a + ((int64_t)hd * HEAD + j) * HEAD;
                    const double *wx = W_x + ((int64_t)hd * HEAD + j) * HEAD;
                    double pr = b_a[d], pi = b_x[d];
                    for (int q = 0; q < HEAD; ++q) {
                        pr += wa[q] * xg[q];
                        pi += wx[q] * xg[q];
                    }
                    const double r = sigmoid(pr);
                    const double ig = sigmoid(pi);
                    const double ell = c * r * log_sigmoid(lambda[d]);
                    const double a = exp(ell);
                    if (pos == 0)
                        h[j] = ig * xc[j];
                    else
                        h[j] = a * h[j] + sqrt(-expm1(2.0 * ell)) * (ig * xc[j]);
                    const int64_t e = (int64_t)t * D + d;
                    y[b * TD + e] = gelu_tanh(gb[e]) * h[j];
                    if (tr_xc) tr_xc[b * TD + e] = xc[j];
                    if (tr_r) tr_r[b * TD + e] = r;
                    if (tr_i) tr_i[b * TD + e] = ig;
                    if (tr_a) tr_a[b * TD + e] = a;
                    if (tr_h) tr_h[b * TD + e] = h[j];
                }
            }
            /* step 6: carried state out (new rows computed before writing) */
            for (int k = 0; k < 3; ++k) {
                const int ts = T - 3 + k;
                for (int j = 0; j < HEAD; ++j) {
                    const int d = d0 + j;
                    newcs[k][j] = ts >= 0 ? xb[(int64_t)ts * D + d] : cs[(3 + ts) * D + d];
                }
            }
            for (int k = 0; k < 3; ++k)
                for (int j = 0; j < HEAD; ++j)
                    cs[k * D + d0 + j] = newcs[k][j];
            for (int j = 0; j < HEAD; ++j)
                h_state[(int64_t)b * D + d0 + j] = h[j];
        }
    }
    return 0;
}
