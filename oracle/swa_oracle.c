/*
 * swa_oracle.c -- plain fp64 CPU definition of the gated sliding-window
 * attention core (GatedSWA without its projections).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * Sources (pages about ZGCM-1):
 *  [P1] "7.39B 오픈 모델로 256K 문맥의 수학 추론과 에이전트 검색을 겨냥한
 *       ZGCM-1" (onedev.kr), section "어떻게 동작하나" (how it works):
 *       GatedSWA(h) = o_proj(A_SWA(q,k,v) ⊙ σ(g_proj(h))); 32 query heads,
 *       8 KV heads, head dim 128; 128-token window; QK normalisation is
 *       RMSNorm; partial RoPE with rotary fraction 0.33; the gate modulates
 *       the local attention output element by element.
 *  [P3] "ZGCM-1: A Fully Open and Extremely Efficient Foundation Model for
 *       Math and Agentic Search" (jaehun.me), section "How Gated SWA
 *       Behaves": RMS normalisation then partial RoPE on q and k; A_SWA is the
 *       GQA output inside the window; the worked example shows that a token
 *       sees a window that includes itself.
 *  [P1] section "무엇과 다른가": RoPE base 10M at the 256K stage.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - rot_dim R = 42 (0.33 x 128 rounded to an even count); the first R dims
 *    rotate in rotate-half pairs (j, j + R/2), j < R/2, by the angle
 *    p * base^(-2j/R); dims R..D-1 pass through.
 *  - RMSNorm per head over D dims: y = x / sqrt(mean(x^2) + eps) * w, one
 *    weight vector for q and one for k, shared across heads; norm first,
 *    then RoPE.
 *  - score scale 1/sqrt(D) unless given; query i sees keys
 *    max(0, i-W+1) .. i; q head h reads kv head h / (Hq/Hkv).
 *  - sigma(g) = 1 / (1 + exp(-g)), the gate is per output element.
 *  - prefill positions are pos0 + t; in decode a ring of W slots holds
 *    position p - ((p - s) mod W) in slot s (valid when >= 0); slot p mod W
 *    is first overwritten with the new k (after norm and RoPE, rounded to
 *    bf16) and the new v.
 *
 * All arithmetic is IEEE fp64 in the order written; no blocking, fusion or
 * reordering beyond the definition.  Inputs arrive as fp64 arrays (bf16
 * values upcast exactly by the caller), row-major [B, T, H, D].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX4(b, t, h, d, T, H, D) ((((int64_t)(b) * (T) + (t)) * (H) + (h)) * (D) + (d))

/* ---------------------------------------------------------------- pieces */

/* RMSNorm of one head vector x[D] with weight w[D] ([P1] QK-RMSNorm).
 * Writes xhat = x / r (before the weight) and y = xhat * w; returns r. */
static double rms_norm(const double *x, const double *w, int D, double eps,
                       double *xhat, double *y) {
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    double r = sqrt(ss / D + eps);
    for (int d = 0; d < D; ++d) {
        xhat[d] = x[d] / r;
        y[d] = xhat[d] * w[d];
    }
    return r;
}

/* Partial RoPE in place on y[D] at position p ([P1] partial RoPE). */
static void rope_apply(double *y, int R, double base, double p) {
    int half = R / 2;
    for (int j = 0; j < half; ++j) {
        double theta = p * pow(base, -2.0 * j / R);
        double c = cos(theta), s = sin(theta);
        double a = y[j], b = y[j + half];
        y[j] = a * c - b * s;
        y[j + half] = b * c + a * s;
    }
}

/* Transpose of the rotation (rotation by -theta), for the chain rule. */
static void rope_apply_transpose(double *dy, int R, double base, double p) {
    int half = R / 2;
    for (int j = 0; j < half; ++j) {
        double theta = p * pow(base, -2.0 * j / R);
        double c = cos(theta), s = sin(theta);
        double a = dy[j], b = dy[j + half];
        dy[j] = a * c + b * s;
        dy[j + half] = b * c - a * s;
    }
}

static double sigmoid(double g) { return 1.0 / (1.0 + exp(-g)); }

static double dot(const double *a, const double *b, int D) {
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/* Round an fp64 value to the nearest bf16 (ties to even) and return its bits.
 * bf16 keeps 8 significant bits; the grid spacing in the binade of x is
 * 2^(e-8) where x = m * 2^e, 0.5 <= |m| < 1, floored at the smallest
 * subnormal 2^-133. */
uint16_t oracle_bf16_bits(double x) {
    if (isnan(x)) return 0x7FC0;
    if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
    if (isinf(x)) return x > 0 ? 0x7F80 : 0xFF80;
    int e;
    frexp(x, &e);
    int qe = e - 8;
    if (qe < -133) qe = -133;
    double q = ldexp(1.0, qe);
    double r = nearbyint(x / q) * q; /* default rounding mode: ties to even */
    if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, x);
    float f = (float)r; /* exact: r lies on the bf16 grid */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

double oracle_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* ------------------------------------------------------------ norm + rope */

/* y[rows, H, D] = RoPE(RMSNorm(x, w), pos[row]).  Exposed so tests can check
 * the two steps on their own and fill decode rings. */
void oracle_norm_rope(int64_t rows, int H, int D, int R, double base, double eps,
                      const double *x, const double *w, const double *pos,
                      double *y) {
    double *xhat = (double *)malloc(sizeof(double) * D);
    for (int64_t r = 0; r < rows; ++r)
        for (int h = 0; h < H; ++h) {
            const double *xr = x + (r * H + h) * D;
            double *yr = y + (r * H + h) * D;
            rms_norm(xr, w, D, eps, xhat, yr);
            rope_apply(yr, R, base, pos[r]);
        }
    free(xhat);
}

/* --------------------------------------------------------------- forward */

/*
 * One or more sequences of T tokens at positions pos0 .. pos0+T-1.
 * k, v: [B, T, Hkv, D].  q, g: [B, T - q_begin, Hq, D] hold the query rows
 * t = q_begin .. T-1 only (rows before q_begin serve as keys).  Outputs
 * o [B, T - q_begin, Hq, D] and lse [B, T - q_begin, Hq] (natural log of the
 * softmax normaliser of the scaled scores, nullable).
 *
 * Steps ([P1], [P3] "How Gated SWA Behaves"):
 *  1. q' = RoPE(RMSNorm(q, wq)), k' = RoPE(RMSNorm(k, wk));
 *  2. s_j = scale * q'_i . k'_j for max(0, i-W+1) <= j <= i;
 *  3. P = softmax_j(s) (max subtracted); A_i = sum_j P_ij v_j;
 *  4. O_i = A_i * sigma(g_i), element-wise.
 */
void oracle_fwd(int64_t B, int64_t T, int Hq, int Hkv, int D, int W, int R,
                double base, double eps, double scale, int64_t pos0,
                int64_t q_begin, const double *q, const double *k,
                const double *v, const double *g, const double *wq,
                const double *wk, double *o, double *lse) {
    int group = Hq / Hkv;
    int64_t Tq = T - q_begin;
    /* Normalised and rotated keys for every token and kv head. */
    double *kp = (double *)malloc(sizeof(double) * B * T * Hkv * D);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < T; ++t) {
            double *xhat = (double *)malloc(sizeof(double) * D);
            for (int h = 0; h < Hkv; ++h) {
                double *y = kp + IDX4(b, t, h, 0, T, Hkv, D);
                rms_norm(k + IDX4(b, t, h, 0, T, Hkv, D), wk, D, eps, xhat, y);
                rope_apply(y, R, base, (double)(pos0 + t));
            }
            free(xhat);
        }

#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t i = q_begin; i < T; ++i) {
            double *xhat = (double *)malloc(sizeof(double) * D);
            double *qp = (double *)malloc(sizeof(double) * D);
            double *s = (double *)malloc(sizeof(double) * W);
            double *a = (double *)malloc(sizeof(double) * D);
            int64_t j0 = i - W + 1;
            if (j0 < 0) j0 = 0;
            /* keys before the first provided token do not exist */
            for (int h = 0; h < Hq; ++h) {
                int kvh = h / group;
                const double *qi = q + IDX4(b, i - q_begin, h, 0, Tq, Hq, D);
                rms_norm(qi, wq, D, eps, xhat, qp);
                rope_apply(qp, R, base, (double)(pos0 + i));
                double m = -INFINITY;
                for (int64_t j = j0; j <= i; ++j) {
                    s[j - j0] = scale * dot(qp, kp + IDX4(b, j, kvh, 0, T, Hkv, D), D);
                    if (s[j - j0] > m) m = s[j - j0];
                }
                double l = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    s[j - j0] = exp(s[j - j0] - m);
                    l += s[j - j0];
                }
                for (int d = 0; d < D; ++d) a[d] = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    const double *vj = v + IDX4(b, j, kvh, 0, T, Hkv, D);
                    double p = s[j - j0] / l;
                    for (int d = 0; d < D; ++d) a[d] += p * vj[d];
                }
                const double *gi = g + IDX4(b, i - q_begin, h, 0, Tq, Hq, D);
                double *oi = o + IDX4(b, i - q_begin, h, 0, Tq, Hq, D);
                for (int d = 0; d < D; ++d) oi[d] = a[d] * sigmoid(gi[d]);
                if (lse) lse[((int64_t)b * Tq + (i - q_begin)) * Hq + h] = m + log(l);
            }
            free(xhat);
            free(qp);
            free(s);
            free(a);
        }
    free(kp);
}

/* -------------------------------------------------------------- backward */

/*
 * Exact chain rule of the forward above for full sequences (pos0 = 0,
 * q_begin = 0).  Inputs as in oracle_fwd plus dO [B, T, Hq, D].  Outputs
 * dq, dg [B, T, Hq, D]; dk, dv [B, T, Hkv, D]; dwq, dwk [D] (overwritten).
 *
 * For each query row and head (sigma = sigma(g), A = the attention output
 * before the gate):
 *   dg = dO * A * sigma * (1 - sigma);   dA = dO * sigma;
 *   dp_j = dA . v_j;  dv_j += P_j dA;  Dsum = sum_j P_j dp_j;
 *   ds_j = P_j (dp_j - Dsum);  dq' = scale sum_j ds_j k'_j;
 *   dk'_j += scale ds_j q'.
 * Then through RoPE (rotation by -theta) and RMSNorm:
 *   dy = R^T dy';  dw += dy * xhat;  dxhat = dy * w;
 *   dx = (dxhat - xhat * mean(dxhat * xhat)) / r.
 */
static void norm_rope_backward(const double *x, const double *w, int D, int R,
                               double base, double eps, double p,
                               const double *dyp, double *dx, double *dw_acc,
                               double *xhat, double *y, double *dy) {
    double r = rms_norm(x, w, D, eps, xhat, y);
    for (int d = 0; d < D; ++d) dy[d] = dyp[d];
    rope_apply_transpose(dy, R, base, p);
    double mean = 0.0;
    for (int d = 0; d < D; ++d) {
        dw_acc[d] += dy[d] * xhat[d];
        mean += dy[d] * w[d] * xhat[d];
    }
    mean /= D;
    for (int d = 0; d < D; ++d) dx[d] = (dy[d] * w[d] - xhat[d] * mean) / r;
}

void oracle_bwd(int64_t B, int64_t T, int Hq, int Hkv, int D, int W, int R,
                double base, double eps, double scale, const double *q,
                const double *k, const double *v, const double *g,
                const double *wq, const double *wk, const double *dO,
                double *dq, double *dk, double *dv, double *dg, double *dwq,
                double *dwk) {
    int group = Hq / Hkv;
    int64_t chains = B * Hkv;
    double *dwq_part = (double *)calloc((size_t)chains * D, sizeof(double));
    double *dwk_part = (double *)calloc((size_t)chains * D, sizeof(double));

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t c = 0; c < chains; ++c) {
        int64_t b = c / Hkv;
        int kvh = (int)(c % Hkv);
        double *kp = (double *)malloc(sizeof(double) * T * D);   /* k' rows */
        double *dkp = (double *)calloc((size_t)T * D, sizeof(double)); /* dk' */
        double *xhat = (double *)malloc(sizeof(double) * D);
        double *y = (double *)malloc(sizeof(double) * D);
        double *dy = (double *)malloc(sizeof(double) * D);
        double *qp = (double *)malloc(sizeof(double) * D);
        double *a = (double *)malloc(sizeof(double) * D);
        double *dA = (double *)malloc(sizeof(double) * D);
        double *dqp = (double *)malloc(sizeof(double) * D);
        double *P = (double *)malloc(sizeof(double) * W);
        double *dp = (double *)malloc(sizeof(double) * W);

        for (int64_t t = 0; t < T; ++t) {
            rms_norm(k + IDX4(b, t, kvh, 0, T, Hkv, D), wk, D, eps, xhat, kp + t * D);
            rope_apply(kp + t * D, R, base, (double)t);
            for (int d = 0; d < D; ++d) dv[IDX4(b, t, kvh, d, T, Hkv, D)] = 0.0;
        }

        for (int hh = 0; hh < group; ++hh) {
            int h = kvh * group + hh;
            for (int64_t i = 0; i < T; ++i) {
                int64_t j0 = i - W + 1;
                if (j0 < 0) j0 = 0;
                const double *qi = q + IDX4(b, i, h, 0, T, Hq, D);
                rms_norm(qi, wq, D, eps, xhat, qp);
                rope_apply(qp, R, base, (double)i);
                /* recompute the softmax row and A */
                double m = -INFINITY;
                for (int64_t j = j0; j <= i; ++j) {
                    P[j - j0] = scale * dot(qp, kp + j * D, D);
                    if (P[j - j0] > m) m = P[j - j0];
                }
                double l = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    P[j - j0] = exp(P[j - j0] - m);
                    l += P[j - j0];
                }
                for (int64_t j = j0; j <= i; ++j) P[j - j0] /= l;
                for (int d = 0; d < D; ++d) a[d] = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    const double *vj = v + IDX4(b, j, kvh, 0, T, Hkv, D);
                    for (int d = 0; d < D; ++d) a[d] += P[j - j0] * vj[d];
                }
                /* gate */
                const double *gi = g + IDX4(b, i, h, 0, T, Hq, D);
                const double *dOi = dO + IDX4(b, i, h, 0, T, Hq, D);
                double *dgi = dg + IDX4(b, i, h, 0, T, Hq, D);
                for (int d = 0; d < D; ++d) {
                    double sg = sigmoid(gi[d]);
                    dgi[d] = dOi[d] * a[d] * sg * (1.0 - sg);
                    dA[d] = dOi[d] * sg;
                }
                /* softmax and the two products */
                double Dsum = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    const double *vj = v + IDX4(b, j, kvh, 0, T, Hkv, D);
                    dp[j - j0] = dot(dA, vj, D);
                    Dsum += P[j - j0] * dp[j - j0];
                    double *dvj = dv + IDX4(b, j, kvh, 0, T, Hkv, D);
                    for (int d = 0; d < D; ++d) dvj[d] += P[j - j0] * dA[d];
                }
                for (int d = 0; d < D; ++d) dqp[d] = 0.0;
                for (int64_t j = j0; j <= i; ++j) {
                    double ds = P[j - j0] * (dp[j - j0] - Dsum);
                    for (int d = 0; d < D; ++d) {
                        dqp[d] += scale * ds * kp[j * D + d];
                        dkp[j * D + d] += scale * ds * qp[d];
                    }
                }
                norm_rope_backward(qi, wq, D, R, base, eps, (double)i, dqp,
                                   dq + IDX4(b, i, h, 0, T, Hq, D),
                                   dwq_part + c * D, xhat, y, dy);
            }
        }
        for (int64_t t = 0; t < T; ++t)
            norm_rope_backward(k + IDX4(b, t, kvh, 0, T, Hkv, D), wk, D, R, base,
                               eps, (double)t, dkp + t * D,
                               dk + IDX4(b, t, kvh, 0, T, Hkv, D),
                               dwk_part + c * D, xhat, y, dy);
        free(kp); free(dkp); free(xhat); free(y); free(dy); free(qp);
        free(a); free(dA); free(dqp); free(P); free(dp);
    }
    for (int d = 0; d < D; ++d) {
        dwq[d] = 0.0;
        dwk[d] = 0.0;
    }
    for (int64_t c = 0; c < chains; ++c)
        for (int d = 0; d < D; ++d) {
            dwq[d] += dwq_part[c * D + d];
            dwk[d] += dwk_part[c * D + d];
        }
    free(dwq_part);
    free(dwk_part);
}

/* ---------------------------------------------------------------- decode */

/*
 * One decode step for N sequences, each at position pos[n] ([P1] and [P3]:
 * the SWA layers keep only a window of W tokens, so the cache is a ring of
 * W slots per sequence and kv head).
 * q, g: [N, Hq, D]; k_new, v_new: [N, Hkv, D] (fp64);
 * k_cache, v_cache: [N, Hkv, W, D] bf16 bits, updated in place: slot
 * pos mod W receives bf16(RoPE(RMSNorm(k_new))) and bf16 v_new (v_new holds
 * bf16 values, so that copy is exact).  Output o [N, Hq, D].
 */
void oracle_decode(int64_t N, int Hq, int Hkv, int D, int W, int R,
                   double base, double eps, double scale, const int64_t *pos,
                   const double *q, const double *k_new, const double *v_new,
                   const double *g, const double *wq, const double *wk,
                   uint16_t *k_cache, uint16_t *v_cache, double *o) {
    int group = Hq / Hkv;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        double *xhat = (double *)malloc(sizeof(double) * D);
        double *y = (double *)malloc(sizeof(double) * D);
        double *qp = (double *)malloc(sizeof(double) * D);
        double *kv = (double *)malloc(sizeof(double) * D);
        double *s = (double *)malloc(sizeof(double) * W);
        int *valid = (int *)malloc(sizeof(int) * W);
        double *a = (double *)malloc(sizeof(double) * D);
        int64_t p = pos[n];
        int64_t slot = p % W;
        for (int h = 0; h < Hkv; ++h) {
            rms_norm(k_new + (n * Hkv + h) * D, wk, D, eps, xhat, y);
            rope_apply(y, R, base, (double)p);
            uint16_t *kc = k_cache + ((n * Hkv + h) * (int64_t)W + slot) * D;
            uint16_t *vc = v_cache + ((n * Hkv + h) * (int64_t)W + slot) * D;
            for (int d = 0; d < D; ++d) {
                kc[d] = oracle_bf16_bits(y[d]);
                vc[d] = oracle_bf16_bits(v_new[(n * Hkv + h) * D + d]);
            }
        }
        for (int si = 0; si < W; ++si) {
            int64_t ps = p - ((p - si) % W + W) % W;
            valid[si] = ps >= 0;
        }
        for (int h = 0; h < Hq; ++h) {
            int kvh = h / group;
            rms_norm(q + (n * Hq + h) * D, wq, D, eps, xhat, qp);
            rope_apply(qp, R, base, (double)p);
            double m = -INFINITY;
            for (int si = 0; si < W; ++si) {
                if (!valid[si]) continue;
                const uint16_t *kc = k_cache + ((n * Hkv + kvh) * (int64_t)W + si) * D;
                for (int d = 0; d < D; ++d) kv[d] = oracle_bf16_value(kc[d]);
                s[si] = scale * dot(qp, kv, D);
                if (s[si] > m) m = s[si];
            }
            double l = 0.0;
            for (int si = 0; si < W; ++si) {
                if (!valid[si]) continue;
                s[si] = exp(s[si] - m);
                l += s[si];
            }
            for (int d = 0; d < D; ++d) a[d] = 0.0;
            for (int si = 0; si < W; ++si) {
                if (!valid[si]) continue;
                const uint16_t *vc = v_cache + ((n * Hkv + kvh) * (int64_t)W + si) * D;
                for (int d = 0; d < D; ++d) a[d] += (s[si] / l) * oracle_bf16_value(vc[d]);
            }
            for (int d = 0; d < D; ++d)
                o[(n * Hq + h) * D + d] = a[d] * sigmoid(g[(n * Hq + h) * D + d]);
        }
        free(xhat); free(y); free(qp); free(kv); free(s); free(valid); free(a);
    }
}

/* ------------------------------------------------------------ footprint */

/* KV-cache bytes per token for L layers that keep every token, H KV heads of
 * dim d, `bytes` per element: one K and one V vector per layer and head
 * ([P3] "Why the KV Cache Shrinks by 6.4x"). */
int64_t oracle_kv_bytes_per_token(int64_t layers, int64_t kv_heads,
                                  int64_t head_dim, int64_t bytes) {
    return 2 * layers * kv_heads * head_dim * bytes;
}

/* Threads an OpenMP region in this library would use (for reporting). */
#ifdef _OPENMP
#include <omp.h>
int oracle_threads(void) { return omp_get_max_threads(); }
#else
int oracle_threads(void) { return 1; }
#endif
