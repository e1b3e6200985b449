/*
 * Float64 CPU oracle for the Vision-RWKV spatial-mix core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * with the CUDA library and includes nothing from it.
 *
 * Sources (page titles as given in the reference pages):
 *   [VRWKV]  "OpenGVLab&港中文&复旦&南大&清华提出Vision-RWKV Backbone"
 *            (cloud.tencent.com article 2395249):
 *              - Linear Complexity Bidirectional Attention, eq. 5 (summation
 *                form of Bi-WKV) and eq. 6-7 (RNN form, hidden states a,b,c,d);
 *              - Quad-Directional Token Shift, eq. 9 (Q-Shift);
 *              - Overall Architecture, eq. 2 (sigma(R) (.) wkv gate) and
 *                eq. 3-4 (channel mix);
 *              - the Bi-WKV backward pass, which the pages place in an
 *                appendix they do not reproduce: here it is the plain
 *                derivative of eq. 5, written out below.
 *   [BLOG]   "LinXin's Blog" (linxin.blog), Vision-RWKV entry: the q_shift
 *            listing (patch_resolution, shift_pixel, gamma, zero-initialised
 *            output, four slice assignments, copy of the remaining channels).
 *
 * Layout of every token tensor: row-major (B, T, C), channel fastest, token
 * index t = h*W + w (the listing's transpose/reshape of (B,N,C) to (B,C,H,W)).
 *
 * Readings of the pages taken here (each also listed in the design notes):
 *   - eq. 9 prints "X + (1-mu)X^dagger" but calls it a linear interpolation of
 *     X and X^dagger; the interpolation mu*X + (1-mu)*X^dagger is computed.
 *   - channel-group order follows the listing (w-s, w+s, h-s, h+s); eq. 9's
 *     order (h-1, h+1, w-1, w+1) is available through eq9_order=1.
 *   - the channel groups end where the listing's slices end: at
 *     b_j = int(C*gamma*j), j = 1..4, with C*gamma formed first, then times
 *     j, in double precision (Python's left-to-right order), and truncated
 *     as Python int() does; channels >= b_4 are copied.  Eq. 9's C/4, C/2,
 *     3C/4, C are the same bounds at gamma = 1/4.
 *   - a shift_pixel at or beyond the grid extent empties that group (zeros).
 *   - the garbled "ki" in eq. 5 is k_i; T is the total token count.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Q-Shift: the gather X^dagger (eq. 9 and the q_shift listing)        */
/* ------------------------------------------------------------------ */

/* End of channel group j-1 (j = 1..4): the listing's slice bound
 * int(C*gamma*j).  Python evaluates C*gamma first and then multiplies by j,
 * both in double precision, and int() truncates toward zero. */
static int qshift_bound(int C, double gamma, int j) {
    double cg = (double)C * gamma;
    return (int)(cg * (double)j);
}

/* Channel group of channel c: 0..3 for the four slices
 * [b_{j}, b_{j+1}) (b_0 = 0), 4 for the copied channels c >= b_4
 * (output[:, int(C*gamma*4):] = input[:, int(C*gamma*4):]). */
static int qshift_group(int c, int C, double gamma) {
    for (int j = 1; j <= 4; ++j)
        if (c < qshift_bound(C, gamma, j)) return j - 1;
    return 4;
}

/* Source pixel of output pixel (h,w) for channel c, following the listing's
 * slice assignments.  Returns 0 when the output stays at its zero initial
 * value (border, or an emptied group), 1 with (*sh,*sw) set otherwise. */
static int qshift_source(int c, int h, int w, int H, int W, int C, int s,
                         double gamma, int eq9_order, int* sh, int* sw) {
    int grp = qshift_group(c, C, gamma);
    if (eq9_order && grp < 4) {
        /* eq. 9 order: h-1, h+1, w-1, w+1  ->  listing groups 2,3,0,1 */
        static const int perm[4] = {2, 3, 0, 1};
        grp = perm[grp];
    }
    int srch = h, srcw = w;
    switch (grp) {
    case 0: /* output[..., s:W] = input[..., 0:W-s]: value comes from w-s */
        srcw = w - s;
        break;
    case 1: /* output[..., 0:W-s] = input[..., s:W]: value comes from w+s */
        srcw = w + s;
        break;
    case 2: /* output[.., s:H, :] = input[.., 0:H-s, :]: from h-s */
        srch = h - s;
        break;
    case 3: /* output[.., 0:H-s, :] = input[.., s:H, :]: from h+s */
        srch = h + s;
        break;
    default:
        break;
    }
    if (srch < 0 || srch >= H || srcw < 0 || srcw >= W) return 0;
    *sh = srch;
    *sw = srcw;
    return 1;
}

/* out = X^dagger (mu == NULL) or mu*X + (1-mu)*X^dagger, in float64. */
void oracle_qshift_f64(const double* x, double* out, const double* mu, int B,
                       int H, int W, int C, int s, double gamma,
                       int eq9_order) {
    const long T = (long)H * W;
#pragma omp parallel for schedule(static)
    for (long bt = 0; bt < (long)B * T; ++bt) {
        long b = bt / T, t = bt % T;
        int h = (int)(t / W), w = (int)(t % W);
        for (int c = 0; c < C; ++c) {
            int sh, sw;
            double xd = 0.0;
            if (qshift_source(c, h, w, H, W, C, s, gamma, eq9_order, &sh, &sw))
                xd = x[(b * T + (long)sh * W + sw) * C + c];
            double xv = x[(b * T + t) * C + c];
            out[(b * T + t) * C + c] =
                mu ? mu[c] * xv + (1.0 - mu[c]) * xd : xd;
        }
    }
}

/* Round a float to the nearest bfloat16 (ties to even), returned as float.
 * bfloat16 keeps the top 16 bits of the IEEE binary32 pattern. */
static float round_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) { /* inf or nan */
        if (u & 0x007fffffu) u |= 0x00400000u; /* keep nan quiet */
        u &= 0xffff0000u;
    } else {
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7fffu + lsb;
        u &= 0xffff0000u;
    }
    float r;
    memcpy(&r, &u, 4);
    return r;
}

void oracle_round_bf16(const float* in, float* out, long n) {
    for (long i = 0; i < n; ++i) out[i] = round_to_bf16(in[i]);
}

/* The interpolation evaluated in binary32 with each operation rounded on its
 * own (t1 = mu*x, t2 = (1-mu)*x^dagger, out = t1 + t2; no fused multiply-add,
 * enforced by -ffp-contract=off), then optionally rounded to bfloat16.  This
 * is the fixed operation order the bit-exact Q-Shift comparison uses. */
void oracle_qshift_f32(const float* x, float* out, const float* mu, int B,
                       int H, int W, int C, int s, double gamma,
                       int round_bf16) {
    const long T = (long)H * W;
#pragma omp parallel for schedule(static)
    for (long bt = 0; bt < (long)B * T; ++bt) {
        long b = bt / T, t = bt % T;
        int h = (int)(t / W), w = (int)(t % W);
        for (int c = 0; c < C; ++c) {
            int sh, sw;
            float xd = 0.0f;
            if (qshift_source(c, h, w, H, W, C, s, gamma, 0, &sh, &sw))
                xd = x[(b * T + (long)sh * W + sw) * C + c];
            float r;
            if (mu) {
                volatile float t1 = mu[c] * x[(b * T + t) * C + c];
                volatile float om = 1.0f - mu[c];
                volatile float t2 = om * xd;
                r = t1 + t2;
            } else {
                r = xd;
            }
            out[(b * T + t) * C + c] = round_bf16 ? round_to_bf16(r) : r;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Bi-WKV, summation form (eq. 5)                                      */
/* ------------------------------------------------------------------ */

/* wkv_t for one channel column, directly from eq. 5:
 *   num = sum_{i != t} exp(-(|t-i|-1)/T * w + k_i) v_i + exp(u + k_t) v_t
 *   den = the same sums with v replaced by 1.                          */
static double biwkv_direct_one(const double* kc, const double* vc, long T,
                               double w, double u, long t) {
    double num = 0.0, den = 0.0;
    for (long i = 0; i < T; ++i) {
        double e;
        if (i == t) {
            e = exp(u + kc[i]);
        } else {
            long d = i > t ? i - t : t - i;
            e = exp(-((double)(d - 1) / (double)T) * w + kc[i]);
        }
        num += e * vc[i];
        den += e;
    }
    return num / den;
}

static void gather_column(const double* src, double* col, long b, long T,
                          long C, long c) {
    for (long t = 0; t < T; ++t) col[t] = src[(b * T + t) * C + c];
}

void oracle_biwkv_direct(const double* k, const double* v, const double* w,
                         const double* u, double* out, int B, int T, int C) {
#pragma omp parallel
    {
        double* kc = (double*)malloc(sizeof(double) * (size_t)T);
        double* vc = (double*)malloc(sizeof(double) * (size_t)T);
#pragma omp for schedule(dynamic, 1)
        for (long bc = 0; bc < (long)B * C; ++bc) {
            long b = bc / C, c = bc % C;
            gather_column(k, kc, b, T, C, c);
            gather_column(v, vc, b, T, C, c);
            for (long t = 0; t < T; ++t)
                out[(b * T + t) * C + c] =
                    biwkv_direct_one(kc, vc, T, w[c], u[c], t);
        }
        free(kc);
        free(vc);
    }
}

/* eq. 5 at selected flat indices idx[j] = (b*T + t)*C + c only. */
void oracle_biwkv_direct_points(const double* k, const double* v,
                                const double* w, const double* u, int B, int T,
                                int C, const int64_t* idx, long n,
                                double* out) {
    (void)B;
#pragma omp parallel
    {
        double* kc = (double*)malloc(sizeof(double) * (size_t)T);
        double* vc = (double*)malloc(sizeof(double) * (size_t)T);
#pragma omp for schedule(dynamic, 16)
        for (long j = 0; j < n; ++j) {
            long f = (long)idx[j];
            long c = f % C, bt = f / C, t = bt % T, b = bt / T;
            gather_column(k, kc, b, T, C, c);
            gather_column(v, vc, b, T, C, c);
            out[j] = biwkv_direct_one(kc, vc, T, w[c], u[c], t);
        }
        free(kc);
        free(vc);
    }
}

/* ------------------------------------------------------------------ */
/* Bi-WKV, RNN form (eq. 6-7)                                          */
/* ------------------------------------------------------------------ */

/* Hidden states for output t (eq. 6):
 *   a_{t-1} = sum_{i<t} e^{-(|t-i|-1)/T w + k_i} v_i,   c_{t-1}: v -> 1
 *   b_{t-1} = sum_{i>t} e^{-(|t-i|-1)/T w + k_i} v_i,   d_{t-1}: v -> 1
 * and eq. 7: wkv_t = (a+b+e^{k_t+u} v_t) / (c+d+e^{k_t+u}).
 * Each step adds one term and multiplies by e^{-w/T}.  The forward pair (a,c)
 * is run for increasing t; the backward pair (b,d) is run as its own pass for
 * decreasing t (b_{t-1} = e^{-w/T} b_t + e^{k_{t+1}} v_{t+1}), which is the
 * same sum built from the other end. */
void oracle_biwkv_rnn(const double* k, const double* v, const double* w,
                      const double* u, double* out, int B, int T, int C) {
#pragma omp parallel
    {
        double* bb = (double*)malloc(sizeof(double) * (size_t)T);
        double* dd = (double*)malloc(sizeof(double) * (size_t)T);
#pragma omp for schedule(static)
        for (long bc = 0; bc < (long)B * C; ++bc) {
            long b = bc / C, c = bc % C;
            const double decay = exp(-w[c] / (double)T);
            /* backward pass: bb[t] = b_{t-1}, dd[t] = d_{t-1} */
            double sb = 0.0, sd = 0.0;
            for (long t = T - 1; t >= 0; --t) {
                bb[t] = sb;
                dd[t] = sd;
                double e = exp(k[(b * T + t) * C + c]);
                sb = decay * sb + e * v[(b * T + t) * C + c];
                sd = decay * sd + e;
            }
            /* forward pass and eq. 7 */
            double sa = 0.0, sc = 0.0;
            for (long t = 0; t < T; ++t) {
                double kt = k[(b * T + t) * C + c];
                double vt = v[(b * T + t) * C + c];
                double eu = exp(u[c] + kt);
                out[(b * T + t) * C + c] =
                    (sa + bb[t] + eu * vt) / (sc + dd[t] + eu);
                double e = exp(kt);
                sa = decay * sa + e * vt;
                sc = decay * sc + e;
            }
        }
        free(bb);
        free(dd);
    }
}

/* The RNN form exactly as the pages phrase it: b and d start as full sums
 * over i > 0 and each later state is obtained by removing the term that
 * becomes the current token and dividing by e^{-w/T}.  Subtraction makes it
 * lose precision for long sequences; it is used on short sequences only. */
void oracle_biwkv_rnn_literal(const double* k, const double* v,
                              const double* w, const double* u, double* out,
                              int B, int T, int C) {
    for (long b = 0; b < B; ++b)
        for (long c = 0; c < C; ++c) {
            const double decay = exp(-w[c] / (double)T);
            double sa = 0.0, sc = 0.0, sb = 0.0, sd = 0.0;
            for (long i = 1; i < T; ++i) { /* b_{-1}, d_{-1} for t = 0 */
                double e = exp(-((double)(i - 1) / (double)T) * w[c] +
                               k[(b * T + i) * C + c]);
                sb += e * v[(b * T + i) * C + c];
                sd += e;
            }
            for (long t = 0; t < T; ++t) {
                double kt = k[(b * T + t) * C + c];
                double vt = v[(b * T + t) * C + c];
                double eu = exp(u[c] + kt);
                out[(b * T + t) * C + c] = (sa + sb + eu * vt) / (sc + sd + eu);
                /* a,c: add the current term, multiply by e^{-w/T} */
                double e = exp(kt);
                sa = decay * sa + e * vt;
                sc = decay * sc + e;
                /* b,d: remove the term of token t+1, divide by e^{-w/T} */
                if (t + 1 < T) {
                    double e1 = exp(k[(b * T + t + 1) * C + c]);
                    sb = (sb - e1 * v[(b * T + t + 1) * C + c]) / decay;
                    sd = (sd - e1) / decay;
                }
            }
        }
}

/* ------------------------------------------------------------------ */
/* Gate (eq. 2): sigma(R) (.) wkv, sigma(z) = 1 / (1 + e^{-z})         */
/* ------------------------------------------------------------------ */
void oracle_gate(const double* r, const double* wkv, double* out, long n) {
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) out[i] = wkv[i] * (1.0 / (1.0 + exp(-r[i])));
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* The spatial-mix core at selected output positions                   */
/* ------------------------------------------------------------------ */

/* Q-Shifted value of tensor x at (b, t, c): mu*x + (1-mu)*x^dagger, or
 * x^dagger when mu is NULL, or x itself when qshift_on is 0. */
static double qs_value(const double* x, const double* mu, long b, long t, int c,
                       int H, int W, int C, int s, double gamma,
                       int qshift_on) {
    const long T = (long)H * W;
    double xv = x[(b * T + t) * C + c];
    if (!qshift_on) return xv;
    int sh, sw;
    double xd = 0.0;
    if (qshift_source(c, (int)(t / W), (int)(t % W), H, W, C, s, gamma, 0,
                      &sh, &sw))
        xd = x[(b * T + (long)sh * W + sw) * C + c];
    return mu ? mu[c] * xv + (1.0 - mu[c]) * xd : xd;
}

/* out[j] = sigma(QS_R(r))[p] * Bi-WKV(QS_K(k), QS_V(v))[p] at the flat
 * position p = idx[j] = (b*T + t)*C + c, evaluating eq. 5 directly over the
 * (b, c) column (gate_on = 0 drops the sigma factor; r is then unused). */
void oracle_spatial_core_points(const double* r, const double* k,
                                const double* v, const double* w,
                                const double* u, const double* mu_r,
                                const double* mu_k, const double* mu_v, int B,
                                int H, int W, int C, int s, double gamma,
                                int qshift_on, int gate_on,
                                const int64_t* idx, long n, double* out) {
    (void)B;
    const long T = (long)H * W;
#pragma omp parallel
    {
        double* kc = (double*)malloc(sizeof(double) * (size_t)T);
        double* vc = (double*)malloc(sizeof(double) * (size_t)T);
#pragma omp for schedule(dynamic, 4)
        for (long j = 0; j < n; ++j) {
            long f = (long)idx[j];
            int c = (int)(f % C);
            long bt = f / C, t = bt % T, b = bt / T;
            for (long i = 0; i < T; ++i) {
                kc[i] = qs_value(k, mu_k, b, i, c, H, W, C, s, gamma, qshift_on);
                vc[i] = qs_value(v, mu_v, b, i, c, H, W, C, s, gamma, qshift_on);
            }
            double y = biwkv_direct_one(kc, vc, T, w[c], u[c], t);
            if (gate_on) {
                double rs = qs_value(r, mu_r, b, t, c, H, W, C, s, gamma,
                                     qshift_on);
                y = y * (1.0 / (1.0 + exp(-rs)));
            }
            out[j] = y;
        }
        free(kc);
        free(vc);
    }
}

/* ------------------------------------------------------------------ */
/* Channel mix without projections (eq. 3-4 with identity W_R, W_K,   */
/* W_V and no W_O):  out = sigma(QS_R(x)) (.) SquaredReLU(QS_K(x)),   */
/* SquaredReLU(z) = max(z, 0)^2.                                      */
/* ------------------------------------------------------------------ */
void oracle_channel_mix(const double* x, const double* mu_r,
                        const double* mu_k, double* out, int B, int H, int W,
                        int C, int s, double gamma) {
    const long T = (long)H * W;
#pragma omp parallel for schedule(static)
    for (long bt = 0; bt < (long)B * T; ++bt) {
        long b = bt / T, t = bt % T;
        for (int c = 0; c < C; ++c) {
            double rs = qs_value(x, mu_r, b, t, c, H, W, C, s, gamma, 1);
            double ks = qs_value(x, mu_k, b, t, c, H, W, C, s, gamma, 1);
            double kp = ks > 0.0 ? ks : 0.0;
            out[bt * C + c] = (1.0 / (1.0 + exp(-rs))) * (kp * kp);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Bi-WKV backward: derivatives of eq. 5                               */
/* ------------------------------------------------------------------ */
/* For one (b, c) column with weights
 *   W_ti = exp(-(|t-i|-1)/T * w)  (i != t),   W_tt = exp(u),
 *   N_t = sum_i W_ti e^{k_i} v_i,  D_t = sum_i W_ti e^{k_i},  y_t = N_t / D_t,
 * and the upstream gradient g_t = dL/dy_t, the chain rule gives
 *   dL/dv_i = e^{k_i} sum_t W_ti g_t / D_t
 *   dL/dk_i = e^{k_i} sum_t W_ti g_t (v_i - y_t) / D_t
 *   dL/du   = sum_t e^{u + k_t} g_t (v_t - y_t) / D_t
 *   dL/dw   = -(1/T) sum_t sum_{i != t} (|t-i|-1) W_ti e^{k_i} g_t (v_i - y_t) / D_t
 * Every term is a ratio e^{k_i} / D_t, so e^{k} is evaluated as e^{k - max k}
 * (the factor cancels) to keep the exponentials in range.  O(T^2) per column. */
static void biwkv_bwd_column(const double* kc, const double* vc,
                             const double* gc, long T, double w, double u,
                             double* gk, double* gv, double* gw, double* gu,
                             double* y, double* q, double* scale) {
    double M = kc[0];
    for (long i = 1; i < T; ++i)
        if (kc[i] > M) M = kc[i];
    /* forward values: y_t and q_t = g_t / D_t (D_t scaled by e^{-M}) */
    for (long t = 0; t < T; ++t) {
        double num = 0.0, den = 0.0;
        for (long i = 0; i < T; ++i) {
            double e;
            if (i == t) {
                e = exp(u + kc[i] - M);
            } else {
                long d = i > t ? i - t : t - i;
                e = exp(-((double)(d - 1) / (double)T) * w + kc[i] - M);
            }
            num += e * vc[i];
            den += e;
        }
        y[t] = num / den;
        q[t] = gc[t] / den;
    }
    double sgu = 0.0, sgw = 0.0, agu = 0.0, agw = 0.0;
    for (long i = 0; i < T; ++i) {
        double sv = 0.0, sk = 0.0, av = 0.0, ak = 0.0;
        for (long t = 0; t < T; ++t) {
            double e;  /* W_ti e^{k_i - M} */
            const double m = fabs(q[t]) * (fabs(vc[i]) + fabs(y[t]));
            if (t == i) {
                e = exp(u + kc[i] - M);
                sgu += e * q[t] * (vc[i] - y[t]);
                agu += e * m;
            } else {
                long d = i > t ? i - t : t - i;
                e = exp(-((double)(d - 1) / (double)T) * w + kc[i] - M);
                sgw += (double)(d - 1) * e * q[t] * (vc[i] - y[t]);
                agw += (double)(d - 1) * e * m;
            }
            sv += e * q[t];
            sk += e * q[t] * (vc[i] - y[t]);
            av += e * fabs(q[t]);
            ak += e * m;
        }
        gv[i] = sv;
        gk[i] = sk;
        if (scale) {  /* sums of the absolute values of the terms */
            scale[i] = ak;
            scale[T + i] = av;
        }
    }
    *gu = sgu;
    *gw = -sgw / (double)T;
    if (scale) {
        scale[2 * T] = agw / (double)T;
        scale[2 * T + 1] = agu;
    }
}

/* Gradients of every column.  gk, gv: (B, T, C); gw, gu: (B, C), the
 * contribution of each batch element (the batch gradient is their sum). */
void oracle_biwkv_bwd_direct(const double* k, const double* v, const double* w,
                             const double* u, const double* gy, int B, int T,
                             int C, double* gk, double* gv, double* gw,
                             double* gu) {
#pragma omp parallel
    {
        double* buf = (double*)malloc(sizeof(double) * (size_t)T * 7);
        double *kc = buf, *vc = buf + T, *gc = buf + 2 * T, *ok = buf + 3 * T,
               *ov = buf + 4 * T, *y = buf + 5 * T, *q = buf + 6 * T;
#pragma omp for schedule(dynamic, 1)
        for (long bc = 0; bc < (long)B * C; ++bc) {
            long b = bc / C, c = bc % C;
            gather_column(k, kc, b, T, C, c);
            gather_column(v, vc, b, T, C, c);
            gather_column(gy, gc, b, T, C, c);
            biwkv_bwd_column(kc, vc, gc, T, w[c], u[c], ok, ov, &gw[bc], &gu[bc],
                             y, q, NULL);
            for (long t = 0; t < T; ++t) {
                gk[(b * T + t) * C + c] = ok[t];
                gv[(b * T + t) * C + c] = ov[t];
            }
        }
        free(buf);
    }
}

/* The same for selected columns cols[j] = b*C + c only: gk, gv are (n, T),
 * gw, gu are (n).  If scale is not NULL it receives, per column, the sums of
 * the absolute values of the terms of each gradient (an error scale for
 * comparisons), laid out as (n, 2T + 2): gk's T, gv's T, then gw, gu. */
void oracle_biwkv_bwd_columns(const double* k, const double* v,
                              const double* w, const double* u,
                              const double* gy, int B, int T, int C,
                              const int64_t* cols, long n, double* gk,
                              double* gv, double* gw, double* gu,
                              double* scale) {
    (void)B;
#pragma omp parallel
    {
        double* buf = (double*)malloc(sizeof(double) * (size_t)T * 5);
        double *kc = buf, *vc = buf + T, *gc = buf + 2 * T, *y = buf + 3 * T,
               *q = buf + 4 * T;
#pragma omp for schedule(dynamic, 1)
        for (long j = 0; j < n; ++j) {
            long b = (long)cols[j] / C, c = (long)cols[j] % C;
            gather_column(k, kc, b, T, C, c);
            gather_column(v, vc, b, T, C, c);
            gather_column(gy, gc, b, T, C, c);
            biwkv_bwd_column(kc, vc, gc, T, w[c], u[c], gk + j * (long)T,
                             gv + j * (long)T, &gw[j], &gu[j], y, q,
                             scale ? scale + j * (2 * (long)T + 2) : NULL);
        }
        free(buf);
    }
}

/* ------------------------------------------------------------------ */
/* Bidirectional shift for sparse (MAE) inputs                          */
/* ------------------------------------------------------------------ */
/* The pages pre-train with MAE after changing Q-Shift into a bidirectional
 * shift, and say no more.  Reading taken: of Q-Shift's four channel groups
 * only the two that shift along the token row remain -- [0, b_1) from token
 * w-s, [b_1, b_2) from token w+s (b_j the listing's int(C*gamma*j)), zero
 * past the row's ends -- and every other channel, the two vertical groups
 * included, passes through unchanged.  A sparse input is one row of its
 * visible tokens (H = 1, W = their count). */
static int bishift_source(int c, int h, int w, int W, int C, int s,
                          double gamma, int* sh, int* sw) {
    int grp = qshift_group(c, C, gamma);
    int srcw = w;
    if (grp == 0) srcw = w - s;
    else if (grp == 1) srcw = w + s;
    if (srcw < 0 || srcw >= W) return 0;
    *sh = h;
    *sw = srcw;
    return 1;
}

void oracle_bishift_f64(const double* x, double* out, const double* mu, int B,
                        int H, int W, int C, int s, double gamma) {
    const long T = (long)H * W;
#pragma omp parallel for schedule(static)
    for (long bt = 0; bt < (long)B * T; ++bt) {
        long b = bt / T, t = bt % T;
        int h = (int)(t / W), w = (int)(t % W);
        for (int c = 0; c < C; ++c) {
            int sh, sw;
            double xd = 0.0;
            if (bishift_source(c, h, w, W, C, s, gamma, &sh, &sw))
                xd = x[(b * T + (long)sh * W + sw) * C + c];
            double xv = x[(b * T + t) * C + c];
            out[(b * T + t) * C + c] = mu ? mu[c] * xv + (1.0 - mu[c]) * xd : xd;
        }
    }
}

/* The same with the binary32 operation order of oracle_qshift_f32. */
void oracle_bishift_f32(const float* x, float* out, const float* mu, int B,
                        int H, int W, int C, int s, double gamma,
                        int round_bf16) {
    const long T = (long)H * W;
#pragma omp parallel for schedule(static)
    for (long bt = 0; bt < (long)B * T; ++bt) {
        long b = bt / T, t = bt % T;
        int h = (int)(t / W), w = (int)(t % W);
        for (int c = 0; c < C; ++c) {
            int sh, sw;
            float xd = 0.0f;
            if (bishift_source(c, h, w, W, C, s, gamma, &sh, &sw))
                xd = x[(b * T + (long)sh * W + sw) * C + c];
            float r;
            if (mu) {
                volatile float t1 = mu[c] * x[(b * T + t) * C + c];
                volatile float om = 1.0f - mu[c];
                volatile float t2 = om * xd;
                r = t1 + t2;
            } else {
                r = xd;
            }
            out[(b * T + t) * C + c] = round_bf16 ? round_to_bf16(r) : r;
        }
    }
}
