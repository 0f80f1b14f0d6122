/*
 * oracle.c -- float64 CPU oracle for per-row L2 normalisation.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h): loaded by the tests, the smoke
 * check and the benchmark's CPU-baseline leg, never by the product path.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fPIC -shared -pthread
 * (oracle/build.py).  No FMA contraction, no fast-math: each line below is
 * one IEEE double operation in the order written.
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits.  A finite
 * non-zero bf16 is m * 2^q with q = E - 7 in the binade [2^E, 2^(E+1)) for
 * E >= -126, and q = -133 below 2^-126 (subnormals).  Rounding a double to
 * bf16 is: count the quanta of its binade, round that count to the nearest
 * integer with ties to even (rint under the default rounding mode), and
 * rebuild.  Results at or above 2^128 overflow to infinity.                 */

uint16_t or_bf16_rne(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v))
        return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(v);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;

    int e;
    (void)frexp(a, &e);             /* a in [2^(e-1), 2^e) */
    int E = e - 1;
    int q = (E >= -126) ? E - 7 : -133;
    double n = rint(ldexp(a, -q)); /* quanta, ties to even; exact scaling */
    if (n == 0.0)
        return sign;
    double r = ldexp(n, q);        /* the rounded magnitude, exact */
    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    if (r < ldexp(1.0, -126))
        return (uint16_t)(sign | (uint16_t)n); /* subnormal: n < 128 quanta */

    int e2;
    (void)frexp(r, &e2);
    int E2 = e2 - 1;
    unsigned frac = (unsigned)(ldexp(r, 7 - E2) - 128.0);
    return (uint16_t)(sign | (unsigned)((E2 + 127) << 7) | frac);
}

double or_bf16_value(uint16_t bits)
{
    int s = bits >> 15;
    int e = (bits >> 7) & 0xFF;
    int m = bits & 0x7F;
    double v;
    if (e == 0xFF)
        v = m ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)m, -133);
    else
        v = ldexp((double)(128 + m), e - 127 - 7);
    return s ? -v : v;
}

void or_bf16_rne_array(const double *src, int64_t n, uint16_t *dst)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = or_bf16_rne(src[i]);
}

static double round_bf16(double v) { return or_bf16_value(or_bf16_rne(v)); }

/* ------------------------------------------------------------------------ */
/* Row helpers.                                                              */

static double sum_sq(const double *x, int64_t C)
{
    double S = 0.0;
    for (int64_t j = 0; j < C; ++j)
        S += x[j] * x[j];
    return S;
}

/* The row norm.  [DS] eq. W_eff divides by the row length; the sum carries
 * eps inside the square root as [TF] states for its rows. */
static double row_norm(double S, double eps, unsigned flags)
{
    if (flags & OR_EPS_ZERO)
        return sqrt(S);
    if (flags & OR_EPS_OUTSIDE)
        return sqrt(S) + eps;
    return sqrt(S + eps);
}

/* [DS] "What DragonScale changes", eq. W_eff = diag(g) r W / ||W||_row. */
void or_wn_forward_row(const double *w, int64_t C, double g, double rho,
                       double eps, unsigned flags, double *out)
{
    double n = row_norm(sum_sq(w, C), eps, flags);
    for (int64_t j = 0; j < C; ++j)
        out[j] = g * rho * w[j] / n;
}

/* Chain rule on the forward above, L = sum_j gy_j out_j:
 *   dL/dg   = rho sum_j gy_j w_j / n                       = rho D / n
 *   dL/dw_k = g rho (gy_k / n - w_k D / n^3)               (dn/dw_k = w_k / n)
 *           = (g rho / n) (gy_k - w_k D / (S + eps)).
 * [DS] eq. dL/dW prints the eps = 0 form (g r/||W||)(I - w^ w^T) dL/dW_eff. */
void or_wn_backward_row(const double *w, const double *gy, int64_t C, double g,
                        double rho, double eps, unsigned flags, double *grad_w,
                        double *grad_g)
{
    double S = sum_sq(w, C);
    double D = 0.0;
    for (int64_t j = 0; j < C; ++j)
        D += w[j] * gy[j];
    double e = (flags & OR_EPS_ZERO) ? 0.0 : eps;
    double n = sqrt(S + e);
    double n2 = (flags & OR_BWD_PRINTED) ? S : S + e;
    if (grad_g)
        *grad_g = rho * D / n;
    for (int64_t j = 0; j < C; ++j)
        grad_w[j] = (g * rho / n) * (gy[j] - w[j] * D / n2);
}

/* [DS] "Optimizer", method "rescale", before the step: the part of the
 * gradient that would change the row's length -- its component along the
 * row -- is removed:  D = sum_j w_j G_j,  out_j = G_j - w_j * D / (S + eps).
 * At eps = 0 this is the orthogonal projection onto the row's complement. */
void or_grad_project_row(const double *w, const double *G, int64_t C,
                         double eps, unsigned flags, double *out)
{
    double S = sum_sq(w, C);
    double D = 0.0;
    for (int64_t j = 0; j < C; ++j)
        D += w[j] * G[j];
    double n2 = (flags & OR_EPS_ZERO) ? S : S + eps;
    for (int64_t j = 0; j < C; ++j)
        out[j] = G[j] - w[j] * D / n2;
}

/* [DS] "Optimizer", after the step: the same component removed from the
 * momentum, and the row rescaled back to its radius, both from the row as
 * the step left it (the rescale does not change its direction):
 *   m_out_j = m_j - w_j * (sum_k w_k m_k) / (S + eps),
 *   w_out_j = rho * w_j / sqrt(S + eps). */
void or_renorm_momentum_row(const double *w, const double *m, int64_t C,
                            double rho, double eps, unsigned flags,
                            double *w_out, double *m_out)
{
    or_grad_project_row(w, m, C, eps, flags, m_out);
    or_row_renorm_row(w, C, rho, eps, flags, w_out);
}

/* [DS] "Optimizer": after the step each row is rescaled back to its radius. */
void or_row_renorm_row(const double *w, int64_t C, double rho, double eps,
                       unsigned flags, double *out)
{
    double n = row_norm(sum_sq(w, C), eps, flags);
    for (int64_t j = 0; j < C; ++j)
        out[j] = rho * w[j] / n;
}

/* [TF] tf_l2_rows.  The sum of two bf16 values is rounded once, from its f64
 * value: when f64 cannot hold the sum exactly the smaller term is below
 * 2^-45 of the larger, far from any bf16 halfway point, so the f64 detour
 * cannot move the result across one. */
void or_l2_row(const double *x, const double *r, int64_t C, double eps,
               unsigned flags, double *s, uint16_t *y, double *y_exact)
{
    for (int64_t j = 0; j < C; ++j) {
        if (!r)
            s[j] = x[j];
        else if (flags & OR_DROP_SUM_ROUND)
            s[j] = x[j] + r[j];
        else
            s[j] = round_bf16(x[j] + r[j]);
    }
    double n = row_norm(sum_sq(s, C), eps, flags);
    for (int64_t j = 0; j < C; ++j) {
        double v = s[j] / n;
        y[j] = or_bf16_rne(v);
        if (y_exact)
            y_exact[j] = v;
    }
}

/* [TF] tf_slerp_rows: a normalised lerp between two unit rows. */
void or_slerp_row(const double *res, const double *out, const double *alpha,
                  int64_t C, double eps, unsigned flags, double *tmp,
                  uint16_t *h, double *h_exact)
{
    double *a = tmp, *b = tmp + C, *t = tmp + 2 * C;
    double na = row_norm(sum_sq(res, C), eps, flags);
    double nb = row_norm(sum_sq(out, C), eps, flags);
    for (int64_t j = 0; j < C; ++j) {
        a[j] = res[j] / na;
        if (!(flags & OR_DROP_SLERP_A))
            a[j] = round_bf16(a[j]);
        b[j] = out[j] / nb;
        if (!(flags & OR_DROP_SLERP_B))
            b[j] = round_bf16(b[j]);
    }
    for (int64_t j = 0; j < C; ++j)
        t[j] = a[j] + fabs(alpha[j]) * (b[j] - a[j]);
    double nt = row_norm(sum_sq(t, C), eps, flags);
    for (int64_t j = 0; j < C; ++j) {
        double v = t[j] / nt;
        h[j] = or_bf16_rne(v);
        if (h_exact)
            h_exact[j] = v;
    }
}

/* ------------------------------------------------------------------------ */
/* Backward of the activation rows (derived: the pages give the forward
 * only).  Gradients pass straight through the bf16 rounding points: the
 * backward uses the rounded values wherever the forward does (s, a, b) and
 * takes the rounding itself as the identity.                                */

/* y = s / n, n = sqrt(S + eps), s = x or bf16(x + r):
 *   dx_j = (dy_j - s_j D / (S + eps)) / n,  D = sum_k s_k dy_k
 * (with a residual, dr = dx). */
void or_l2_backward_row(const double *x, const double *r, const double *dy,
                        int64_t C, double eps, unsigned flags, double *s,
                        double *dx)
{
    for (int64_t j = 0; j < C; ++j) {
        if (!r)
            s[j] = x[j];
        else if (flags & OR_DROP_SUM_ROUND)
            s[j] = x[j] + r[j];
        else
            s[j] = round_bf16(x[j] + r[j]);
    }
    double S = sum_sq(s, C);
    double D = 0.0;
    for (int64_t j = 0; j < C; ++j)
        D += s[j] * dy[j];
    double e = (flags & OR_EPS_ZERO) ? 0.0 : eps;
    double n = sqrt(S + e);
    for (int64_t j = 0; j < C; ++j)
        dx[j] = (dy[j] - s[j] * D / (S + e)) / n;
}

/* h = t / nt, t = a + |alpha| (b - a), a = bf16(res / na), b = bf16(out / nb):
 *   dt = (dh - t (t . dh) / nt^2) / nt,
 *   da = (1 - |alpha|) dt,  db = |alpha| dt,
 *   dres = (da - res (res . da) / na^2) / na,  dout likewise with out, db, nb,
 *   dalpha_j (this row's part) = sign(alpha_j) (b_j - a_j) dt_j  (sign(0) = 0).
 * tmp holds 4*C doubles; dalpha_row may be NULL. */
void or_slerp_backward_row(const double *res, const double *out,
                           const double *alpha, const double *dh, int64_t C,
                           double eps, unsigned flags, double *tmp,
                           double *dres, double *dout, double *dalpha_row)
{
    double *a = tmp, *b = tmp + C, *t = tmp + 2 * C, *dt = tmp + 3 * C;
    double e = (flags & OR_EPS_ZERO) ? 0.0 : eps;
    double na2 = sum_sq(res, C) + e, nb2 = sum_sq(out, C) + e;
    double na = sqrt(na2), nb = sqrt(nb2);
    for (int64_t j = 0; j < C; ++j) {
        a[j] = res[j] / na;
        if (!(flags & OR_DROP_SLERP_A))
            a[j] = round_bf16(a[j]);
        b[j] = out[j] / nb;
        if (!(flags & OR_DROP_SLERP_B))
            b[j] = round_bf16(b[j]);
        t[j] = a[j] + fabs(alpha[j]) * (b[j] - a[j]);
    }
    double nt2 = sum_sq(t, C) + e, Dt = 0.0;
    for (int64_t j = 0; j < C; ++j)
        Dt += t[j] * dh[j];
    double nt = sqrt(nt2);
    double Da = 0.0, Db = 0.0;
    for (int64_t j = 0; j < C; ++j) {
        double m = fabs(alpha[j]);
        dt[j] = (dh[j] - t[j] * Dt / nt2) / nt;
        Da += res[j] * ((1.0 - m) * dt[j]);
        Db += out[j] * (m * dt[j]);
    }
    for (int64_t j = 0; j < C; ++j) {
        double m = fabs(alpha[j]);
        dres[j] = ((1.0 - m) * dt[j] - res[j] * Da / na2) / na;
        dout[j] = (m * dt[j] - out[j] * Db / nb2) / nb;
        if (dalpha_row) {
            double sg = alpha[j] > 0.0 ? 1.0 : alpha[j] < 0.0 ? -1.0 : 0.0;
            dalpha_row[j] = sg * (b[j] - a[j]) * dt[j];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Interval forms.                                                           */

static double dmin(double a, double b) { return a < b ? a : b; }
static double dmax(double a, double b) { return a > b ? a : b; }

/* bf16 bits of both ends of [v - delta|v|, v + delta|v|] (rounding is
 * monotone, so every value inside rounds between them). */
static void round_ends(double v, double delta, uint16_t *lo, uint16_t *hi)
{
    double w = delta * fabs(v);
    *lo = or_bf16_rne(v - w);
    *hi = or_bf16_rne(v + w);
}

void or_l2_row_interval(const double *x, const double *r, int64_t C,
                        double eps, double delta, unsigned flags, double *s,
                        uint16_t *lo, uint16_t *hi)
{
    for (int64_t j = 0; j < C; ++j) {
        if (!r)
            s[j] = x[j];
        else if (flags & OR_DROP_SUM_ROUND)
            s[j] = x[j] + r[j];
        else
            s[j] = round_bf16(x[j] + r[j]);
    }
    double n = row_norm(sum_sq(s, C), eps, flags);
    for (int64_t j = 0; j < C; ++j)
        round_ends(s[j] / n, delta, &lo[j], &hi[j]);
}

/* Interval of x / sqrt(S + eps) over x in [xl, xh], norm in [nl, nh] > 0. */
static void quotient_ends(double xl, double xh, double nl, double nh,
                          double delta, double *ql, double *qh)
{
    double c0 = xl / nl, c1 = xl / nh, c2 = xh / nl, c3 = xh / nh;
    double a = dmin(dmin(c0, c1), dmin(c2, c3));
    double b = dmax(dmax(c0, c1), dmax(c2, c3));
    *ql = a - delta * fabs(a);
    *qh = b + delta * fabs(b);
}

void or_slerp_row_interval(const double *res, const double *out,
                           const double *alpha, int64_t C, double eps,
                           double delta, unsigned flags, double *tmp,
                           uint16_t *lo, uint16_t *hi)
{
    double *tl = tmp, *th = tmp + C;
    double na = row_norm(sum_sq(res, C), eps, flags);
    double nb = row_norm(sum_sq(out, C), eps, flags);
    double Sl = 0.0, Sh = 0.0;
    for (int64_t j = 0; j < C; ++j) {
        /* a = bf16(l2(res)), b = bf16(l2(out)): both roundings of the ends */
        double va = res[j] / na, vb = out[j] / nb;
        double al = va - delta * fabs(va), ah = va + delta * fabs(va);
        double bl = vb - delta * fabs(vb), bh = vb + delta * fabs(vb);
        if (!(flags & OR_DROP_SLERP_A)) {
            al = round_bf16(al);
            ah = round_bf16(ah);
        }
        if (!(flags & OR_DROP_SLERP_B)) {
            bl = round_bf16(bl);
            bh = round_bf16(bh);
        }
        /* t = a + m (b - a) is affine in a and b: extremes at the corners */
        double m = fabs(alpha[j]);
        double t0 = al + m * (bl - al), t1 = al + m * (bh - al);
        double t2 = ah + m * (bl - ah), t3 = ah + m * (bh - ah);
        double lo_t = dmin(dmin(t0, t1), dmin(t2, t3));
        double hi_t = dmax(dmax(t0, t1), dmax(t2, t3));
        /* fp32 steps: the difference b - a (exact whenever float can hold
         * it), then a + m (b - a) rounded once (a fused multiply-add) */
        double dmag = dmax(dmax(fabs(bl - al), fabs(bh - al)),
                           dmax(fabs(bl - ah), fabs(bh - ah)));
        int d_exact = (double)(float)(bl - al) == bl - al &&
                      (double)(float)(bh - al) == bh - al &&
                      (double)(float)(bl - ah) == bl - ah &&
                      (double)(float)(bh - ah) == bh - ah;
        double dslack = d_exact ? 0.0 : delta * m * dmag;
        tl[j] = lo_t - delta * fabs(lo_t) - dslack;
        th[j] = hi_t + delta * fabs(hi_t) + dslack;
        double ql = tl[j] * tl[j], qh = th[j] * th[j];
        Sl += (tl[j] > 0.0 || th[j] < 0.0) ? dmin(ql, qh) : 0.0;
        Sh += dmax(ql, qh);
    }
    double nl = row_norm(Sl * (1.0 - delta), eps, flags);
    double nh = row_norm(Sh * (1.0 + delta), eps, flags);
    if (!(nl > 0.0) || !isfinite(nh)) {
        /* degenerate norm (zero row at eps = 0, non-finite input): the point
         * form decides; both ends carry its bits */
        or_slerp_row(res, out, alpha, C, eps, flags, tmp, lo, NULL);
        memcpy(hi, lo, sizeof(uint16_t) * (size_t)C);
        return;
    }
    for (int64_t j = 0; j < C; ++j) {
        double ql, qh;
        quotient_ends(tl[j], th[j], nl, nh, delta, &ql, &qh);
        lo[j] = or_bf16_rne(ql);
        hi[j] = or_bf16_rne(qh);
    }
}

/* ------------------------------------------------------------------------ */
/* [TF] Dory's gated and SwiGLU rows and their L2 norm: the rounding points
 * are the ones the pages list (the gated row; the scaled gate, the scaled up
 * and the product), then the output.  sigmoid and silu are the plain
 * definitions 1/(1+exp(-x)) and x/(1+exp(-x)) in double.                    */

static double sigmoid64(double z) { return 1.0 / (1.0 + exp(-z)); }
static double silu64(double x) { return x / (1.0 + exp(-x)); }

static double gate_value(double o, double g, double sg, unsigned flags)
{
    double v = o * sigmoid64(g * sg);
    return (flags & OR_DROP_GATED) ? v : round_bf16(v);
}

static double swiglu_value(double g, double u, double sug, double suu,
                           unsigned flags)
{
    double gs = g * sug, us = u * suu;
    if (!(flags & OR_DROP_SGATE))
        gs = round_bf16(gs);
    if (!(flags & OR_DROP_SUP))
        us = round_bf16(us);
    double v = silu64(gs) * us;
    return (flags & OR_DROP_PRODUCT) ? v : round_bf16(v);
}

/* The sigmoid, silu and per-element values above, exported so that the
 * tests can pin them at interior points against independent identities
 * (they are otherwise reachable only through a row's norm). */
double or_sigmoid(double z) { return sigmoid64(z); }
double or_silu(double x) { return silu64(x); }
double or_gate_value(double o, double g, double sg, unsigned flags) { return gate_value(o, g, sg, flags); }
double or_swiglu_value(double g, double u, double sug, double suu, unsigned flags)
{
    return swiglu_value(g, u, sug, suu, flags);
}

/* y = bf16(s / sqrt(sum s^2 + eps)) for a row whose s is already formed. */
static void l2_of(const double *s, int64_t C, double eps, unsigned flags,
                  uint16_t *y, double *y_exact)
{
    double n = row_norm(sum_sq(s, C), eps, flags);
    for (int64_t j = 0; j < C; ++j) {
        double v = s[j] / n;
        y[j] = or_bf16_rne(v);
        if (y_exact)
            y_exact[j] = v;
    }
}

/* The range an fp32 evaluation of sigmoid(z) can reach: the argument's own
 * rounding (2^-24 relative, through exp a relative |z| 2^-24), exp's 2 ulps,
 * 1 + e and the division move it by about (1 - s)(|z| 2^-23 + 2^-21) + 2^-22
 * (never less than delta); where -z > 87, exp(-z) is at or past fp32's
 * largest value and 1/(1+e) is subnormal or 0, so 0 is reachable. */
static void sigmoid_range(double z, double delta, double *lo, double *hi)
{
    double s = sigmoid64(z);
    double rel = (1.0 - s) * (fabs(z) * 0x1p-23 + 0x1p-21) + 0x1p-22;
    if (rel < delta)
        rel = delta;
    *lo = s * (1.0 - rel);
    *hi = s * (1.0 + rel);
    if (-z > 87.0) {
        *lo = 0.0;
        *hi = s * (1.0 + rel) + 0x1p-149;
    }
}

/* silu over [xl, xh] (xl <= xh), with the fp32 spread of each evaluation;
 * silu falls to its minimum at x0 = -1.2784645... and rises on both sides. */
static void silu_range(double xl, double xh, double delta, double *lo,
                       double *hi)
{
    double l = 1e300, h = -1e300;
    const double xs[2] = {xl, xh};
    for (int k = 0; k < 2; ++k) {
        double x = xs[k];
        double sl, sh;
        sigmoid_range(x, delta, &sl, &sh);
        double a = x * sl, b = x * sh; /* silu = x sigmoid(x) */
        double vl = dmin(a, b), vh = dmax(a, b);
        vl -= fabs(vl) * delta;
        vh += fabs(vh) * delta;
        if (-x > 87.0) { /* x / (1 + exp(-x)) is -0 once exp overflows */
            vh = dmax(vh, 0.0);
        }
        l = dmin(l, vl);
        h = dmax(h, vh);
    }
    const double x0 = -1.2784645427610738;
    if (xl <= x0 && x0 <= xh) {
        double m = silu64(x0);
        l = dmin(l, m - fabs(m) * delta);
    }
    *lo = l;
    *hi = h;
}

/* bf16 ends of [vl, vh] (or the ends themselves when the point is dropped). */
static void bf16_ends(double vl, double vh, int drop, double *l, double *h)
{
    if (drop) {
        *l = vl;
        *h = vh;
    } else {
        *l = round_bf16(vl);
        *h = round_bf16(vh);
    }
}

/* The product of two ranges. */
static void mul_range(double al, double ah, double bl, double bh, double *l,
                      double *h)
{
    double c0 = al * bl, c1 = al * bh, c2 = ah * bl, c3 = ah * bh;
    *l = dmin(dmin(c0, c1), dmin(c2, c3));
    *h = dmax(dmax(c0, c1), dmax(c2, c3));
}

/* l2 of a row whose elements lie in [sl_j, sh_j]: bf16 ends of each output. */
static void l2_interval_of(const double *sl, const double *sh, int64_t C,
                           double eps, double delta, unsigned flags,
                           uint16_t *lo, uint16_t *hi)
{
    double Sl = 0.0, Sh = 0.0;
    for (int64_t j = 0; j < C; ++j) {
        double ql = sl[j] * sl[j], qh = sh[j] * sh[j];
        Sl += (sl[j] > 0.0 || sh[j] < 0.0) ? dmin(ql, qh) : 0.0;
        Sh += dmax(ql, qh);
    }
    double nl = row_norm(Sl * (1.0 - delta), eps, flags);
    double nh = row_norm(Sh * (1.0 + delta), eps, flags);
    for (int64_t j = 0; j < C; ++j) {
        double ql, qh;
        if (!(nl > 0.0) || !isfinite(nh)) {
            ql = -INFINITY;
            qh = INFINITY;
        } else {
            quotient_ends(sl[j], sh[j], nl, nh, delta, &ql, &qh);
        }
        lo[j] = or_bf16_rne(ql);
        hi[j] = or_bf16_rne(qh);
    }
}

static void gate_row(const double *o, const double *g, const double *sg,
                     int64_t C, double eps, unsigned flags, double *s,
                     uint16_t *y, double *y_exact)
{
    for (int64_t j = 0; j < C; ++j)
        s[j] = gate_value(o[j], g[j], sg[j], flags);
    l2_of(s, C, eps, flags, y, y_exact);
}

static void swiglu_row(const double *g, const double *u, const double *sug,
                       const double *suu, int64_t C, double eps,
                       unsigned flags, double *s, uint16_t *y, double *y_exact)
{
    for (int64_t j = 0; j < C; ++j)
        s[j] = swiglu_value(g[j], u[j], sug[j], suu[j], flags);
    l2_of(s, C, eps, flags, y, y_exact);
}

static void gate_row_interval(const double *o, const double *g,
                              const double *sg, int64_t C, double eps,
                              double delta, unsigned flags, double *tmp,
                              uint16_t *lo, uint16_t *hi)
{
    double *sl = tmp, *sh = tmp + C;
    for (int64_t j = 0; j < C; ++j) {
        /* z = g sg is one fp32 product */
        double z = g[j] * sg[j], zl = z - fabs(z) * 0x1p-24, zh = z + fabs(z) * 0x1p-24;
        double a0, a1, b0, b1;
        sigmoid_range(zl, delta, &a0, &a1);
        sigmoid_range(zh, delta, &b0, &b1);
        double gl = dmin(a0, b0), gh = dmax(a1, b1), vl, vh;
        mul_range(o[j], o[j], gl, gh, &vl, &vh);
        vl -= fabs(vl) * delta;
        vh += fabs(vh) * delta;
        bf16_ends(vl, vh, flags & OR_DROP_GATED, &sl[j], &sh[j]);
    }
    l2_interval_of(sl, sh, C, eps, delta, flags, lo, hi);
}

static void swiglu_row_interval(const double *g, const double *u,
                                const double *sug, const double *suu,
                                int64_t C, double eps, double delta,
                                unsigned flags, double *tmp, uint16_t *lo,
                                uint16_t *hi)
{
    double *sl = tmp, *sh = tmp + C;
    for (int64_t j = 0; j < C; ++j) {
        double p = g[j] * sug[j], q = u[j] * suu[j];
        double gl, gh, ul, uh;
        bf16_ends(p - fabs(p) * 0x1p-24, p + fabs(p) * 0x1p-24, flags & OR_DROP_SGATE, &gl, &gh);
        bf16_ends(q - fabs(q) * 0x1p-24, q + fabs(q) * 0x1p-24, flags & OR_DROP_SUP, &ul, &uh);
        double fl, fh, vl, vh;
        silu_range(gl, gh, delta, &fl, &fh);
        mul_range(fl, fh, ul, uh, &vl, &vh);
        vl -= fabs(vl) * delta;
        vh += fabs(vh) * delta;
        bf16_ends(vl, vh, flags & OR_DROP_PRODUCT, &sl[j], &sh[j]);
    }
    l2_interval_of(sl, sh, C, eps, delta, flags, lo, hi);
}

/* ------------------------------------------------------------------------ */
/* Matrix drivers.  Each worker owns a contiguous range of rows and its own
 * scratch rows; inputs are widened to double exactly before the row call.   */

enum { OP_FWD, OP_BWD, OP_RENORM, OP_L2, OP_SLERP, OP_L2_IV, OP_SLERP_IV, OP_PROJECT, OP_MOMENTUM,
       OP_L2_BWD, OP_SLERP_BWD, OP_GATE, OP_SWIGLU, OP_GATE_IV, OP_SWIGLU_IV };

typedef struct {
    int op;
    int64_t r0, r1, C, ld, ld2;
    const float *w;
    const float *g;
    const void *gy;
    int gy_bf16;
    const uint16_t *x, *r;
    const float *alpha;
    const float *alpha2; /* swiglu: suu (alpha holds sg / sug) */
    double rho, eps, delta;
    unsigned flags;
    double *out_d;   /* dense [R, C] doubles */
    double *out_g;   /* [R] */
    double *out_d2;  /* dense [R, C] doubles (second output) */
    const uint16_t *dy; /* bf16 bits [R, ld] (activation backward) */
    uint16_t *out_h; /* dense [R, C] bf16 bits */
    uint16_t *out_h2; /* dense [R, C] bf16 bits (interval upper ends) */
    int status;
} job_t;

static void *run_job(void *arg)
{
    job_t *jb = (job_t *)arg;
    int64_t C = jb->C;
    double *buf = (double *)malloc(sizeof(double) * (size_t)(9 * C));
    if (!buf) {
        jb->status = -1;
        return NULL;
    }
    double *u = buf, *v = buf + C, *tmp = buf + 2 * C, *al = buf + 6 * C, *dv = buf + 7 * C, *al2 = buf + 8 * C;
    if (jb->op == OP_SLERP || jb->op == OP_SLERP_IV || jb->op == OP_SLERP_BWD || jb->op >= OP_GATE)
        for (int64_t j = 0; j < C; ++j)
            al[j] = (double)jb->alpha[j];
    if (jb->op == OP_SWIGLU || jb->op == OP_SWIGLU_IV)
        for (int64_t j = 0; j < C; ++j)
            al2[j] = (double)jb->alpha2[j];

    for (int64_t row = jb->r0; row < jb->r1; ++row) {
        size_t o = (size_t)row * (size_t)C;
        switch (jb->op) {
        case OP_FWD:
        case OP_RENORM: {
            const float *wr = jb->w + row * jb->ld;
            for (int64_t j = 0; j < C; ++j)
                u[j] = (double)wr[j];
            if (jb->op == OP_FWD)
                or_wn_forward_row(u, C, jb->g ? (double)jb->g[row] : 1.0,
                                  jb->rho, jb->eps, jb->flags, jb->out_d + o);
            else
                or_row_renorm_row(u, C, jb->rho, jb->eps, jb->flags,
                                  jb->out_d + o);
            break;
        }
        case OP_BWD: {
            const float *wr = jb->w + row * jb->ld;
            for (int64_t j = 0; j < C; ++j)
                u[j] = (double)wr[j];
            if (jb->gy_bf16) {
                const uint16_t *gr = (const uint16_t *)jb->gy + row * jb->ld2;
                for (int64_t j = 0; j < C; ++j)
                    v[j] = or_bf16_value(gr[j]);
            } else {
                const float *gr = (const float *)jb->gy + row * jb->ld2;
                for (int64_t j = 0; j < C; ++j)
                    v[j] = (double)gr[j];
            }
            double gg = 0.0;
            or_wn_backward_row(u, v, C, jb->g ? (double)jb->g[row] : 1.0,
                               jb->rho, jb->eps, jb->flags, jb->out_d + o, &gg);
            if (jb->out_g)
                jb->out_g[row] = gg;
            break;
        }
        case OP_PROJECT:
        case OP_MOMENTUM: {
            const float *wr = jb->w + row * jb->ld;
            const float *gr = (const float *)jb->gy + row * jb->ld2;
            for (int64_t j = 0; j < C; ++j) {
                u[j] = (double)wr[j];
                v[j] = (double)gr[j];
            }
            if (jb->op == OP_PROJECT)
                or_grad_project_row(u, v, C, jb->eps, jb->flags, jb->out_d + o);
            else
                or_renorm_momentum_row(u, v, C, jb->rho, jb->eps, jb->flags,
                                       jb->out_d2 + o, jb->out_d + o);
            break;
        }
        case OP_GATE:
        case OP_SWIGLU:
        case OP_GATE_IV:
        case OP_SWIGLU_IV: {
            const uint16_t *xr = jb->x + row * jb->ld;
            const uint16_t *rr = jb->r + row * jb->ld;
            for (int64_t j = 0; j < C; ++j) {
                u[j] = or_bf16_value(xr[j]);
                v[j] = or_bf16_value(rr[j]);
            }
            double *ye = jb->out_d ? jb->out_d + o : NULL;
            if (jb->op == OP_GATE)
                gate_row(u, v, al, C, jb->eps, jb->flags, tmp, jb->out_h + o, ye);
            else if (jb->op == OP_SWIGLU)
                swiglu_row(u, v, al, al2, C, jb->eps, jb->flags, tmp, jb->out_h + o, ye);
            else if (jb->op == OP_GATE_IV)
                gate_row_interval(u, v, al, C, jb->eps, jb->delta, jb->flags, tmp, jb->out_h + o,
                                  jb->out_h2 + o);
            else
                swiglu_row_interval(u, v, al, al2, C, jb->eps, jb->delta, jb->flags, tmp, jb->out_h + o,
                                    jb->out_h2 + o);
            break;
        }
        case OP_L2_BWD:
        case OP_SLERP_BWD: {
            const uint16_t *xr = jb->x + row * jb->ld;
            const uint16_t *dr = jb->dy + row * jb->ld;
            for (int64_t j = 0; j < C; ++j) {
                u[j] = or_bf16_value(xr[j]);
                dv[j] = or_bf16_value(dr[j]);
            }
            if (jb->r) {
                const uint16_t *rr = jb->r + row * jb->ld;
                for (int64_t j = 0; j < C; ++j)
                    v[j] = or_bf16_value(rr[j]);
            }
            if (jb->op == OP_L2_BWD)
                or_l2_backward_row(u, jb->r ? v : NULL, dv, C, jb->eps, jb->flags, tmp, jb->out_d + o);
            else
                or_slerp_backward_row(u, v, al, dv, C, jb->eps, jb->flags, tmp, jb->out_d + o,
                                      jb->out_d2 + o, NULL);
            break;
        }
        case OP_L2:
        case OP_L2_IV: {
            const uint16_t *xr = jb->x + row * jb->ld;
            for (int64_t j = 0; j < C; ++j)
                u[j] = or_bf16_value(xr[j]);
            const double *rp = NULL;
            if (jb->r) {
                const uint16_t *rr = jb->r + row * jb->ld;
                for (int64_t j = 0; j < C; ++j)
                    v[j] = or_bf16_value(rr[j]);
                rp = v;
            }
            if (jb->op == OP_L2)
                or_l2_row(u, rp, C, jb->eps, jb->flags, tmp, jb->out_h + o,
                          jb->out_d ? jb->out_d + o : NULL);
            else
                or_l2_row_interval(u, rp, C, jb->eps, jb->delta, jb->flags,
                                   tmp, jb->out_h + o, jb->out_h2 + o);
            break;
        }
        case OP_SLERP:
        case OP_SLERP_IV: {
            const uint16_t *xr = jb->x + row * jb->ld;
            const uint16_t *rr = jb->r + row * jb->ld;
            for (int64_t j = 0; j < C; ++j) {
                u[j] = or_bf16_value(xr[j]);
                v[j] = or_bf16_value(rr[j]);
            }
            if (jb->op == OP_SLERP)
                or_slerp_row(u, v, al, C, jb->eps, jb->flags, tmp,
                             jb->out_h + o, jb->out_d ? jb->out_d + o : NULL);
            else
                or_slerp_row_interval(u, v, al, C, jb->eps, jb->delta,
                                      jb->flags, tmp, jb->out_h + o,
                                      jb->out_h2 + o);
            break;
        }
        }
    }
    free(buf);
    jb->status = 0;
    return NULL;
}

static int run_rows(const job_t *proto, int64_t R, int nthreads)
{
    if (R <= 0)
        return 0;
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > R)
        nthreads = (int)R;
    job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t *tid = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    int *started = (int *)calloc((size_t)nthreads, sizeof(int));
    if (!jobs || !tid || !started) {
        free(jobs);
        free(tid);
        free(started);
        return -1;
    }
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = *proto;
        jobs[t].r0 = R * t / nthreads;
        jobs[t].r1 = R * (t + 1) / nthreads;
        jobs[t].status = -1;
    }
    for (int t = 1; t < nthreads; ++t)
        started[t] = pthread_create(&tid[t], NULL, run_job, &jobs[t]) == 0;
    run_job(&jobs[0]);
    int rc = jobs[0].status;
    for (int t = 1; t < nthreads; ++t) {
        if (started[t])
            pthread_join(tid[t], NULL);
        else
            run_job(&jobs[t]);
        if (jobs[t].status != 0)
            rc = -1;
    }
    free(jobs);
    free(tid);
    free(started);
    return rc;
}

static int bad_shape(int64_t R, int64_t C, int64_t ld)
{
    return R < 0 || C < 1 || ld < C;
}

int or_wn_forward(const float *w, int64_t R, int64_t C, int64_t ld,
                  const float *g, double rho, double eps, unsigned flags,
                  double *out, int nthreads)
{
    if (bad_shape(R, C, ld) || (R > 0 && (!w || !out)))
        return -1;
    job_t jb = {0};
    jb.op = OP_FWD;
    jb.C = C;
    jb.ld = ld;
    jb.w = w;
    jb.g = g;
    jb.rho = rho;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_d = out;
    return run_rows(&jb, R, nthreads);
}

int or_wn_backward(const float *w, int64_t R, int64_t C, int64_t ld,
                   const void *gy, int gy_is_bf16, int64_t ld_gy,
                   const float *g, double rho, double eps, unsigned flags,
                   double *grad_w, double *grad_g, int nthreads)
{
    if (bad_shape(R, C, ld) || ld_gy < C || (R > 0 && (!w || !gy || !grad_w)))
        return -1;
    if (flags & ~(OR_EPS_ZERO | OR_BWD_PRINTED))
        return -1;
    job_t jb = {0};
    jb.op = OP_BWD;
    jb.C = C;
    jb.ld = ld;
    jb.ld2 = ld_gy;
    jb.w = w;
    jb.g = g;
    jb.gy = gy;
    jb.gy_bf16 = gy_is_bf16;
    jb.rho = rho;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_d = grad_w;
    jb.out_g = grad_g;
    return run_rows(&jb, R, nthreads);
}

int or_grad_project(const float *w, int64_t R, int64_t C, int64_t ld,
                    const float *G, int64_t ld_g, double eps, unsigned flags,
                    double *out, int nthreads)
{
    if (bad_shape(R, C, ld) || ld_g < C || (R > 0 && (!w || !G || !out)))
        return -1;
    if (flags & ~OR_EPS_ZERO)
        return -1;
    job_t jb = {0};
    jb.op = OP_PROJECT;
    jb.C = C;
    jb.ld = ld;
    jb.ld2 = ld_g;
    jb.w = w;
    jb.gy = G;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_d = out;
    return run_rows(&jb, R, nthreads);
}

int or_renorm_momentum(const float *w, int64_t R, int64_t C, int64_t ld,
                       const float *m, int64_t ld_m, double rho, double eps,
                       unsigned flags, double *w_out, double *m_out,
                       int nthreads)
{
    if (bad_shape(R, C, ld) || ld_m < C ||
        (R > 0 && (!w || !m || !w_out || !m_out)))
        return -1;
    if (flags & ~OR_EPS_ZERO)
        return -1;
    job_t jb = {0};
    jb.op = OP_MOMENTUM;
    jb.C = C;
    jb.ld = ld;
    jb.ld2 = ld_m;
    jb.w = w;
    jb.gy = m;
    jb.rho = rho;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_d = m_out;
    jb.out_d2 = w_out;
    return run_rows(&jb, R, nthreads);
}

static int fused_rows(int op, const uint16_t *a, const uint16_t *b,
                      const float *sa, const float *sb, int64_t R, int64_t C,
                      int64_t ld, double eps, double delta, unsigned flags,
                      uint16_t *y, uint16_t *y2, double *y_exact, int nthreads)
{
    const unsigned allowed = (op == OP_GATE || op == OP_GATE_IV)
                                 ? (OR_DROP_GATED | OR_EPS_ZERO | OR_EPS_OUTSIDE)
                                 : (OR_DROP_SGATE | OR_DROP_SUP | OR_DROP_PRODUCT | OR_EPS_ZERO | OR_EPS_OUTSIDE);
    if (bad_shape(R, C, ld) || !sa || ((op == OP_SWIGLU || op == OP_SWIGLU_IV) && !sb) ||
        (R > 0 && (!a || !b || !y || ((op == OP_GATE_IV || op == OP_SWIGLU_IV) && !y2))) || (flags & ~allowed))
        return -1;
    job_t jb = {0};
    jb.op = op;
    jb.C = C;
    jb.ld = ld;
    jb.x = a;
    jb.r = b;
    jb.alpha = sa;
    jb.alpha2 = sb;
    jb.eps = eps;
    jb.delta = delta;
    jb.flags = flags;
    jb.out_h = y;
    jb.out_h2 = y2;
    jb.out_d = y_exact;
    return run_rows(&jb, R, nthreads);
}

int or_gate_l2_rows(const uint16_t *o, const uint16_t *g, const float *sg,
                    int64_t R, int64_t C, int64_t ld, double eps,
                    unsigned flags, uint16_t *y, double *y_exact, int nthreads)
{
    return fused_rows(OP_GATE, o, g, sg, NULL, R, C, ld, eps, 0.0, flags, y, NULL, y_exact, nthreads);
}

int or_swiglu_l2_rows(const uint16_t *g, const uint16_t *u, const float *sug,
                      const float *suu, int64_t R, int64_t C, int64_t ld,
                      double eps, unsigned flags, uint16_t *y, double *y_exact,
                      int nthreads)
{
    return fused_rows(OP_SWIGLU, g, u, sug, suu, R, C, ld, eps, 0.0, flags, y, NULL, y_exact, nthreads);
}

int or_gate_l2_rows_interval(const uint16_t *o, const uint16_t *g,
                             const float *sg, int64_t R, int64_t C, int64_t ld,
                             double eps, double delta, unsigned flags,
                             uint16_t *lo, uint16_t *hi, int nthreads)
{
    return fused_rows(OP_GATE_IV, o, g, sg, NULL, R, C, ld, eps, delta, flags, lo, hi, NULL, nthreads);
}

int or_swiglu_l2_rows_interval(const uint16_t *g, const uint16_t *u,
                               const float *sug, const float *suu, int64_t R,
                               int64_t C, int64_t ld, double eps, double delta,
                               unsigned flags, uint16_t *lo, uint16_t *hi,
                               int nthreads)
{
    return fused_rows(OP_SWIGLU_IV, g, u, sug, suu, R, C, ld, eps, delta, flags, lo, hi, NULL, nthreads);
}

int or_l2_rows_backward(const uint16_t *x, const uint16_t *r,
                        const uint16_t *dy, int64_t R, int64_t C, int64_t ld,
                        double eps, unsigned flags, double *dx, int nthreads)
{
    if (bad_shape(R, C, ld) || (R > 0 && (!x || !dy || !dx)))
        return -1;
    if (flags & ~(OR_EPS_ZERO | OR_DROP_SUM_ROUND))
        return -1;
    job_t jb = {0};
    jb.op = OP_L2_BWD;
    jb.C = C;
    jb.ld = ld;
    jb.x = x;
    jb.r = r;
    jb.dy = dy;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_d = dx;
    return run_rows(&jb, R, nthreads);
}

int or_slerp_rows_backward(const uint16_t *res, const uint16_t *out,
                           const float *alpha, const uint16_t *dh, int64_t R,
                           int64_t C, int64_t ld, double eps, unsigned flags,
                           double *dres, double *dout, double *dalpha,
                           int nthreads)
{
    if (bad_shape(R, C, ld) || !alpha || (R > 0 && (!res || !out || !dh || !dres || !dout)))
        return -1;
    if (flags & ~(OR_EPS_ZERO | OR_DROP_SLERP_A | OR_DROP_SLERP_B))
        return -1;
    job_t jb = {0};
    jb.op = OP_SLERP_BWD;
    jb.C = C;
    jb.ld = ld;
    jb.x = res;
    jb.r = out;
    jb.alpha = alpha;
    jb.dy = dh;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_d = dres;
    jb.out_d2 = dout;
    int rc = run_rows(&jb, R, nthreads);
    if (rc != 0 || !dalpha)
        return rc;
    /* dalpha: the rows' parts summed in row order (one thread) */
    double *tmp = (double *)malloc(sizeof(double) * (size_t)(9 * C));
    if (!tmp)
        return -1;
    double *u = tmp + 4 * C, *v = tmp + 5 * C, *al = tmp + 6 * C, *dv = tmp + 7 * C, *part = tmp + 8 * C;
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(2 * C));
    if (!scratch) {
        free(tmp);
        return -1;
    }
    for (int64_t j = 0; j < C; ++j) {
        al[j] = (double)alpha[j];
        dalpha[j] = 0.0;
    }
    for (int64_t row = 0; row < R; ++row) {
        for (int64_t j = 0; j < C; ++j) {
            u[j] = or_bf16_value(res[row * ld + j]);
            v[j] = or_bf16_value(out[row * ld + j]);
            dv[j] = or_bf16_value(dh[row * ld + j]);
        }
        or_slerp_backward_row(u, v, al, dv, C, eps, flags, tmp, scratch, scratch + C, part);
        for (int64_t j = 0; j < C; ++j)
            dalpha[j] += part[j];
    }
    free(scratch);
    free(tmp);
    return 0;
}

int or_row_renorm(const float *w, int64_t R, int64_t C, int64_t ld, double rho,
                  double eps, unsigned flags, double *out, int nthreads)
{
    if (bad_shape(R, C, ld) || (R > 0 && (!w || !out)))
        return -1;
    job_t jb = {0};
    jb.op = OP_RENORM;
    jb.C = C;
    jb.ld = ld;
    jb.w = w;
    jb.rho = rho;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_d = out;
    return run_rows(&jb, R, nthreads);
}

int or_l2_rows(const uint16_t *x, const uint16_t *r, int64_t R, int64_t C,
               int64_t ld, double eps, unsigned flags, uint16_t *y,
               double *y_exact, int nthreads)
{
    if (bad_shape(R, C, ld) || (R > 0 && (!x || !y)))
        return -1;
    job_t jb = {0};
    jb.op = OP_L2;
    jb.C = C;
    jb.ld = ld;
    jb.x = x;
    jb.r = r;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_h = y;
    jb.out_d = y_exact;
    return run_rows(&jb, R, nthreads);
}

int or_slerp_rows(const uint16_t *res, const uint16_t *out, const float *alpha,
                  int64_t R, int64_t C, int64_t ld, double eps, unsigned flags,
                  uint16_t *h, double *h_exact, int nthreads)
{
    if (bad_shape(R, C, ld) || (R > 0 && (!res || !out || !alpha || !h)))
        return -1;
    job_t jb = {0};
    jb.op = OP_SLERP;
    jb.C = C;
    jb.ld = ld;
    jb.x = res;
    jb.r = out;
    jb.alpha = alpha;
    jb.eps = eps;
    jb.flags = flags;
    jb.out_h = h;
    jb.out_d = h_exact;
    return run_rows(&jb, R, nthreads);
}

int or_l2_rows_interval(const uint16_t *x, const uint16_t *r, int64_t R,
                        int64_t C, int64_t ld, double eps, double delta,
                        unsigned flags, uint16_t *lo, uint16_t *hi,
                        int nthreads)
{
    if (bad_shape(R, C, ld) || !(delta >= 0.0) || (R > 0 && (!x || !lo || !hi)))
        return -1;
    job_t jb = {0};
    jb.op = OP_L2_IV;
    jb.C = C;
    jb.ld = ld;
    jb.x = x;
    jb.r = r;
    jb.eps = eps;
    jb.delta = delta;
    jb.flags = flags;
    jb.out_h = lo;
    jb.out_h2 = hi;
    return run_rows(&jb, R, nthreads);
}

int or_slerp_rows_interval(const uint16_t *res, const uint16_t *out,
                           const float *alpha, int64_t R, int64_t C,
                           int64_t ld, double eps, double delta,
                           unsigned flags, uint16_t *lo, uint16_t *hi,
                           int nthreads)
{
    if (bad_shape(R, C, ld) || !(delta >= 0.0) ||
        (R > 0 && (!res || !out || !alpha || !lo || !hi)))
        return -1;
    job_t jb = {0};
    jb.op = OP_SLERP_IV;
    jb.C = C;
    jb.ld = ld;
    jb.x = res;
    jb.r = out;
    jb.alpha = alpha;
    jb.eps = eps;
    jb.delta = delta;
    jb.flags = flags;
    jb.out_h = lo;
    jb.out_h2 = hi;
    return run_rows(&jb, R, nthreads);
}

/* ------------------------------------------------------------------------ */
/* [TF] tf_qk_rows_l2: rotate-half RoPE on a head's bf16 values (the halves
 * x_i, x_{i+h} turned by the fp32 angle p inv_i, as the tern-tc listing's
 * apply_rope computes in fp32 and casts back), the head's L2 norm with eps on
 * the sum, and q's fp32 scale after the normalized head's rounding.         */

/* The angle torch forms: fp32(p) * inv_i, one fp32 product.  A 24-bit by
 * 24-bit product is exact in double; the cast rounds it to fp32. */
static double rope_angle(int32_t p, float inv)
{
    return (double)(float)((double)(float)p * (double)inv);
}

static void rope_head(const double *x, int32_t D, int32_t p, const float *inv,
                      unsigned flags, double *rot)
{
    const int32_t h = D / 2;
    for (int32_t i = 0; i < h; ++i) {
        double th = rope_angle(p, inv[i]);
        double c = cos(th), s = sin(th);
        double a = x[i] * c - x[i + h] * s;
        double b = x[i] * s + x[i + h] * c;
        rot[i] = (flags & OR_DROP_ROT) ? a : round_bf16(a);
        rot[i + h] = (flags & OR_DROP_ROT) ? b : round_bf16(b);
    }
}

/* One head: rot, then y = rot / n; q scales y (rounded unless dropped). */
static void qk_head(const double *x, int32_t D, int32_t p, const float *inv,
                    const float *scale, int is_q, double eps, unsigned flags,
                    double *rot, uint16_t *out, double *out_exact)
{
    rope_head(x, D, p, inv, flags, rot);
    double n = row_norm(sum_sq(rot, D), eps, flags);
    for (int32_t j = 0; j < D; ++j) {
        double y = rot[j] / n, v;
        if (is_q) {
            double yr = (flags & OR_DROP_QNORM) ? y : round_bf16(y);
            v = scale ? yr * (double)scale[j] : yr;
        } else {
            v = y;
        }
        out[j] = or_bf16_rne(v);
        if (out_exact)
            out_exact[j] = v;
    }
}

/* fp32's unit in the last place of v (subnormal spacing below 2^-126). */
static double ulp32(double v)
{
    double a = fabs(v);
    if (!(a >= 0x1p-126))
        return 0x1p-149;
    int e;
    (void)frexp(a, &e); /* a in [2^(e-1), 2^e) */
    return ldexp(1.0, e - 1 - 23);
}

static void qk_head_interval(const double *x, int32_t D, int32_t p,
                             const float *inv, const float *scale, int is_q,
                             double eps, double delta, unsigned flags,
                             double *tmp, uint16_t *lo, uint16_t *hi)
{
    const int32_t h = D / 2;
    double *sl = tmp, *sh = tmp + D, *yl = tmp + 2 * D, *yh = tmp + 3 * D;
    const double w32 = delta > 0x1p-23 ? delta : 0x1p-23;
    for (int32_t i = 0; i < h; ++i) {
        double th = rope_angle(p, inv[i]);
        double c = cos(th), s = sin(th);
        /* cosf / sinf: 2 ulps of the result, never less than delta */
        double ec = 2.0 * ulp32(c) + fabs(c) * delta, es = 2.0 * ulp32(s) + fabs(s) * delta;
        double cl = c - ec, ch = c + ec, s_l = s - es, s_h = s + es;
        double cm = dmax(fabs(cl), fabs(ch)), smx = dmax(fabs(s_l), fabs(s_h));
        const double x1 = x[i], x2 = x[i + h];
        double p0, p1, q0, q1, r0, r1, t0, t1;
        mul_range(x1, x1, cl, ch, &p0, &p1);  /* x1 cos */
        mul_range(x2, x2, s_l, s_h, &q0, &q1); /* x2 sin */
        mul_range(x1, x1, s_l, s_h, &r0, &r1); /* x1 sin */
        mul_range(x2, x2, cl, ch, &t0, &t1);  /* x2 cos */
        /* two fp32 products and their sum: each rounding within w32 of
         * the magnitudes it touches */
        double wa = w32 * (fabs(x1) * cm + fabs(x2) * smx) * 2.0;
        double wb = w32 * (fabs(x1) * smx + fabs(x2) * cm) * 2.0;
        bf16_ends(p0 - q1 - wa, p1 - q0 + wa, flags & OR_DROP_ROT, &sl[i], &sh[i]);
        bf16_ends(r0 + t0 - wb, r1 + t1 + wb, flags & OR_DROP_ROT, &sl[i + h], &sh[i + h]);
    }
    double Sl = 0.0, Sh = 0.0;
    for (int32_t j = 0; j < D; ++j) {
        double ql = sl[j] * sl[j], qh = sh[j] * sh[j];
        Sl += (sl[j] > 0.0 || sh[j] < 0.0) ? dmin(ql, qh) : 0.0;
        Sh += dmax(ql, qh);
    }
    double nl = row_norm(Sl * (1.0 - delta), eps, flags);
    double nh = row_norm(Sh * (1.0 + delta), eps, flags);
    for (int32_t j = 0; j < D; ++j) {
        if (!(nl > 0.0) || !isfinite(nh)) {
            yl[j] = -INFINITY;
            yh[j] = INFINITY;
        } else {
            quotient_ends(sl[j], sh[j], nl, nh, delta, &yl[j], &yh[j]);
        }
        double vl = yl[j], vh = yh[j];
        if (is_q) {
            bf16_ends(vl, vh, flags & OR_DROP_QNORM, &vl, &vh);
            if (scale) {
                double a = vl * (double)scale[j], b = vh * (double)scale[j];
                vl = dmin(a, b);
                vh = dmax(a, b);
                vl -= fabs(vl) * delta;
                vh += fabs(vh) * delta;
            }
        }
        lo[j] = or_bf16_rne(vl);
        hi[j] = or_bf16_rne(vh);
    }
}

typedef struct {
    int iv;
    int64_t r0, r1, ld_q, ld_k;
    int32_t D, hq, hk;
    const uint16_t *q, *k;
    const int32_t *pos;
    const float *inv, *scale;
    double eps, delta;
    unsigned flags;
    uint16_t *qa, *qb, *ka, *kb; /* point: q_out, -, k_out, -; interval: lo, hi */
    double *qe, *ke;
    int status;
} qk_job_t;

static void *run_qk_job(void *arg)
{
    qk_job_t *jb = (qk_job_t *)arg;
    const int32_t D = jb->D;
    double *buf = (double *)malloc(sizeof(double) * (size_t)(5 * D));
    if (!buf) {
        jb->status = -1;
        return NULL;
    }
    double *x = buf, *tmp = buf + D;
    for (int64_t row = jb->r0; row < jb->r1; ++row) {
        const int32_t p = jb->pos[row];
        for (int part = 0; part < 2; ++part) {
            const int is_q = part == 0;
            const int32_t H = is_q ? jb->hq : jb->hk;
            const uint16_t *src = is_q ? jb->q + row * jb->ld_q : jb->k + row * jb->ld_k;
            const int64_t o = row * (int64_t)H * D;
            for (int32_t hd = 0; hd < H; ++hd) {
                for (int32_t j = 0; j < D; ++j)
                    x[j] = or_bf16_value(src[(int64_t)hd * D + j]);
                const float *sc = (is_q && jb->scale) ? jb->scale + (int64_t)hd * D : NULL;
                const int64_t oo = o + (int64_t)hd * D;
                if (jb->iv) {
                    qk_head_interval(x, D, p, jb->inv, sc, is_q, jb->eps, jb->delta, jb->flags, tmp,
                                     (is_q ? jb->qa : jb->ka) + oo, (is_q ? jb->qb : jb->kb) + oo);
                } else {
                    double *ex = is_q ? jb->qe : jb->ke;
                    qk_head(x, D, p, jb->inv, sc, is_q, jb->eps, jb->flags, tmp,
                            (is_q ? jb->qa : jb->ka) + oo, ex ? ex + oo : NULL);
                }
            }
        }
    }
    free(buf);
    jb->status = 0;
    return NULL;
}

static int run_qk(const qk_job_t *proto, int64_t R, int nthreads)
{
    if (R <= 0)
        return 0;
    if (nthreads < 1)
        nthreads = 1;
    if ((int64_t)nthreads > R)
        nthreads = (int)R;
    qk_job_t *jobs = (qk_job_t *)calloc((size_t)nthreads, sizeof(qk_job_t));
    pthread_t *tid = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    int *started = (int *)calloc((size_t)nthreads, sizeof(int));
    if (!jobs || !tid || !started) {
        free(jobs);
        free(tid);
        free(started);
        return -1;
    }
    for (int t = 0; t < nthreads; ++t) {
        jobs[t] = *proto;
        jobs[t].r0 = R * t / nthreads;
        jobs[t].r1 = R * (t + 1) / nthreads;
        jobs[t].status = -1;
    }
    for (int t = 1; t < nthreads; ++t)
        started[t] = pthread_create(&tid[t], NULL, run_qk_job, &jobs[t]) == 0;
    run_qk_job(&jobs[0]);
    int rc = jobs[0].status;
    for (int t = 1; t < nthreads; ++t) {
        if (started[t])
            pthread_join(tid[t], NULL);
        else
            run_qk_job(&jobs[t]);
        if (jobs[t].status != 0)
            rc = -1;
    }
    free(jobs);
    free(tid);
    free(started);
    return rc;
}

static int qk_bad(int64_t R, int32_t D, int32_t hq, int32_t hk, int64_t ld_q,
                  int64_t ld_k, const uint16_t *q, const uint16_t *k,
                  const int32_t *pos, const float *inv, unsigned flags)
{
    const unsigned allowed = OR_DROP_ROT | OR_DROP_QNORM | OR_EPS_ZERO | OR_EPS_OUTSIDE;
    if (R < 0 || D < 2 || D % 2 || hq < 0 || hk < 0 || (flags & ~allowed))
        return 1;
    if (ld_q < (int64_t)hq * D || ld_k < (int64_t)hk * D)
        return 1;
    return R > 0 && (!pos || !inv || (hq && !q) || (hk && !k));
}

int or_qk_rows_l2(const uint16_t *q, int64_t ld_q, const uint16_t *k,
                  int64_t ld_k, int64_t R, int32_t D, int32_t hq, int32_t hk,
                  const int32_t *pos, const float *inv, const float *q_scale,
                  double eps, unsigned flags, uint16_t *q_out, uint16_t *k_out,
                  double *q_exact, double *k_exact, int nthreads)
{
    if (qk_bad(R, D, hq, hk, ld_q, ld_k, q, k, pos, inv, flags) ||
        (R > 0 && ((hq && !q_out) || (hk && !k_out))))
        return -1;
    qk_job_t jb = {0};
    jb.ld_q = ld_q;
    jb.ld_k = ld_k;
    jb.D = D;
    jb.hq = hq;
    jb.hk = hk;
    jb.q = q;
    jb.k = k;
    jb.pos = pos;
    jb.inv = inv;
    jb.scale = q_scale;
    jb.eps = eps;
    jb.flags = flags;
    jb.qa = q_out;
    jb.ka = k_out;
    jb.qe = q_exact;
    jb.ke = k_exact;
    return run_qk(&jb, R, nthreads);
}

int or_qk_rows_l2_interval(const uint16_t *q, int64_t ld_q, const uint16_t *k,
                           int64_t ld_k, int64_t R, int32_t D, int32_t hq,
                           int32_t hk, const int32_t *pos, const float *inv,
                           const float *q_scale, double eps, double delta,
                           unsigned flags, uint16_t *q_lo, uint16_t *q_hi,
                           uint16_t *k_lo, uint16_t *k_hi, int nthreads)
{
    if (qk_bad(R, D, hq, hk, ld_q, ld_k, q, k, pos, inv, flags) ||
        (R > 0 && ((hq && (!q_lo || !q_hi)) || (hk && (!k_lo || !k_hi)))))
        return -1;
    qk_job_t jb = {0};
    jb.iv = 1;
    jb.ld_q = ld_q;
    jb.ld_k = ld_k;
    jb.D = D;
    jb.hq = hq;
    jb.hk = hk;
    jb.q = q;
    jb.k = k;
    jb.pos = pos;
    jb.inv = inv;
    jb.scale = q_scale;
    jb.eps = eps;
    jb.delta = delta;
    jb.flags = flags;
    jb.qa = q_lo;
    jb.qb = q_hi;
    jb.ka = k_lo;
    jb.kb = k_hi;
    return run_qk(&jb, R, nthreads);
}

/* ------------------------------------------------------------------------ */
/* [DS] "Monitor" and `init` "preserve": the row length sqrt(sum w^2 + eps),
 * divided by `div` (1, or rho for the gain that keeps W_eff = w).           */

int or_row_norms(const float *w, int64_t R, int64_t C, int64_t ld, double eps,
                 double div, double *out, int nthreads)
{
    (void)nthreads; /* one pass of R sums: no threads needed */
    if (bad_shape(R, C, ld) || (R > 0 && (!w || !out)) || !(div > 0.0))
        return -1;
    for (int64_t r = 0; r < R; ++r) {
        const float *wr = w + r * ld;
        double S = 0.0;
        for (int64_t j = 0; j < C; ++j)
            S += (double)wr[j] * (double)wr[j];
        out[r] = sqrt(S + eps) / div;
    }
    return 0;
}

/* [DS] `gain` "scalar": the channel backward with every g_r = g, and the
 * per-row gain gradients summed in row order. */
int or_wn_backward_scalar_gain(const float *w, int64_t R, int64_t C,
                               int64_t ld, const void *gy, int gy_is_bf16,
                               int64_t ld_gy, float g, double rho, double eps,
                               unsigned flags, double *grad_w, double *gg_rows,
                               double *gg_sum, int nthreads)
{
    if (bad_shape(R, C, ld) || !gg_sum || (R > 0 && !gg_rows))
        return -1;
    float *gv = (float *)calloc((size_t)(R > 0 ? R : 1), sizeof(float));
    if (!gv)
        return -1;
    for (int64_t r = 0; r < R; ++r)
        gv[r] = g;
    int rc = or_wn_backward(w, R, C, ld, gy, gy_is_bf16, ld_gy, gv, rho, eps,
                            flags, grad_w, gg_rows, nthreads);
    free(gv);
    if (rc != 0)
        return rc;
    double acc = 0.0;
    for (int64_t r = 0; r < R; ++r)
        acc += gg_rows[r];
    *gg_sum = acc;
    return 0;
}
