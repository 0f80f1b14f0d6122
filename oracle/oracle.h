/*
 * oracle.h -- float64 CPU oracle for per-row L2 normalisation.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library under l2_row_b200/) never calls it, shares no code, header,
 * table or constant with it, and must fail loudly when its own extension is
 * missing instead of falling back here.
 *
 * Every function is the plain definition of the operation, written one row
 * at a time, left to right, in double precision, with the bf16 rounding
 * points the sources state applied explicitly (f64 -> bf16 directly, round to
 * nearest, ties to even; never through float).
 *
 * Sources:
 *   [DS]  DragonScale package description (PyPI), sections "What DragonScale
 *         changes" (eq. W_eff, eq. dL/dW), "Patching options" (options table:
 *         mode, method) and "Optimizer" (rescale after the step).
 *   [TF]  TensorFold pull request #1260 (Dory native CUDA family),
 *         Conversation, the norms.cu commit describing tf_l2_rows and
 *         tf_slerp_rows.
 *
 * Parity pins live in tests/ (closed forms, invariants, central finite
 * differences, exact-rational fixtures under tests/golden/, negative controls).
 */
#ifndef L2ROW_ORACLE_H
#define L2ROW_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Variant flags.  0 = the definition.  Every other bit plants one deliberate
 * deviation so that tests can show the checker is sharp (negative controls). */
#define OR_DROP_SUM_ROUND 0x01u /* l2_rows: use x + r unrounded instead of bf16(x + r)   */
#define OR_DROP_SLERP_A   0x02u /* slerp: use l2(res) unrounded instead of bf16(l2(res)) */
#define OR_DROP_SLERP_B   0x04u /* slerp: use l2(out) unrounded instead of bf16(l2(out)) */
#define OR_EPS_OUTSIDE    0x08u /* norm = sqrt(S) + eps instead of sqrt(S + eps)         */
#define OR_EPS_ZERO       0x10u /* norm = sqrt(S), eps ignored                           */
#define OR_BWD_PRINTED    0x20u /* backward: project with S instead of S + eps (the
                                   eps-free form of the printed dL/dW)                   */
#define OR_DROP_GATED     0x40u /* gate_l2: use o * sigmoid(g sg) unrounded (the gated row) */
#define OR_DROP_SGATE     0x80u /* swiglu_l2: use g * sug unrounded (the scaled gate)       */
#define OR_DROP_SUP       0x100u /* swiglu_l2: use u * suu unrounded (the scaled up)        */
#define OR_DROP_PRODUCT   0x200u /* swiglu_l2: use silu(.) * (.) unrounded (the product)    */
#define OR_DROP_ROT       0x400u /* qk_rows_l2: use the rotated head unrounded              */
#define OR_DROP_QNORM     0x800u /* qk_rows_l2: use q's normalized head unrounded           */

/* bf16 helpers.  or_bf16_rne rounds a double straight to bf16 bits. */
uint16_t or_bf16_rne(double v);
double   or_bf16_value(uint16_t bits);

/* [TF] Dory rows, one element: sigmoid(z) = 1/(1+exp(-z)), silu(x) =
 * x/(1+exp(-x)), the gated value bf16(o sigmoid(g sg)) and the SwiGLU value
 * bf16(silu(bf16(g sug)) bf16(u suu)) (flags drop their rounding points). */
double or_sigmoid(double z);
double or_silu(double x);
double or_gate_value(double o, double g, double sg, unsigned flags);
double or_swiglu_value(double g, double u, double sug, double suu, unsigned flags);
/* or_bf16_rne over an array (dst[i] = or_bf16_rne(src[i])). */
void     or_bf16_rne_array(const double *src, int64_t n, uint16_t *dst);

/* ---- one row, all values already exact doubles -------------------------- */

/* [DS] eq. W_eff: out_j = g * rho * w_j / sqrt(sum_k w_k^2 + eps). */
void or_wn_forward_row(const double *w, int64_t C, double g, double rho,
                       double eps, unsigned flags, double *out);

/* Exact derivative of or_wn_forward_row for L = sum_j gy_j * out_j:
 *   D = sum w_j gy_j, n = sqrt(S + eps),
 *   grad_g   = rho * D / n,
 *   grad_w_j = (g rho / n) * (gy_j - w_j * D / (S + eps)).
 * At eps = 0 this is [DS] eq. dL/dW. */
void or_wn_backward_row(const double *w, const double *gy, int64_t C, double g,
                        double rho, double eps, unsigned flags, double *grad_w,
                        double *grad_g);

/* [DS] "Optimizer" (method "rescale"), before the step: the gradient's
 * component along the row removed, out_j = G_j - w_j * (w . G) / (S + eps). */
void or_grad_project_row(const double *w, const double *G, int64_t C,
                         double eps, unsigned flags, double *out);

/* [DS] "Optimizer", after the step: the same component removed from the
 * momentum m, and the row rescaled back to its radius:
 *   m_out_j = m_j - w_j (w . m) / (S + eps),  w_out_j = rho w_j / sqrt(S + eps). */
void or_renorm_momentum_row(const double *w, const double *m, int64_t C,
                            double rho, double eps, unsigned flags,
                            double *w_out, double *m_out);

/* [DS] "Optimizer": rescale the row back to its radius, out_j = rho w_j / n. */
void or_row_renorm_row(const double *w, int64_t C, double rho, double eps,
                       unsigned flags, double *out);

/* Backward of the activation rows (derived; the pages give the forward
 * only).  Gradients pass straight through the bf16 rounding points, which
 * keep their rounded values (s, a, b) as in the forward.
 *   l2:    dx_j = (dy_j - s_j (s . dy) / (S + eps)) / sqrt(S + eps);  s_tmp C doubles.
 *   slerp: dt = (dh - t (t . dh)/nt^2)/nt, da = (1-|alpha|) dt, db = |alpha| dt,
 *          dres = (da - res (res . da)/na^2)/na, dout likewise,
 *          dalpha_row_j = sign(alpha_j) (b_j - a_j) dt_j (may be NULL);
 *          tmp 4*C doubles. */
void or_l2_backward_row(const double *x, const double *r, const double *dy,
                        int64_t C, double eps, unsigned flags, double *s_tmp,
                        double *dx);
void or_slerp_backward_row(const double *res, const double *out,
                           const double *alpha, const double *dh, int64_t C,
                           double eps, unsigned flags, double *tmp,
                           double *dres, double *dout, double *dalpha_row);

/* [TF] tf_l2_rows: s = x or bf16(x + r); y = bf16(s / sqrt(sum s^2 + eps)).
 * r may be NULL.  s_tmp holds C doubles.  y_exact (may be NULL) receives the
 * value before the final rounding. */
void or_l2_row(const double *x, const double *r, int64_t C, double eps,
               unsigned flags, double *s_tmp, uint16_t *y, double *y_exact);

/* [TF] tf_slerp_rows: a = bf16(l2(res)), b = bf16(l2(out)),
 * t_j = a_j + |alpha_j| (b_j - a_j), h = bf16(t / sqrt(sum t^2 + eps)).
 * tmp holds 3*C doubles.  h_exact may be NULL. */
void or_slerp_row(const double *res, const double *out, const double *alpha,
                  int64_t C, double eps, unsigned flags, double *tmp,
                  uint16_t *h, double *h_exact);

/* ---- interval forms ----------------------------------------------------- *
 * [TF] checks each output against "float64's value at the bf16 rounding
 * points as a range over the fp32 run's spread".  These forms take the same
 * steps as the point forms but carry an interval: every fp32 evaluation of a
 * step may be off by a relative `delta`; at each bf16 rounding point both
 * roundings of the interval's ends are kept.  Output: the lowest and highest
 * bf16 results (bits) an fp32 evaluation within `delta` can produce.  The
 * slerp lerp is taken as fp32 steps: the difference b - a, then a + m(b - a)
 * rounded once (fused multiply-add).  With delta = 0 both equal the point
 * form.  tmp: l2 needs C doubles, slerp 3*C. */
void or_l2_row_interval(const double *x, const double *r, int64_t C,
                        double eps, double delta, unsigned flags, double *tmp,
                        uint16_t *lo, uint16_t *hi);
void or_slerp_row_interval(const double *res, const double *out,
                           const double *alpha, int64_t C, double eps,
                           double delta, unsigned flags, double *tmp,
                           uint16_t *lo, uint16_t *hi);

/* ---- matrices: row-major with leading dimension ld (elements) ----------- *
 * Outputs are dense [R, C].  nthreads <= 1 runs on the calling thread;
 * otherwise rows are split into nthreads contiguous ranges (each row is still
 * computed by one thread in the same order, so results do not depend on it).
 * Return 0 on success, -1 on a bad argument or allocation failure. */

/* g may be NULL (mode "unit": g = 1). */
int or_wn_forward(const float *w, int64_t R, int64_t C, int64_t ld,
                  const float *g, double rho, double eps, unsigned flags,
                  double *out, int nthreads);

/* gy is float32 (gy_is_bf16 = 0) or bf16 bits (gy_is_bf16 = 1), leading
 * dimension ld_gy.  grad_g may be NULL. */
int or_wn_backward(const float *w, int64_t R, int64_t C, int64_t ld,
                   const void *gy, int gy_is_bf16, int64_t ld_gy,
                   const float *g, double rho, double eps, unsigned flags,
                   double *grad_w, double *grad_g, int nthreads);

int or_row_renorm(const float *w, int64_t R, int64_t C, int64_t ld, double rho,
                  double eps, unsigned flags, double *out, int nthreads);

/* G, m: float32 [R, C], leading dimension ld_g / ld_m.  flags: 0 or
 * OR_EPS_ZERO. */
int or_grad_project(const float *w, int64_t R, int64_t C, int64_t ld,
                    const float *G, int64_t ld_g, double eps, unsigned flags,
                    double *out, int nthreads);
int or_renorm_momentum(const float *w, int64_t R, int64_t C, int64_t ld,
                       const float *m, int64_t ld_m, double rho, double eps,
                       unsigned flags, double *w_out, double *m_out,
                       int nthreads);

/* x, r: bf16 bits; r may be NULL.  y_exact may be NULL. */
int or_l2_rows(const uint16_t *x, const uint16_t *r, int64_t R, int64_t C,
               int64_t ld, double eps, unsigned flags, uint16_t *y,
               double *y_exact, int nthreads);

int or_slerp_rows(const uint16_t *res, const uint16_t *out, const float *alpha,
                  int64_t R, int64_t C, int64_t ld, double eps, unsigned flags,
                  uint16_t *h, double *h_exact, int nthreads);

/* [TF] Dory's gated and SwiGLU rows, then their L2 norm (the norms.cu
 * family; sigmoid and silu in torch's fp32 forms 1/(1+exp(-x)), x/(1+exp(-x))):
 *   gate_l2:   y = bf16(l2(bf16(o * sigmoid(g * sg))))
 *   swiglu_l2: y = bf16(l2(bf16(silu(bf16(g * sug)) * bf16(u * suu))))
 * o, g, u bf16 bits [R, ld]; sg, sug, suu fp32 [C].  The interval forms give,
 * per output, the bf16 ends any fp32 evaluation within relative `delta` per
 * step (and 2 ulps in exp) can reach, with fp32's exp range (exp(-x)
 * overflows for -x > 88.72: the gate or silu is 0) and subnormal steps. */
int or_gate_l2_rows(const uint16_t *o, const uint16_t *g, const float *sg,
                    int64_t R, int64_t C, int64_t ld, double eps,
                    unsigned flags, uint16_t *y, double *y_exact, int nthreads);
int or_swiglu_l2_rows(const uint16_t *g, const uint16_t *u, const float *sug,
                      const float *suu, int64_t R, int64_t C, int64_t ld,
                      double eps, unsigned flags, uint16_t *y, double *y_exact,
                      int nthreads);
int or_gate_l2_rows_interval(const uint16_t *o, const uint16_t *g,
                             const float *sg, int64_t R, int64_t C, int64_t ld,
                             double eps, double delta, unsigned flags,
                             uint16_t *lo, uint16_t *hi, int nthreads);
int or_swiglu_l2_rows_interval(const uint16_t *g, const uint16_t *u,
                               const float *sug, const float *suu, int64_t R,
                               int64_t C, int64_t ld, double eps, double delta,
                               unsigned flags, uint16_t *lo, uint16_t *hi,
                               int nthreads);

/* [DS] "Monitor" (each layer's raw row lengths) and options table, `init`
 * "preserve" (gain = row length, same output): len[r] = sqrt(sum_j w^2 + eps)
 * / div for fp32 rows w [R, ld]; div = 1 for the lengths, div = rho for the
 * preserving gain (W_eff = g rho w / len = w).  f64 out [R]. */
int or_row_norms(const float *w, int64_t R, int64_t C, int64_t ld, double eps,
                 double div, double *out, int nthreads);

/* [DS] options table, `gain` "scalar" (one gain for the layer): W_eff =
 * g rho w_r / n_r for every row, so dL/dg = sum_r rho (w_r . GY_r) / n_r, the
 * per-row grad_g of the channel form summed over the rows in row order.
 * gg_rows [R] (those parts) and *gg_sum.  grad_w as or_wn_backward with
 * every g_r = g. */
int or_wn_backward_scalar_gain(const float *w, int64_t R, int64_t C,
                               int64_t ld, const void *gy, int gy_is_bf16,
                               int64_t ld_gy, float g, double rho, double eps,
                               unsigned flags, double *grad_w, double *gg_rows,
                               double *gg_sum, int nthreads);

/* [TF] tf_qk_rows_l2 (Dory's q and k rows, in dory.py's order): per row t and
 * head, with D = head_dim, h = D/2 and the fp32 angle th_i = fp32(p_t * inv_i),
 *   rot_i   = bf16(x_i cos th_i - x_{i+h} sin th_i)        (rotate-half RoPE,
 *   rot_i+h = bf16(x_i sin th_i + x_{i+h} cos th_i)         the rotated head)
 *   y = bf16(rot / sqrt(sum rot^2 + eps))                   (the normalized head)
 *   q: out = bf16(y * q_scale_j) (q_scale fp32 [hq*D], or NULL: out = y);
 *   k: out = y.
 * q bf16 bits [R, ld_q] (hq heads), k [R, ld_k] (hk heads), pos [R], inv fp32
 * [h].  Outputs dense: q_out [R, hq*D], k_out [R, hk*D]; the *_exact outputs
 * (may be NULL) hold each output before its last rounding.  The interval form
 * gives the bf16 ends reachable with cosf/sinf within 2 ulps of the fp32
 * angle's cosine and sine, the rotation's fp32 products and sum, and each
 * later fp32 step within relative `delta`. */
int or_qk_rows_l2(const uint16_t *q, int64_t ld_q, const uint16_t *k,
                  int64_t ld_k, int64_t R, int32_t D, int32_t hq, int32_t hk,
                  const int32_t *pos, const float *inv, const float *q_scale,
                  double eps, unsigned flags, uint16_t *q_out, uint16_t *k_out,
                  double *q_exact, double *k_exact, int nthreads);
int or_qk_rows_l2_interval(const uint16_t *q, int64_t ld_q, const uint16_t *k,
                           int64_t ld_k, int64_t R, int32_t D, int32_t hq,
                           int32_t hk, const int32_t *pos, const float *inv,
                           const float *q_scale, double eps, double delta,
                           unsigned flags, uint16_t *q_lo, uint16_t *q_hi,
                           uint16_t *k_lo, uint16_t *k_hi, int nthreads);

/* Backward of the activation rows over matrices (bf16 bits in, f64 out).
 * dalpha (may be NULL) = the rows' parts summed in row order. */
int or_l2_rows_backward(const uint16_t *x, const uint16_t *r,
                        const uint16_t *dy, int64_t R, int64_t C, int64_t ld,
                        double eps, unsigned flags, double *dx, int nthreads);
int or_slerp_rows_backward(const uint16_t *res, const uint16_t *out,
                           const float *alpha, const uint16_t *dh, int64_t R,
                           int64_t C, int64_t ld, double eps, unsigned flags,
                           double *dres, double *dout, double *dalpha,
                           int nthreads);

int or_l2_rows_interval(const uint16_t *x, const uint16_t *r, int64_t R,
                        int64_t C, int64_t ld, double eps, double delta,
                        unsigned flags, uint16_t *lo, uint16_t *hi,
                        int nthreads);
int or_slerp_rows_interval(const uint16_t *res, const uint16_t *out,
                           const float *alpha, int64_t R, int64_t C,
                           int64_t ld, double eps, double delta,
                           unsigned flags, uint16_t *lo, uint16_t *hi,
                           int nthreads);

#ifdef __cplusplus
}
#endif

#endif /* L2ROW_ORACLE_H */
