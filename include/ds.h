/*
 * ds.h -- C ABI of libds: per-row L2 normalisation of weight and activation
 * rows on NVIDIA B200 (sm_100a).
 *
 * Fourteen operations, each over a table of segments (matrices), so that
 * every weight of a model is handled by one call:
 *
 *   ds_wn_forward   W_eff[r,:] = g_r * rho * w[r,:] / sqrt(sum_j w[r,j]^2 + eps)
 *                   DragonScale package description, "What DragonScale
 *                   changes", eq. W_eff (unit rows times one gain per row,
 *                   radius rho: 1 for linears/convs, sqrt(dim) for embeddings).
 *   ds_wn_backward  the exact gradient of ds_wn_forward:
 *                   grad_g_r = rho * (w_r . GY_r) / n_r,
 *                   grad_w_r = (g_r rho / n_r) * (GY_r - w_r (w_r . GY_r) / n_r^2),
 *                   n_r = sqrt(sum w_r^2 + eps); same section, eq. dL/dW
 *                   (printed there at eps = 0: the gradient tangent to the row).
 *   ds_row_renorm   w[r,:] <- rho * w[r,:] / n_r in place; DragonScale,
 *                   "Optimizer" (method "rescale": after the step each row is
 *                   rescaled back to its radius).
 *   ds_grad_project G[r,:] <- G[r,:] - w[r,:] (w_r . G_r) / n_r^2 in place;
 *                   DragonScale, "Optimizer" (method "rescale": before each
 *                   step the part of each gradient that would change a row's
 *                   length is removed).
 *   ds_renorm_momentum  m[r,:] <- m[r,:] - w[r,:] (w_r . m_r) / n_r^2 and
 *                   w[r,:] <- rho * w[r,:] / n_r, both in place and both from
 *                   the row as the step left it; same section (after the step
 *                   the same part is removed from the momentum -- Adam's
 *                   exp_avg, SGD's or Muon's momentum_buffer -- and each row
 *                   is rescaled back to its radius).
 *   ds_row_norms, ds_gain_preserve  the row lengths sqrt(sum w^2 + eps) (over
 *                   rho for the preserving gain); DragonScale, "Monitor" and
 *                   the options table (`init` "preserve").
 *   ds_l2_rows      y = bf16(s / sqrt(sum s^2 + eps)), s = x or s = bf16(x + r);
 *                   TensorFold PR #1260, Conversation, the norms.cu commit
 *                   (tf_l2_rows: a loop's entry l2(state + input), or its exit).
 *   ds_slerp_rows   a = bf16(l2(x)), b = bf16(l2(r)),
 *                   t_j = a_j + |alpha_j| (b_j - a_j)  (fp32, one rounding),
 *                   y = bf16(t / sqrt(sum t^2 + eps)); same commit (tf_slerp_rows,
 *                   the normalised-lerp residual).
 *   ds_gate_l2_rows  y = bf16(l2(bf16(o * sigmoid(g * sg))))  and
 *   ds_swiglu_l2_rows  y = bf16(l2(bf16(silu(bf16(g * sug)) * bf16(u * suu)))):
 *                   Dory's output gate and SwiGLU MLP rows, then the norm over
 *                   the whole row; same PR (tf_gate_l2_rows, tf_swiglu_l2_rows),
 *                   sigmoid and silu in fp32 as 1/(1+expf(-x)) and
 *                   x/(1+expf(-x)) with IEEE division.
 *   ds_qk_rows_l2   Dory's attention rows, in dory.py's order: rotate-half
 *                   RoPE on each bf16 head of q and k at the fp32 angle
 *                   th_i = fp32(pos) * inv_i,
 *                     r_i   = bf16(x_i cos th_i - x_{i+D/2} sin th_i),
 *                     r_i+D/2 = bf16(x_i sin th_i + x_{i+D/2} cos th_i),
 *                   then y = bf16(r / sqrt(sum r^2 + eps)) per head; q out =
 *                   bf16(y * q_scale) (q_scale fp32, (sqk f)^2 as torch forms
 *                   it), k out = y into its cache row, v copied as is into its
 *                   cache row; same PR (tf_qk_rows_l2).  cos and sin are
 *                   CUDA's cosf / sinf of the fp32 angle, the products and sums
 *                   fp32 as the tern-tc listing's apply_rope computes them.
 *   ds_l2_rows_backward, ds_slerp_rows_backward  the gradients of the two
 *                   activation calls (derived: the pages give the forward only),
 *                   straight through the bf16 rounding points, which keep the
 *                   rounded values the forward uses:
 *                   l2:    dx = (dy - s (s . dy) / n^2) / n   (= dr with a residual)
 *                   slerp: dt = (dh - t (t . dh)/nt^2)/nt, da = (1-|alpha|) dt,
 *                          db = |alpha| dt, dres = (da - res (res . da)/na^2)/na,
 *                          dout likewise, dalpha_j = sum over rows of
 *                          sign(alpha_j) (b_j - a_j) dt_j.
 *
 * Numerics: every row reduction accumulates in fp32 in an order fixed by the
 * row length and the operation alone, so a row's bits never depend on the
 * row count, the segment table or the launch.  bf16 results are rounded to
 * nearest even.  Rows whose fp32 sum of squares overflows (or, at eps = 0,
 * falls below 2^-100) are recomputed with an exact power-of-two rescaling.
 *
 * Memory: all pointers are DEVICE pointers owned by the caller (the segment
 * tables themselves are HOST memory, read only during the call).  The library
 * allocates nothing, keeps no per-call state and may be called from several
 * host threads.  Matrices are row-major with leading dimension ld (elements)
 * >= cols; every row start must be 16-byte aligned (base pointer 16-byte
 * aligned, ld * element size a multiple of 16), and each buffer must be
 * readable up to the 16-byte boundary that follows its last element (any
 * cudaMalloc or PyTorch allocation is).  Elements past cols in a row are never
 * written.
 *
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 * default stream) and never synchronise, except ds_get_device_status.
 * Arguments are validated on the host before anything is launched; a failed
 * call launches nothing.  Kernels never trap: a bounded device-side wait that
 * runs out records DS_ERR_DEVICE_TIMEOUT, and ds_qk_rows_l2 records
 * DS_ERR_INVALID_ARG for a cache slot out of range (device data the host does
 * not read); ds_get_device_status returns and clears the first such record.
 */
#ifndef DS_H
#define DS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DS_OK = 0,
    DS_ERR_INVALID_ARG = 1,       /* NULL pointer, bad shape, bad eps, bad dtype value */
    DS_ERR_ALIGNMENT = 2,         /* a row start not 16-byte aligned                    */
    DS_ERR_UNSUPPORTED_DTYPE = 3, /* dtype not allowed for this call                    */
    DS_ERR_TOO_MANY_SEGMENTS = 4, /* nseg above DS_MAX_SEGMENTS                         */
    DS_ERR_CUDA = 5,              /* a CUDA runtime call failed (see ds_last_error)     */
    DS_ERR_DEVICE_TIMEOUT = 6,    /* a bounded device-side wait ran out                 */
    DS_ERR_OVERLAP = 7            /* an output overlaps an input or another output      */
} ds_status;

typedef enum { DS_F32 = 0, DS_BF16 = 1 } ds_dtype;

typedef void *ds_stream; /* cudaStream_t */

#define DS_MAX_SEGMENTS 65536

/* One weight matrix (Linear, Embedding, or a Conv flattened to [out, in*k...]).
 * Which fields a call reads:
 *   forward:  w, gain, w_eff (written), rows, cols, ld, ld_out, radius
 *   backward: w, gain, gy, grad_w (written), grad_g (written if gain != NULL),
 *             rows, cols, ld, ld_out, radius
 *   renorm:   w (read and written in place), rows, cols, ld, radius
 *   grad_project:    w (read), grad_w = the gradient G (read and written in
 *                    place), rows, cols, ld
 *   renorm_momentum: w (read and written in place), grad_w = the momentum
 *                    buffer m (read and written in place), rows, cols, ld,
 *                    radius
 *   row_norms, gain_preserve: w (read), rnorm (written), rows, cols, ld,
 *                    radius (gain_preserve)
 * (gain, w_eff, gy, grad_g and ld_out are ignored by the projections and
 * renorm; rnorm by every call but the last two.)
 *
 * gain_scalar (DragonScale options table, `gain` "scalar": one gain for the
 * layer): gain points to ONE float used by every row, and the backward's
 * grad_g holds rows + 1 floats: grad_g[r] = rho (w_r . GY_r) / n_r for each
 * row, then grad_g[rows] = their sum (dL/dg), summed in a fixed order so
 * that it is the same on every run. */
typedef struct {
    float *w;          /* fp32 [rows, ld] master rows                                */
    const float *gain; /* fp32 [rows] ([1] with gain_scalar), or NULL: mode "unit"   */
    void *w_eff;       /* forward output [rows, ld_out], dtype per call               */
    const void *gy;    /* backward input dL/dW_eff [rows, ld_out], dtype per call     */
    float *grad_w;     /* backward output fp32 [rows, ld], overwritten                */
    float *grad_g;     /* backward output fp32 [rows] ([rows + 1] with gain_scalar)   */
    int64_t rows;      /* >= 0                                                        */
    int64_t cols;      /* >= 1, <= 2^31 - 1                                           */
    int64_t ld;        /* leading dimension of w and grad_w, >= cols                  */
    int64_t ld_out;    /* leading dimension of w_eff and gy, >= cols                  */
    float radius;      /* rho: 1 for linears and convs, sqrt(cols) for embeddings     */
    int32_t gain_scalar; /* 0: one gain per row; 1: one gain for the matrix          */
    float *rnorm;      /* row_norms / gain_preserve output fp32 [rows]                */
    int32_t transposed; /* 1: the rows are the COLUMNS of w, w_eff, gy and grad_w,
                          stored [cols, ld] (element j of row r at [j * ld + r],
                          ld >= rows): GPT-2's Conv1D [in, out] weights.  Forward,
                          backward, renorm and the projections; not row_norms. */
    int32_t tgroup;     /* with transposed = 1: G >= 1 consecutive stored columns
                          per row (0 reads as 1), for ConvTranspose weights
                          [in, out, k...] stored [in, out * G] with G the kernel's
                          volume: row r holds the stored columns [r G, r G + G) of
                          every stored row, element (j, m) at [j * ld + r G + m],
                          so cols = in * G (a multiple of G), ld and ld_out >=
                          rows * G.  1 <= G <= 256.  Must be 0 or 1 when
                          transposed = 0.  (Grouped ConvTranspose: one segment per
                          group.)  DragonScale package description, "Supported
                          layers": ConvTranspose1d/2d/3d. */
} ds_wseg;

/* One activation matrix; x, r and y share the leading dimension ld.
 *   l2_rows:    x bf16 (required), r bf16 residual or NULL, y bf16 output
 *               (y may be exactly x or exactly r; partial overlap is refused)
 *   slerp_rows: x = res (required), r = out (required), alpha fp32 [cols]
 *               (|alpha_j| is the lerp weight), y = output (may alias x or r) */
typedef struct {
    const void *x;
    const void *r;
    void *y;
    const float *alpha;
    int64_t rows; /* >= 0 */
    int64_t cols; /* >= 1, <= 2^31 - 1 */
    int64_t ld;   /* >= cols */
} ds_aseg;

/* One activation matrix for the Dory rows: a, b and y bf16 [rows, ld]
 * (y may be exactly a or b), scale vectors fp32 [cols].
 *   gate_l2_rows:   a = o, b = g, sa = sg (sb ignored)
 *   swiglu_l2_rows: a = g (gate), b = u (up), sa = sug, sb = suu */
typedef struct {
    const void *a;
    const void *b;
    void *y;
    const float *sa;
    const float *sb;
    int64_t rows; /* >= 0 */
    int64_t cols; /* >= 1 */
    int64_t ld;   /* >= cols */
} ds_fseg;

/* One activation matrix for the backward calls.  x, r and dy share the
 * leading dimension ld; dx and dr share ld_d.
 *   l2_rows_backward:    x bf16, r bf16 residual or NULL, dy bf16 = dL/dy,
 *                        dx fp32 = dL/dx (also dL/dr when r is set); dr ignored
 *   slerp_rows_backward: x = res, r = out (both bf16, required), dy = dL/dh
 *                        bf16, alpha fp32 [cols], dx = dL/dres and dr = dL/dout
 *                        (fp32).  Outputs never overlap inputs. */
typedef struct {
    const void *x;
    const void *r;
    const void *dy;
    float *dx;
    float *dr;
    const float *alpha;
    int64_t rows; /* >= 0 */
    int64_t cols; /* >= 1 */
    int64_t ld;   /* >= cols, of x, r and dy */
    int64_t ld_d; /* >= cols, of dx and dr  */
} ds_agseg;

/* out_dtype: DS_BF16 or DS_F32 for every segment's w_eff. */
ds_status ds_wn_forward(const ds_wseg *segs, int nseg, ds_dtype out_dtype,
                        float eps, ds_stream stream);

/* gy_dtype: DS_BF16 or DS_F32 for every segment's gy.  w, gy and gain are
 * read-only; grad_w and grad_g must not overlap any input. */
ds_status ds_wn_backward(const ds_wseg *segs, int nseg, ds_dtype gy_dtype,
                         float eps, ds_stream stream);

ds_status ds_row_renorm(const ds_wseg *segs, int nseg, float eps,
                        ds_stream stream);

/* grad_w holds the fp32 gradient G [rows, ld]; it is overwritten with its
 * component orthogonal to the row (at eps = 0 exactly; with eps the removed
 * part is scaled by S/(S+eps), S = sum w^2).  w is read-only and must not
 * overlap G. */
ds_status ds_grad_project(const ds_wseg *segs, int nseg, float eps,
                          ds_stream stream);

/* grad_w holds the fp32 momentum m [rows, ld].  One pass per row: S = sum w^2
 * and D = w . m from the row as the optimizer step left it, then
 * m <- m - w D/(S+eps) and w <- rho w/sqrt(S+eps).  w and m must not overlap. */
ds_status ds_renorm_momentum(const ds_wseg *segs, int nseg, float eps,
                             ds_stream stream);

/* rnorm[r] = sqrt(sum_j w[r,j]^2 + eps): DragonScale, "Monitor" (each
 * layer's raw row lengths; eps = 0 gives the plain length).  w is read
 * only; rnorm must not overlap it. */
ds_status ds_row_norms(const ds_wseg *segs, int nseg, float eps,
                       ds_stream stream);

/* rnorm[r] = sqrt(sum_j w[r,j]^2 + eps) / radius: the gain of DragonScale's
 * `init` "preserve" (options table: gain = row length, same output), so that
 * ds_wn_forward with gain = rnorm returns w.  Point rnorm at the gain. */
ds_status ds_gain_preserve(const ds_wseg *segs, int nseg, float eps,
                           ds_stream stream);

ds_status ds_l2_rows(const ds_aseg *segs, int nseg, float eps,
                     ds_stream stream);

ds_status ds_slerp_rows(const ds_aseg *segs, int nseg, float eps,
                        ds_stream stream);

/* a and b are staged in shared memory (32 bytes per 8 columns): rows up to
 * 16,384 columns on one CTA, longer ones split over a cluster of 2, 4 or 8
 * CTAs (a slice of at most 64 KB each), so at most 131,072 columns; longer
 * rows are refused with DS_ERR_INVALID_ARG.  Dory's widths are 4,096 and
 * 7,168. */
ds_status ds_gate_l2_rows(const ds_fseg *segs, int nseg, float eps,
                          ds_stream stream);
ds_status ds_swiglu_l2_rows(const ds_fseg *segs, int nseg, float eps,
                            ds_stream stream);

/* One set of attention rows for ds_qk_rows_l2 (bf16 unless noted; every
 * matrix row-major, rows 16-byte aligned).
 *   q        [rows, hq*head_dim], leading dimension ld_q (hq may be 0)
 *   k        [rows, hk*head_dim], ld_kv (hk may be 0; hq + hk >= 1)
 *   v        [rows, hk*head_dim], ld_kv, or NULL (nothing copied)
 *   q_out    [rows, hq*head_dim], ld_q; may be exactly q
 *   k_cache  [cache_rows, hk*head_dim], ld_cache: row slot[t] (or t when slot
 *            is NULL) receives row t's normalized k heads; may be exactly k
 *            when slot is NULL and ld_cache == ld_kv
 *   v_cache  like k_cache for v (required iff v is set; may be exactly v on
 *            the same terms)
 *   pos      int32 [rows] device positions (any int32; the angle uses
 *            fp32(pos))
 *   slot     int32 [rows] device cache rows, or NULL.  Slots must be distinct;
 *            a slot outside [0, cache_rows) skips that row's k and v stores
 *            and records DS_ERR_INVALID_ARG for ds_get_device_status.
 *   inv_freq fp32 [head_dim/2] device (1/theta^(2i/D) as the caller forms it)
 *   q_scale  fp32 [hq*head_dim] device, 16-byte aligned, or NULL (scale 1)
 * head_dim is 16, 32, 64, 128, 256 or 512.  Buffers written by the call must
 * not overlap anything else it touches, except the exact aliases above. */
typedef struct {
    const void *q;
    const void *k;
    const void *v;
    void *q_out;
    void *k_cache;
    void *v_cache;
    const int32_t *pos;
    const int32_t *slot;
    const float *inv_freq;
    const float *q_scale;
    int64_t rows;       /* >= 0 */
    int64_t cache_rows; /* rows of k_cache / v_cache (>= rows when slot is NULL) */
    int64_t ld_q;
    int64_t ld_kv;
    int64_t ld_cache;
    int32_t head_dim;
    int32_t hq;
    int32_t hk;
} ds_qkseg;

ds_status ds_qk_rows_l2(const ds_qkseg *segs, int nseg, float eps,
                        ds_stream stream);

/* x, r and dy are staged in shared memory (48 bytes per 8 columns; l2 rows
 * without a residual 32): rows up to 10,920 columns (16,384 without a
 * residual) on one CTA, longer ones split over a cluster of 2, 4 or 8 CTAs (a
 * slice of at most 64 KB each), so at most 87,296 columns for slerp and for
 * l2 with a residual, 131,072 for l2 without one; longer rows are refused
 * with DS_ERR_INVALID_ARG.  ds_row_class reports the l2 backward's class for
 * rows with a residual. */
ds_status ds_l2_rows_backward(const ds_agseg *segs, int nseg, float eps,
                              ds_stream stream);

/* dalpha: fp32 [cols] device output, or NULL to skip it.  With dalpha every
 * segment must use the same alpha and cols, and `workspace` must be device
 * memory of at least ds_slerp_rows_backward_workspace(cols) bytes, 256-byte
 * aligned, owned by the caller and not touched by anything else until the
 * call's work on `stream` ends (its contents on entry do not matter).  The
 * column sums are deterministic: per-team partial sums in a fixed row order,
 * then a second launch adds them in a fixed order. */
ds_status ds_slerp_rows_backward(const ds_agseg *segs, int nseg, float eps,
                                 float *dalpha, void *workspace,
                                 uint64_t workspace_bytes, ds_stream stream);

/* Workspace bytes ds_slerp_rows_backward needs for dalpha over rows of
 * `cols` elements on the current device (0 if cols < 1). */
uint64_t ds_slerp_rows_backward_workspace(int64_t cols);

/* ds_slerp_rows_backward for callers that cannot allocate device memory
 * where they run the backward: a runtime that hands all device memory to its
 * own pool at start-up and forbids later cudaMalloc calls, or code that must
 * not risk the implicit device-wide synchronisation cudaMalloc and cudaFree
 * may cause.  Such a caller cannot provide the workspace of
 * ds_slerp_rows_backward, so this entry point allocates nothing: dalpha's
 * per-team partial sums go to a static device array built into the library
 * (64 MB, held on every device that loads the library until the process
 * exits).  Inputs and outputs are still the caller's, as for
 * ds_slerp_rows_backward.
 *   - Limit: the partial sums of rows of cols columns take
 *     ds_slerp_rows_backward_workspace(cols) bytes; rows that need more than
 *     64 MB (more than 8,712 columns on a 148-SM B200) are refused with
 *     DS_ERR_INVALID_ARG and a message in ds_last_error.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (a host-side runtime query, with that device current) and
 *     caches it; make that first call before any stream capture.
 *   - Sharing: every call of this entry point, on any stream, uses the same
 *     array, so calls that overlap on the GPU race and give wrong dalpha; use
 *     one stream or synchronise between calls.  Nothing in the array needs to
 *     start at zero (each call overwrites every partial sum it reads), so a
 *     previous call's leftover contents do no harm.
 * Results are bitwise those of ds_slerp_rows_backward.  The pages have no
 * counterpart: this entry point is this library's own. */
ds_status ds_slerp_rows_backward_noalloc(const ds_agseg *segs, int nseg, float eps,
                                         float *dalpha, ds_stream stream);

/* Static description of a status code. */
const char *ds_status_string(ds_status status);

/* Detail of the last failed call on this host thread ("" if none). */
const char *ds_last_error(void);

/* Synchronises `stream`, then returns and clears the device error word of
 * the current device (DS_OK, or DS_ERR_DEVICE_TIMEOUT after a bounded wait
 * ran out), or DS_ERR_CUDA if the synchronisation itself failed. */
ds_status ds_get_device_status(ds_stream stream);

/* Number of kernels this library has launched in this process. */
uint64_t ds_launch_count(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int ds_version(void);

/* ---- planning introspection (host only, no GPU needed) ------------------ */

typedef enum {
    DS_OP_WN_FORWARD = 0,
    DS_OP_WN_BACKWARD = 1,
    DS_OP_ROW_RENORM = 2,
    DS_OP_L2_ROWS = 3,
    DS_OP_SLERP_ROWS = 4,
    DS_OP_GRAD_PROJECT = 5,
    DS_OP_RENORM_MOMENTUM = 6,
    DS_OP_L2_ROWS_BACKWARD = 7,
    DS_OP_SLERP_ROWS_BACKWARD = 8,
    DS_OP_GATE_L2_ROWS = 9,
    DS_OP_SWIGLU_L2_ROWS = 10
} ds_op;

typedef enum {
    DS_PATH_AUTO = 0,     /* chosen from the row length                       */
    DS_PATH_WARP = 1,     /* staged: rows of <= 16 KB of input in a ring of
                             shared-memory slots filled by bulk copies; one
                             warp (weights) or two (activations) per row      */
    DS_PATH_CTA = 2,      /* staged in 32, 64 or (weights) 112 KB slots: a
                             team of 2..8 warps per row (rows of <= 64 KB of
                             input; weights 112 KB)                           */
    DS_PATH_CLUSTER = 3,  /* staged, a cluster of 2, 4 or 8 CTAs per row:
                             each CTA stages a slice of <= 64 KB of every row
                             of its slots, partial sums meet through
                             distributed shared memory                        */
    DS_PATH_TWO_PASS = 4  /* a cluster streams the row twice through shared
                             memory with bulk (TMA) copies (rows longer than
                             eight slices; not the activation backward or the
                             Dory rows)                                       */
} ds_path;

/* The row class a call would use for rows of `cols` elements: path, threads
 * per row in each CTA (the staged paths' team; 0 on the two-pass path) and
 * CTAs per row (cluster / two-pass; 1 otherwise).
 * Depends on (op, cols) and the forced path only -- never on the row count. */
ds_status ds_row_class(ds_op op, int64_t cols, int *path, int *group_threads,
                       int *cluster_ctas);

/* ---- test knobs (process-wide; not for production use) ------------------ */

/* Force every call onto one path where the row fits it (DS_PATH_AUTO
 * restores automatic choice).  DS_PATH_TWO_PASS fits every row. */
ds_status ds_debug_force_path(ds_path path);

/* Bound, in nanoseconds, of every device-side wait (default 2e9). */
ds_status ds_debug_set_wait_limit_ns(uint64_t limit_ns);

/* Launches one CTA that waits on a shared-memory barrier nothing will ever
 * complete, bounded by limit_ns, so that the timeout path runs: afterwards
 * ds_get_device_status returns DS_ERR_DEVICE_TIMEOUT.  No copy is in flight. */
ds_status ds_debug_wait_timeout_selftest(uint64_t limit_ns, ds_stream stream);

/* Checks, over every fp32 bit pattern v, the reciprocal and quotient the Dory
 * rows compute where their fast range applies (gate: 1/(1 + expf(-v));
 * silu: v/(1 + expf(-v))) against IEEE division (__frcp_rn, __fdiv_rn),
 * bit for bit.  counts: DEVICE array of 4 uint64, overwritten with
 * {reciprocal mismatches, quotient mismatches, inputs checked for the
 * reciprocal, inputs checked for the quotient}.  Asynchronous on `stream`.
 * The pages have no counterpart: it tests this library's arithmetic. */
ds_status ds_debug_division_check(uint64_t *counts, ds_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* DS_H */
