// ds_kernels.cu -- sm_100a kernels for rows too long for the staged path
// (ds_tile.cu takes every row whose slices fit 8 CTAs' shared memory), and
// the small kernels around the row calls (row lengths, scalar-gain sums, the
// bounded-wait self-test).
//
//   * stream  : a cluster of 8 CTAs per row, each streaming its slice
//               through a kStages-deep shared-memory ring filled by bulk
//               (TMA) copies, once per pass (most re-reads hit L2).  Rows of
//               any length; partial sums meet through distributed shared
//               memory.
// Operations (sources cited in include/ds.h):
//   wn_forward, wn_backward, row_renorm : DragonScale unit rows with gains
//   grad_project, renorm_momentum       : DragonScale "Optimizer" (rescale)
//   l2_rows, slerp_rows                 : TensorFold tf_l2_rows, tf_slerp_rows
#include <algorithm>
#include <cuda_runtime.h>

#include "ds_device.cuh"

namespace ds {

namespace {

// ------------------------------------------------------------- unit I/O --

__device__ __forceinline__ float4 quad_f32(const float *row, int u, int cols)
{
    float4 v = as_f4(ld16(row + 4 * u));
    const int valid = cols - 4 * u;
    return valid < 4 ? mask_quad(v, valid) : v;
}

__device__ __forceinline__ float4 quad_bf16(const uint16_t *row, int u, int cols)
{
    const uint2 r = ld8(row + 4 * u);
    float4 v = make_float4(bf_lo(r.x), bf_hi(r.x), bf_lo(r.y), bf_hi(r.y));
    const int valid = cols - 4 * u;
    return valid < 4 ? mask_quad(v, valid) : v;
}

template <bool BF16>
__device__ __forceinline__ float4 quad_gy(const void *row, int u, int cols)
{
    if constexpr (BF16)
        return quad_bf16(static_cast<const uint16_t *>(row), u, cols);
    else
        return quad_f32(static_cast<const float *>(row), u, cols);
}

__device__ __forceinline__ uint4 octet(const uint16_t *row, int u, int cols)
{
    uint4 v = ld16(row + 8 * u);
    const int valid = cols - 8 * u;
    return valid < 8 ? mask_octet(v, valid) : v;
}

__device__ __forceinline__ uint16_t bf_bits(float v)
{
    __nv_bfloat16 h = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&h);
}

// Store a quad of fp32 results as fp32 or bf16; only elements < cols.
template <bool BF16>
__device__ __forceinline__ void store_quad(void *row, int u, int cols, float4 y)
{
    const int valid = cols - 4 * u;
    if constexpr (BF16) {
        uint16_t *o = static_cast<uint16_t *>(row) + 4 * u;
        if (valid >= 4) {
            st8(o, make_uint2(pack_bf2(y.x, y.y), pack_bf2(y.z, y.w)));
        } else {
            o[0] = bf_bits(y.x);
            if (valid > 1) o[1] = bf_bits(y.y);
            if (valid > 2) o[2] = bf_bits(y.z);
        }
    } else {
        float *o = static_cast<float *>(row) + 4 * u;
        if (valid >= 4) {
            st16(o, as_u4(y));
        } else {
            o[0] = y.x;
            if (valid > 1) o[1] = y.y;
            if (valid > 2) o[2] = y.z;
        }
    }
}

__device__ __forceinline__ void store_octet(uint16_t *row, int u, int cols, uint4 v)
{
    const int valid = cols - 8 * u;
    uint16_t *o = row + 8 * u;
    if (valid >= 8) {
        st16(o, v);
    } else {
        for (int e = 0; e < valid; ++e) {
            const uint32_t w = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
            o[e] = static_cast<uint16_t>((e & 1) ? (w >> 16) : (w & 0xFFFFu));
        }
    }
}

__device__ __forceinline__ float4 scale4(float4 v, float pre, float s)
{
    return make_float4((v.x * pre) * s, (v.y * pre) * s, (v.z * pre) * s, (v.w * pre) * s);
}

__device__ __forceinline__ void acc_sq4(float &acc, float4 v)
{
    acc = fmaf(v.x, v.x, acc);
    acc = fmaf(v.y, v.y, acc);
    acc = fmaf(v.z, v.z, acc);
    acc = fmaf(v.w, v.w, acc);
}

__device__ __forceinline__ void acc_dot4(float &acc, float4 a, float4 b)
{
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
    acc = fmaf(a.z, b.z, acc);
    acc = fmaf(a.w, b.w, acc);
}

__device__ __forceinline__ void acc_sq8(float &acc, uint4 v)
{
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float x = bf_get(v, e);
        acc = fmaf(x, x, acc);
    }
}

template <class F>
__device__ __forceinline__ void each4(float4 v, F &&f)
{
    f(v.x);
    f(v.y);
    f(v.z);
    f(v.w);
}

template <class F>
__device__ __forceinline__ void each8(uint4 v, F &&f)
{
#pragma unroll
    for (int e = 0; e < 8; ++e)
        f(bf_get(v, e));
}

// Sum of two bf16 octets, each sum rounded once to bf16 (round to nearest
// even).  The fp32 sum of two bf16 values is exact unless their exponents
// differ by more than 15, and then the smaller is below 2^-15 of the larger,
// far from any bf16 halfway point: one rounding of the fp32 sum equals the
// rounding of the exact sum.
__device__ __forceinline__ uint4 add_bf16x8(uint4 a, uint4 b)
{
    uint4 s;
    s.x = pack_bf2(bf_lo(a.x) + bf_lo(b.x), bf_hi(a.x) + bf_hi(b.x));
    s.y = pack_bf2(bf_lo(a.y) + bf_lo(b.y), bf_hi(a.y) + bf_hi(b.y));
    s.z = pack_bf2(bf_lo(a.z) + bf_lo(b.z), bf_hi(a.z) + bf_hi(b.z));
    s.w = pack_bf2(bf_lo(a.w) + bf_lo(b.w), bf_hi(a.w) + bf_hi(b.w));
    return s;
}

// bf16(v * pre * s) for the 8 entries (see RowScale for `pre`).
__device__ __forceinline__ uint4 scale_bf16x8(uint4 v, RowScale r)
{
    const float p = r.pre, s = r.inv;
    uint4 o;
    o.x = pack_bf2((bf_lo(v.x) * p) * s, (bf_hi(v.x) * p) * s);
    o.y = pack_bf2((bf_lo(v.y) * p) * s, (bf_hi(v.y) * p) * s);
    o.z = pack_bf2((bf_lo(v.z) * p) * s, (bf_hi(v.z) * p) * s);
    o.w = pack_bf2((bf_lo(v.w) * p) * s, (bf_hi(v.w) * p) * s);
    return o;
}

// |alpha| for the 8 elements of unit u, 0 past cols.  The float4 holding the
// last valid element may extend past cols (it never leaves that 16-byte
// block, so the read stays inside the allocation); whatever it holds there
// is dropped, so a NaN beyond the vector cannot reach the row's sums.
__device__ __forceinline__ void alpha8(const float *alpha, int u, int cols, float (&m)[8])
{
    const int e0 = 8 * u;
    const float4 a = e0 < cols ? ld16_cached(alpha + e0) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 b = e0 + 4 < cols ? ld16_cached(alpha + e0 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    m[0] = fabsf(a.x);
    m[1] = fabsf(a.y);
    m[2] = fabsf(a.z);
    m[3] = fabsf(a.w);
    m[4] = fabsf(b.x);
    m[5] = fabsf(b.y);
    m[6] = fabsf(b.z);
    m[7] = fabsf(b.w);
    if (e0 + 8 > cols) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m[i] = e0 + i < cols ? m[i] : 0.f;
    }
}

// The lerp t = a + |alpha| (b - a): the difference, then one fused rounding
// (exact at |alpha| = 0; at |alpha| = 1 the definition gives b, taken as is,
// since b - a itself may round when a and b are far apart in magnitude).
__device__ __forceinline__ float lerp_t(float a, float b, float m) { return m == 1.f ? b : fmaf(m, b - a, a); }

// Epilogues of the two-reduction row (S = sum w^2, D = w . d):
//   kModeGrad      ds_wn_backward: grad_w = (g rho / n)(d - w D/n^2), grad_g = rho D / n
//   kModeProject   ds_grad_project: d <- d - w D/n^2 (d = the gradient, in place)
//   kModeMomentum  ds_renorm_momentum: d <- d - w D/n^2 (d = the momentum) and
//                  w <- rho w / n, both in place
// With the power-of-two rescale (factor 2^m on w) the projection uses the
// scaled row and the scaled quotient, xs * (Ds / n2s) = w * D / n^2, which
// stays finite where the unscaled quotient D / n^2 would overflow.
enum BwdMode { kModeGrad = 0, kModeProject = 1, kModeMomentum = 2 };

// ================================================================ kernels ==

// Operation tags: one kernel template per shape, dispatching on the tag.
enum OpTag { kFwdBf16, kFwdF32, kBwdBf16, kBwdF32, kRenorm, kL2, kSlerp, kProject, kMomentum };

template <int T>
struct IsWeight {
    static constexpr bool value = T <= kRenorm || T >= kProject;
};

template <int T>
struct OpOf {
    static constexpr ds_op value = (T == kFwdBf16 || T == kFwdF32) ? DS_OP_WN_FORWARD
                                 : (T == kBwdBf16 || T == kBwdF32) ? DS_OP_WN_BACKWARD
                                 : T == kRenorm ? DS_OP_ROW_RENORM
                                 : T == kProject ? DS_OP_GRAD_PROJECT
                                 : T == kMomentum ? DS_OP_RENORM_MOMENTUM
                                 : T == kL2 ? DS_OP_L2_ROWS : DS_OP_SLERP_ROWS;
};

template <int T>
using ParamsOf = typename std::conditional<IsWeight<T>::value, WParams, AParams>::type;

// ======================================================= streaming rows ====
//
// Each operation describes the arrays it streams (unit bytes), its passes,
// what a pass does with one unit, and the reduction between passes.  The
// kernel owns the ring: stage s holds chunk i (i = pass * nch + chunk) when
// i % kStages == s; thread 0 refills a stage as soon as all threads are done
// with it, so the next pass's loads (mostly L2 hits) overlap the reduction.

struct StreamCtx {
    int ubeg, len, cols, nu;
};

template <bool OUT_BF16, bool RENORM>
struct SScale {
    static constexpr int kPasses = 2;
    static constexpr int kArrays = 1;
    const WSegK &sg;
    int64_t row;
    float eps;
    float acc = 0.f, sc = 0.f, pre = 1.f;

    __device__ SScale(const WSegK &s, int64_t r, float e) : sg(s), row(r), eps(e) {}
    __device__ int unit_bytes(int) const { return 16; }
    __device__ const char *src(int) const { return reinterpret_cast<const char *>(sg.w + row * sg.ld); }

    __device__ __forceinline__ void consume(int pass, const unsigned char *const *st, int j, int u,
                                            const StreamCtx &c, bool store)
    {
        float4 v = *reinterpret_cast<const float4 *>(st[0] + 16 * j);
        if (c.cols - 4 * u < 4)
            v = mask_quad(v, c.cols - 4 * u);
        if (pass == 0) {
            acc_sq4(acc, v);
        } else if (store) {
            void *out = RENORM ? static_cast<void *>(const_cast<float *>(sg.w) + row * sg.ld)
                               : static_cast<void *>(static_cast<char *>(sg.out) +
                                                     row * sg.ld_out * (OUT_BF16 ? 2 : 4));
            store_quad<OUT_BF16>(out, u, c.cols, scale4(v, pre, sc));
        }
    }

    template <class Red>
    __device__ __forceinline__ void between(int, Red &red, const StreamCtx &c)
    {
        float a[1] = {acc};
        red.sum(a);
        const float *w = sg.w + row * sg.ld;
        const RowScale rs = row_scale(a[0], eps, red, [&](auto f) {
            for (int ul = threadIdx.x; ul < c.len; ul += kCta)
                each4(quad_f32(w, c.ubeg + ul, c.cols), f);
        });
        const float g = (!RENORM && sg.gain) ? __ldg(sg.gain + row * sg.gain_stride) : 1.f;
        sc = (g * sg.radius) * rs.inv;
        pre = rs.pre;
    }
    __device__ void finish(bool, bool) {}
};

template <bool GY_BF16, int MODE>
struct SBackward {
    static constexpr int kPasses = 2;
    static constexpr int kArrays = 2;
    const WSegK &sg;
    int64_t row;
    float eps;
    float acc[2] = {0.f, 0.f};
    float pre = 0.f, q = 0.f, gg = 0.f, sc = 0.f;
    int msh = 0; // power-of-two rescale of w (projection modes)

    __device__ SBackward(const WSegK &s, int64_t r, float e) : sg(s), row(r), eps(e) {}
    __device__ int unit_bytes(int a) const { return a == 0 ? 16 : (GY_BF16 ? 8 : 16); }
    __device__ const char *src(int a) const
    {
        return a == 0 ? reinterpret_cast<const char *>(sg.w + row * sg.ld)
                      : static_cast<const char *>(sg.gy) + row * sg.ld_out * (GY_BF16 ? 2 : 4);
    }

    __device__ __forceinline__ void consume(int pass, const unsigned char *const *st, int j, int u,
                                            const StreamCtx &c, bool store)
    {
        float4 x = *reinterpret_cast<const float4 *>(st[0] + 16 * j);
        float4 d;
        if constexpr (GY_BF16) {
            const uint2 r = *reinterpret_cast<const uint2 *>(st[1] + 8 * j);
            d = make_float4(bf_lo(r.x), bf_hi(r.x), bf_lo(r.y), bf_hi(r.y));
        } else {
            d = *reinterpret_cast<const float4 *>(st[1] + 16 * j);
        }
        const int valid = c.cols - 4 * u;
        if (valid < 4) {
            x = mask_quad(x, valid);
            d = mask_quad(d, valid);
        }
        if (pass == 0) {
            acc_sq4(acc[0], x);
            acc_dot4(acc[1], x, d);
        } else if (store) {
            if constexpr (MODE == kModeGrad) {
                float4 y;
                y.x = pre * fmaf(-x.x, q, d.x);
                y.y = pre * fmaf(-x.y, q, d.y);
                y.z = pre * fmaf(-x.z, q, d.z);
                y.w = pre * fmaf(-x.w, q, d.w);
                store_quad<false>(sg.grad_w + row * sg.ld, u, c.cols, y);
            } else {
                if (msh != 0)
                    x = make_float4(scalbnf(x.x, msh), scalbnf(x.y, msh), scalbnf(x.z, msh), scalbnf(x.w, msh));
                float4 y;
                y.x = fmaf(-x.x, q, d.x);
                y.y = fmaf(-x.y, q, d.y);
                y.z = fmaf(-x.z, q, d.z);
                y.w = fmaf(-x.w, q, d.w);
                store_quad<false>(sg.grad_w + row * sg.ld, u, c.cols, y);
                if constexpr (MODE == kModeMomentum)
                    store_quad<false>(static_cast<float *>(sg.out) + row * sg.ld, u, c.cols,
                                      make_float4(x.x * sc, x.y * sc, x.z * sc, x.w * sc));
            }
        }
    }

    template <class Red>
    __device__ __forceinline__ void between(int, Red &red, const StreamCtx &c)
    {
        red.sum(acc);
        const float *w = sg.w + row * sg.ld;
        const void *gy = src(1);
        int m = 0;
        const bool need = needs_rescale(acc[0], eps);
        if (red.any(need)) {
            float M = 0.f;
            for (int ul = threadIdx.x; ul < c.len; ul += kCta)
                each4(quad_f32(w, c.ubeg + ul, c.cols), [&](float v) { M = fmaxf(M, fabsf(v)); });
            M = red.max(M);
            if (need && M > 0.f && M < __int_as_float(0x7f800000))
                m = 48 - ilogbf(M);
            float a2[2] = {0.f, 0.f};
            for (int ul = threadIdx.x; ul < c.len; ul += kCta) {
                const float4 x = quad_f32(w, c.ubeg + ul, c.cols);
                const float4 d = quad_gy<GY_BF16>(gy, c.ubeg + ul, c.cols);
                const float4 xs = make_float4(scalbnf(x.x, m), scalbnf(x.y, m), scalbnf(x.z, m), scalbnf(x.w, m));
                acc_sq4(a2[0], xs);
                acc_dot4(a2[1], xs, d);
            }
            red.sum(a2);
            if (m != 0) {
                acc[0] = a2[0];
                acc[1] = a2[1];
            }
        }
        const float n2 = acc[0] + (m == 0 ? eps : scalbnf(eps, 2 * m));
        const float inv = 1.0f / sqrtf(n2);
        if constexpr (MODE != kModeGrad) {
            msh = m;
            q = acc[1] / n2;        // times 2^-m; applied to the scaled row
            sc = sg.radius * inv;   // rho / n times 2^-m
            return;
        }
        const float g = sg.gain ? __ldg(sg.gain + row * sg.gain_stride) : 1.f;
        q = m == 0 ? acc[1] / n2 : scalbnf(acc[1] / n2, m);
        pre = (g * sg.radius) * (m == 0 ? inv : scalbnf(inv, m));
        gg = sg.radius * acc[1] * inv;
    }

    __device__ void finish(bool leader, bool store)
    {
        if (MODE == kModeGrad && leader && store && sg.gain)
            sg.grad_g[row] = gg;
    }
};

struct SL2 {
    static constexpr int kPasses = 2;
    static constexpr int kArrays = 2; // x, r (r may be absent: zero bytes)
    const ASegK &sg;
    int64_t row;
    float eps;
    float acc = 0.f;
    RowScale rs{0.f, 1.f};

    __device__ SL2(const ASegK &s, int64_t r, float e) : sg(s), row(r), eps(e) {}
    __device__ int unit_bytes(int a) const { return (a == 0 || sg.r) ? 16 : 0; }
    __device__ const char *src(int a) const
    {
        return reinterpret_cast<const char *>((a == 0 ? sg.x : sg.r) + row * sg.ld);
    }

    __device__ __forceinline__ uint4 unit(const unsigned char *const *st, int j, int u, int cols) const
    {
        uint4 s = *reinterpret_cast<const uint4 *>(st[0] + 16 * j);
        if (sg.r)
            s = add_bf16x8(s, *reinterpret_cast<const uint4 *>(st[1] + 16 * j));
        const int valid = cols - 8 * u;
        return valid < 8 ? mask_octet(s, valid) : s;
    }

    __device__ __forceinline__ void consume(int pass, const unsigned char *const *st, int j, int u,
                                            const StreamCtx &c, bool store)
    {
        const uint4 s = unit(st, j, u, c.cols);
        if (pass == 0)
            acc_sq8(acc, s);
        else if (store)
            store_octet(sg.y + row * sg.ld, u, c.cols, scale_bf16x8(s, rs));
    }

    template <class Red>
    __device__ __forceinline__ void between(int, Red &red, const StreamCtx &c)
    {
        float a[1] = {acc};
        red.sum(a);
        const uint16_t *x = sg.x + row * sg.ld;
        const uint16_t *r = sg.r ? sg.r + row * sg.ld : nullptr;
        rs = row_scale(a[0], eps, red, [&](auto f) {
            for (int ul = threadIdx.x; ul < c.len; ul += kCta) {
                const int u = c.ubeg + ul;
                uint4 s = ld16(x + 8 * u);
                if (r)
                    s = add_bf16x8(s, ld16(r + 8 * u));
                const int valid = c.cols - 8 * u;
                each8(valid < 8 ? mask_octet(s, valid) : s, f);
            }
        });
    }
    __device__ void finish(bool, bool) {}
};

struct SSlerp {
    static constexpr int kPasses = 3;
    static constexpr int kArrays = 2;
    const ASegK &sg;
    int64_t row;
    float eps;
    float acc[2] = {0.f, 0.f};
    RowScale ra{0.f, 1.f}, rb{0.f, 1.f}, rt{0.f, 1.f};

    __device__ SSlerp(const ASegK &s, int64_t r, float e) : sg(s), row(r), eps(e) {}
    __device__ int unit_bytes(int) const { return 16; }
    __device__ const char *src(int a) const
    {
        return reinterpret_cast<const char *>((a == 0 ? sg.x : sg.r) + row * sg.ld);
    }

    template <class F>
    __device__ __forceinline__ void each_t(uint4 xa, uint4 xb, int u, int cols, F &&f) const
    {
        const uint4 a = scale_bf16x8(xa, ra);
        const uint4 b = scale_bf16x8(xb, rb);
        float m[8];
        alpha8(sg.alpha, u, cols, m);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            f(lerp_t(bf_get(a, e), bf_get(b, e), m[e]));
    }

    __device__ __forceinline__ void consume(int pass, const unsigned char *const *st, int j, int u,
                                            const StreamCtx &c, bool store)
    {
        uint4 xa = *reinterpret_cast<const uint4 *>(st[0] + 16 * j);
        uint4 xb = *reinterpret_cast<const uint4 *>(st[1] + 16 * j);
        const int valid = c.cols - 8 * u;
        if (valid < 8) {
            xa = mask_octet(xa, valid);
            xb = mask_octet(xb, valid);
        }
        if (pass == 0) {
            acc_sq8(acc[0], xa);
            acc_sq8(acc[1], xb);
        } else if (pass == 1) {
            each_t(xa, xb, u, c.cols, [&](float t) { acc[0] = fmaf(t, t, acc[0]); });
        } else if (store) {
            float h[8];
            int e = 0;
            each_t(xa, xb, u, c.cols, [&](float t) { h[e++] = (t * rt.pre) * rt.inv; });
            store_octet(sg.y + row * sg.ld, u, c.cols,
                        make_uint4(pack_bf2(h[0], h[1]), pack_bf2(h[2], h[3]), pack_bf2(h[4], h[5]),
                                   pack_bf2(h[6], h[7])));
        }
    }

    template <class Red>
    __device__ __forceinline__ void between(int pass, Red &red, const StreamCtx &c)
    {
        const uint16_t *xr = sg.x + row * sg.ld;
        const uint16_t *orow = sg.r + row * sg.ld;
        if (pass == 0) {
            red.sum(acc);
            ra = row_scale(acc[0], eps, red, [&](auto f) {
                for (int ul = threadIdx.x; ul < c.len; ul += kCta)
                    each8(octet(xr, c.ubeg + ul, c.cols), f);
            });
            rb = row_scale(acc[1], eps, red, [&](auto f) {
                for (int ul = threadIdx.x; ul < c.len; ul += kCta)
                    each8(octet(orow, c.ubeg + ul, c.cols), f);
            });
            acc[0] = 0.f;
        } else {
            float a[1] = {acc[0]};
            red.sum(a);
            rt = row_scale(a[0], eps, red, [&](auto f) {
                for (int ul = threadIdx.x; ul < c.len; ul += kCta) {
                    const int u = c.ubeg + ul;
                    each_t(octet(xr, u, c.cols), octet(orow, u, c.cols), u, c.cols, f);
                }
            });
        }
    }
    __device__ void finish(bool, bool) {}
};

template <int T>
struct StreamOp;
template <> struct StreamOp<kFwdBf16> { using type = SScale<true, false>; };
template <> struct StreamOp<kFwdF32> { using type = SScale<false, false>; };
template <> struct StreamOp<kRenorm> { using type = SScale<false, true>; };
template <> struct StreamOp<kBwdBf16> { using type = SBackward<true, kModeGrad>; };
template <> struct StreamOp<kBwdF32> { using type = SBackward<false, kModeGrad>; };
template <> struct StreamOp<kProject> { using type = SBackward<false, kModeProject>; };
template <> struct StreamOp<kMomentum> { using type = SBackward<false, kModeMomentum>; };
template <> struct StreamOp<kL2> { using type = SL2; };
template <> struct StreamOp<kSlerp> { using type = SSlerp; };

// Units per thread per chunk: 4 where one array streams (16 KB stages), 2
// where two do (16 KB stages for two 16-byte arrays), so that several CTAs
// share an SM (each streams one row slice and leaves).
template <int T>
__host__ __device__ constexpr int stream_k()
{
    return (T == kFwdBf16 || T == kFwdF32 || T == kRenorm) ? 4 : 2;
}

template <int T>
__host__ __device__ constexpr int stream_chunk_units()
{
    return kCta * stream_k<T>();
}

template <int T>
__host__ __device__ constexpr int stream_stage_bytes()
{
    // widest layout of the operation's arrays per stage
    constexpr int cu = stream_chunk_units<T>();
    return (T == kBwdF32 || T == kProject || T == kMomentum) ? 2 * 16 * cu
         : T == kBwdBf16 ? (16 + 8) * cu
         : (T == kL2 || T == kSlerp) ? 2 * 16 * cu
         : 16 * cu;
}

template <int T>
__global__ void __launch_bounds__(kCta, 1) k_stream(const __grid_constant__ ParamsOf<T> p)
{
    using Op = typename StreamOp<T>::type;
    constexpr int CU = stream_chunk_units<T>();
    extern __shared__ __align__(128) unsigned char ring[];
    __shared__ __align__(8) uint64_t full[kStages];
    __shared__ float red_sm[2 * kWarps * 4];
    __shared__ float red_dsm[2 * kMaxCluster * 4];
    cluster_arrive_relaxed();
    ClusterReducer red(red_sm, red_dsm);

    const int64_t unit = blockIdx.x / red.ncta;
    const int si = find_segment(p, unit);
    const auto &sg = p.seg[si];
    const int64_t row = unit - p.unit_start[si];
    Op op(sg, row, p.eps);

    StreamCtx c;
    c.cols = sg.cols;
    c.nu = sg.nu;
    // Even slices keep every slice of 8-byte units 16-byte aligned.
    int per = (c.nu + red.ncta - 1) / red.ncta;
    per = (per + 1) & ~1;
    c.ubeg = min(c.nu, static_cast<int>(red.rank) * per);
    c.len = min(c.nu, c.ubeg + per) - c.ubeg;
    const int nch = (c.len + CU - 1) / CU;
    const int total = Op::kPasses * nch;

    int ub[2], off[2];
    const char *src[2];
    int stage_bytes = 0;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
        ub[a] = a < Op::kArrays ? op.unit_bytes(a) : 0;
        src[a] = ub[a] ? op.src(a) + static_cast<int64_t>(c.ubeg) * ub[a] : nullptr;
        off[a] = stage_bytes;
        stage_bytes += ub[a] * CU;
    }

    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < kStages; ++s)
            mbar_init(&full[s], 1);
        mbar_init_fence();
    }
    __syncthreads();

    auto issue = [&](int i) {
        const int ch = i % nch;
        const int s = i % kStages;
        const int u0 = ch * CU;
        const int n = min(CU, c.len - u0);
        uint32_t bytes[2], tot = 0;
#pragma unroll
        for (int a = 0; a < 2; ++a) {
            bytes[a] = (static_cast<uint32_t>(n * ub[a]) + 15u) & ~15u;
            tot += bytes[a];
        }
        mbar_arrive_expect_tx(&full[s], tot);
#pragma unroll
        for (int a = 0; a < 2; ++a)
            if (bytes[a])
                bulk_g2s(ring + s * stage_bytes + off[a], src[a] + static_cast<int64_t>(u0) * ub[a], bytes[a],
                         &full[s]);
    };

    if (threadIdx.x == 0) {
        fence_proxy_async_smem();
        for (int i = 0; i < min(kStages, total); ++i)
            issue(i);
    }

    bool ok = true;
    for (int pass = 0; pass < Op::kPasses; ++pass) {
        for (int ch = 0; ch < nch; ++ch) {
            const int i = pass * nch + ch;
            const int s = i % kStages;
            if (!mbar_wait_bounded(&full[s], (i / kStages) & 1, p.wait_limit_ns))
                ok = false;
            const unsigned char *st[2] = {ring + s * stage_bytes + off[0], ring + s * stage_bytes + off[1]};
#pragma unroll
            for (int k = 0; k < stream_k<T>(); ++k) {
                const int j = threadIdx.x + k * kCta;
                const int ul = ch * CU + j;
                if (ul < c.len)
                    op.consume(pass, st, j, c.ubeg + ul, c, ok);
            }
            __syncthreads();
            if (threadIdx.x == 0 && i + kStages < total) {
                fence_proxy_async_smem();
                issue(i + kStages);
            }
        }
        if (pass + 1 < Op::kPasses)
            op.between(pass, red, c);
    }
    // a timed-out wait leaves no error silent and no copy in flight at exit
    ok = __syncthreads_and(ok) != 0;
    if (!ok) {
        if (threadIdx.x == 0) {
            raise_device_error(DS_ERR_DEVICE_TIMEOUT, kSiteStreamWait);
            for (int i = max(0, total - kStages); i < total; ++i)
                if (!mbar_wait_bounded(&full[i % kStages], (i / kStages) & 1, p.wait_limit_ns))
                    raise_device_error(DS_ERR_DEVICE_TIMEOUT, kSiteStreamDrain);
        }
        __syncthreads();
    }
    op.finish(threadIdx.x == 0 && red.rank == 0, ok);
    red.finish();
}

__global__ void k_wait_selftest(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
    }
    __syncthreads();
    // nothing arrives on the barrier: the bounded wait must give up
    if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, limit_ns))
        raise_device_error(DS_ERR_DEVICE_TIMEOUT, kSiteSelftest);
}

// =============================================================== launch ====

template <class K, class P>
cudaError_t launch_clustered(K kernel, const P &p, int64_t rows, int cluster, size_t smem, void *stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows * cluster), 1, 1);
    cfg.blockDim = dim3(kCta, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <int T>
cudaError_t launch_op(const RowClass &rc, const ParamsOf<T> &p, int64_t units, void *stream)
{
    switch (rc.path) {
    case DS_PATH_TWO_PASS: {
        constexpr int smem = kStages * stream_stage_bytes<T>();
        static DeviceFlags attr_set;
        if (const cudaError_t e = enable_dynamic_smem(k_stream<T>, smem, attr_set))
            return e;
        return launch_clustered(k_stream<T>, p, units, rc.cluster, smem, stream);
    }
    default:
        return cudaErrorInvalidValue;
    }
}

// ============================================================ row lengths ==
//
// One warp per row (the rows of every segment in one grid-stride walk): the
// lanes sum quads lane, lane + 32, ... in order into two accumulators, then
// the butterfly; rows whose fp32 sum overflows (or, at eps = 0, underflows)
// are summed again after an exact power-of-two scaling, as every row op
// here does.  Lane 0 writes sqrt(S + eps) / div.

struct WarpRowRed {
    __device__ __forceinline__ bool any(bool b) const { return __any_sync(0xffffffffu, b); }
    __device__ __forceinline__ float max(float v) const
    {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        return v;
    }
    template <int N>
    __device__ __forceinline__ void sum(float (&v)[N]) const
    {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i)
                v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
    }
};

__global__ void __launch_bounds__(kCta) k_row_norms(const __grid_constant__ RNParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = (static_cast<int64_t>(blockIdx.x) * kCta + threadIdx.x) >> 5;
    const int64_t nw = (static_cast<int64_t>(gridDim.x) * kCta) >> 5;
    const int64_t total = p.unit_start[p.nseg];
    const WarpRowRed red;
    for (int64_t u = gw; u < total; u += nw) {
        const int si = find_segment(p, u);
        const RNSegK &sg = p.seg[si];
        const int64_t row = u - p.unit_start[si];
        const float *w = sg.w + row * sg.ld;
        const int nq = (sg.cols + 3) / 4;
        float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
        for (int q = lane; q < nq; q += 32) {
            const float4 v = quad_f32(w, q, sg.cols);
            a0 = fmaf(v.x, v.x, a0);
            a1 = fmaf(v.y, v.y, a1);
            a0 = fmaf(v.z, v.z, a0);
            a1 = fmaf(v.w, v.w, a1);
        }
        float S[1] = {a0 + a1};
        red.sum(S);
        float Ss = S[0];
        const int m = rescale_exponent(S[0], p.eps, red, [&](auto f) {
            for (int q = lane; q < nq; q += 32)
                each4(quad_f32(w, q, sg.cols), f);
        }, Ss);
        const float len = m == 0 ? sqrtf(S[0] + p.eps) : scalbnf(sqrtf(Ss + scalbnf(p.eps, 2 * m)), -m);
        if (lane == 0)
            sg.out[row] = __fdiv_rn(len, sg.div);
    }
}

// ===================================================== scalar gain sums ==
//
// One block per buffer: thread t adds parts t, t + 1024, ... in order in
// double, then a fixed tree over the block; the sum is rounded once to fp32.

__global__ void __launch_bounds__(1024) k_gain_sums(const __grid_constant__ GainSumParams p)
{
    __shared__ double part[1024];
    const GainSumK &sg = p.seg[blockIdx.x];
    double acc = 0.0;
    for (int64_t i = threadIdx.x; i < sg.rows; i += 1024)
        acc += static_cast<double>(sg.parts[i]);
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int o = 512; o > 0; o >>= 1) {
        if (threadIdx.x < o)
            part[threadIdx.x] += part[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        sg.parts[sg.rows] = static_cast<float>(part[0]);
}

} // namespace

int launch_wn_forward(const RowClass &rc, const WParams &p, int64_t units, bool out_bf16, void *stream)
{
    return out_bf16 ? launch_op<kFwdBf16>(rc, p, units, stream) : launch_op<kFwdF32>(rc, p, units, stream);
}

int launch_wn_backward(const RowClass &rc, const WParams &p, int64_t units, bool gy_bf16, void *stream)
{
    return gy_bf16 ? launch_op<kBwdBf16>(rc, p, units, stream) : launch_op<kBwdF32>(rc, p, units, stream);
}

int launch_row_renorm(const RowClass &rc, const WParams &p, int64_t units, void *stream)
{
    return launch_op<kRenorm>(rc, p, units, stream);
}

int launch_grad_project(const RowClass &rc, const WParams &p, int64_t units, void *stream)
{
    return launch_op<kProject>(rc, p, units, stream);
}

int launch_renorm_momentum(const RowClass &rc, const WParams &p, int64_t units, void *stream)
{
    return launch_op<kMomentum>(rc, p, units, stream);
}

int launch_l2_rows(const RowClass &rc, const AParams &p, int64_t units, void *stream)
{
    return launch_op<kL2>(rc, p, units, stream);
}

int launch_slerp_rows(const RowClass &rc, const AParams &p, int64_t units, void *stream)
{
    return launch_op<kSlerp>(rc, p, units, stream);
}

int launch_row_norms(const RNParams &p, int sms, void *stream)
{
    const int64_t warps = p.unit_start[p.nseg];
    const int64_t blocks = std::min<int64_t>((warps + kWarps - 1) / kWarps, int64_t(sms) * 8);
    k_row_norms<<<static_cast<int>(blocks), kCta, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError();
}

int launch_gain_sums(const GainSumParams &p, void *stream)
{
    k_gain_sums<<<p.nseg, 1024, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return cudaGetLastError();
}

int launch_wait_selftest(uint64_t limit_ns, void *stream)
{
    k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    return cudaGetLastError();
}

int read_and_clear_device_error(uint32_t *code, uint32_t *site, void *stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess)
        return e;
    *code = 0;
    *site = 0;
    // every module's word is cleared; the first error found is reported
    int (*const readers[3])(uint32_t *, uint32_t *) = {module_read_and_clear_error, tile_read_and_clear_error,
                                                       qk_read_and_clear_error};
    for (auto rd : readers) {
        uint32_t c = 0, st = 0;
        const int r = rd(&c, &st);
        if (r != cudaSuccess)
            return r;
        if (c != 0 && *code == 0) {
            *code = c;
            *site = st;
        }
    }
    return cudaSuccess;
}

} // namespace ds
