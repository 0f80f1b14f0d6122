// ds_api.cpp -- the C ABI of libds: argument validation, row-class planning,
// segment-table packing into kernel parameter blocks, and launches.
//
// Planning: every segment's row class depends on (operation, cols) only.
// Segments of one class go into as few launches as the parameter block
// allows (kSegPerLaunch segments each); a segment with more rows than a grid
// can hold is split by rows (rows are independent).  Nothing is allocated.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "ds.h"
#include "ds_internal.h"

namespace {

using ds::AGSegK;
using ds::AParams;
using ds::ASegK;
using ds::GParams;
using ds::RowClass;
using ds::WParams;
using ds::WSegK;

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_force_path{DS_PATH_AUTO};
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

constexpr int64_t kMaxCols = 0x7fffffff;
constexpr int64_t kMaxGrid = 0x7fffffff;

ds_status fail(ds_status s, const std::string &msg)
{
    g_last_error = msg;
    return s;
}

std::string where(const char *what, int seg)
{
    char buf[96];
    std::snprintf(buf, sizeof(buf), "segment %d: %s", seg, what);
    return buf;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Bytes per unit (quad of a weight row, octet of an activation row) that a
// row stages in shared memory on the staged paths, for the widest layout of
// the operation (fp32 GY; a residual present), so that the class -- and with
// it the row's arithmetic -- depends on (op, cols) only.  The l2 backward
// without a residual (has_r false) is its own layout: two arrays.
int64_t unit_bytes_worst(ds_op op, bool has_r = true)
{
    switch (op) {
    case DS_OP_WN_FORWARD:
    case DS_OP_ROW_RENORM: return 16;
    case DS_OP_WN_BACKWARD:
    case DS_OP_GRAD_PROJECT:
    case DS_OP_RENORM_MOMENTUM: return 32;
    case DS_OP_L2_ROWS_BACKWARD: return has_r ? 48 : 32;
    case DS_OP_SLERP_ROWS_BACKWARD: return 48;
    default: return 32;
    }
}

bool is_act_bwd(ds_op op) { return op == DS_OP_L2_ROWS_BACKWARD || op == DS_OP_SLERP_ROWS_BACKWARD; }
bool is_fused(ds_op op) { return op == DS_OP_GATE_L2_ROWS || op == DS_OP_SWIGLU_L2_ROWS; }
// Operations with staged classes only (no two-pass stream): rows longer
// than a cluster of 8 staged slices are refused.
bool staged_only(ds_op op) { return is_act_bwd(op) || is_fused(op); }

// Warps of a staged team: one (weights) or two (activations) per 16 KB of
// slot; eight for the 112 KB weight slots.
int team_warps(ds_op op, int slot)
{
    if (slot == ds::kTileSlotMaxWeightBytes)
        return 8;
    const int base = (op == DS_OP_L2_ROWS || op == DS_OP_SLERP_ROWS || staged_only(op)) ? 2 : 1;
    return base * slot / ds::kTileSlotBytes;
}

// Largest staged slot of an operation for one CTA per row; a slice of a row
// split over a cluster takes at most 64 KB (three ring positions or more).
int64_t max_slot(ds_op op)
{
    return ds::is_weight_op(op) ? ds::kTileSlotMaxWeightBytes : ds::kTileSlotMaxBytes;
}
constexpr int64_t kClusterSliceMax = 65536;

// Row classes, from (op, cols) alone:
//   WARP     one CTA per row, the row's staged input <= 16 KB (16 KB slots)
//   CTA      one CTA per row, <= 64 KB (activations) or 112 KB (weights)
//   CLUSTER  2, 4 or 8 CTAs per row, each staging a slice of <= 64 KB: the
//            smallest cluster whose slices fit, in the smallest slot that
//            holds a slice
//   TWO_PASS anything longer (operations with a streaming kernel)
// `forced` (a test knob) picks a class where the row allows it.
RowClass classify(ds_op op, int64_t cols, int forced, bool has_r = true)
{
    const int64_t E = ds::elems_per_unit(op);
    const int nu = static_cast<int>((cols + E - 1) / E);
    const int64_t ubw = unit_bytes_worst(op, has_r);
    auto staged = [&](int path, int cl, int min_slot, int64_t top) -> RowClass {
        const int64_t bytes = ds::slice_per(nu, cl) * ubw;
        for (const int slot : {16384, 32768, 65536, 114688})
            if (slot >= min_slot && slot <= top && bytes <= slot)
                return {path, 32 * team_warps(op, slot), cl, 0, slot};
        return {0, 0, 0, 0, 0};
    };
    auto cluster = [&]() -> RowClass {
        for (int cl = 2; cl <= ds::kMaxCluster; cl *= 2)
            if (const RowClass c = staged(DS_PATH_CLUSTER, cl, 16384, kClusterSliceMax); c.path)
                return c;
        return {0, 0, 0, 0, 0};
    };
    const RowClass two_pass = staged_only(op) ? RowClass{0, 0, 0, 0, 0}
                                              : RowClass{DS_PATH_TWO_PASS, 0, ds::kMaxCluster, 0, 0};
    switch (forced) {
    case DS_PATH_WARP:
        if (const RowClass c = staged(DS_PATH_WARP, 1, 16384, 16384); c.path)
            return c;
        break;
    case DS_PATH_CTA:
        if (const RowClass c = staged(DS_PATH_CTA, 1, 32768, max_slot(op)); c.path)
            return c;
        break;
    case DS_PATH_CLUSTER:
        if (const RowClass c = cluster(); c.path)
            return c;
        break;
    case DS_PATH_TWO_PASS:
        if (two_pass.path)
            return two_pass;
        break;
    default:
        break;
    }
    if (const RowClass c = staged(DS_PATH_WARP, 1, 16384, 16384); c.path)
        return c;
    if (const RowClass c = staged(DS_PATH_CTA, 1, 32768, max_slot(op)); c.path)
        return c;
    if (const RowClass c = cluster(); c.path)
        return c;
    return two_pass;
}

// Rows per shared-memory slot of `slot` bytes on the staged paths for the
// actual layout (staged arrays of this segment) of a row slice of `units`
// units (the whole row with one CTA per row), at most kTileMaxRowsPerSlot.
int tile_rows_per_slot(ds_op op, int units, int gy_esize, bool has_r, int slot)
{
    const int64_t q = units, o = units;
    int64_t bytes = 0;
    switch (op) {
    case DS_OP_WN_FORWARD:
    case DS_OP_ROW_RENORM: bytes = q * 16; break;
    case DS_OP_WN_BACKWARD: bytes = q * 16 + (q * gy_esize * 4 + 15) / 16 * 16; break;
    case DS_OP_GRAD_PROJECT:
    case DS_OP_RENORM_MOMENTUM: bytes = 2 * q * 16; break;
    case DS_OP_L2_ROWS: bytes = o * 16 * (has_r ? 2 : 1); break;
    case DS_OP_L2_ROWS_BACKWARD: bytes = o * 16 * (has_r ? 3 : 2); break;
    case DS_OP_GATE_L2_ROWS:
    case DS_OP_SWIGLU_L2_ROWS: bytes = o * 16 * 2; break;
    case DS_OP_SLERP_ROWS_BACKWARD: bytes = o * 16 * 3; break;
    default: bytes = o * 32; break;
    }
    if (bytes == 0)
        return ds::kTileMaxRowsPerSlot;
    return static_cast<int>(std::min<int64_t>(ds::kTileMaxRowsPerSlot, slot / bytes));
}

// Units of the largest slice of a row of `cols` columns in class rc.
int slice_units(ds_op op, int64_t cols, const RowClass &rc)
{
    const int64_t E = ds::elems_per_unit(op);
    return ds::slice_per(static_cast<int>((cols + E - 1) / E), rc.cluster);
}

int sm_count()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    if (!cache[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Rows per work unit: a shared-memory slot (staged paths) or one row (a
// cluster per row).
int64_t rows_per_unit(const RowClass &rc)
{
    return ds::is_staged(rc) ? rc.rps : 1;
}

int64_t units_for(const RowClass &rc, int64_t rows)
{
    const int64_t rpu = rows_per_unit(rc);
    return (rows + rpu - 1) / rpu;
}

// ----------------------------------------------------------- overlap check --

struct Span {
    uintptr_t lo, hi;
    int seg;
    int role;   // 0 = read, 1 = written
    int alias;  // allowed exact-alias key within a segment (-1: none)
};

// Byte span of a row-major matrix: through the end of its last row.
Span span_of(const void *p, int64_t rows, int64_t cols, int64_t ld, int esize, int seg, int role, int alias)
{
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    const uintptr_t n = static_cast<uintptr_t>(((rows - 1) * ld + cols) * esize);
    return {lo, lo + n, seg, role, alias};
}

ds_status check_overlaps(std::vector<Span> &spans)
{
    std::sort(spans.begin(), spans.end(), [](const Span &a, const Span &b) { return a.lo < b.lo; });
    for (size_t i = 0; i < spans.size(); ++i) {
        for (size_t j = i + 1; j < spans.size() && spans[j].lo < spans[i].hi; ++j) {
            const Span &a = spans[i], &b = spans[j];
            if (a.role == 0 && b.role == 0)
                continue;
            const bool exact = a.lo == b.lo && a.hi == b.hi && a.seg == b.seg && a.alias >= 0 &&
                               a.alias == b.alias;
            if (!exact)
                return fail(DS_ERR_OVERLAP, where("an output overlaps another buffer of the call", b.seg));
        }
    }
    return DS_OK;
}

ds_status check_common(int nseg, const void *segs, float eps, void *)
{
    if (nseg < 0)
        return fail(DS_ERR_INVALID_ARG, "nseg < 0");
    if (nseg > DS_MAX_SEGMENTS)
        return fail(DS_ERR_TOO_MANY_SEGMENTS, "nseg above DS_MAX_SEGMENTS");
    if (nseg > 0 && !segs)
        return fail(DS_ERR_INVALID_ARG, "segs is NULL");
    if (!(eps >= 0.f) || !std::isfinite(eps))
        return fail(DS_ERR_INVALID_ARG, "eps must be finite and >= 0");
    return DS_OK;
}

ds_status check_shape(int64_t rows, int64_t cols, int64_t ld, int i)
{
    if (rows < 0)
        return fail(DS_ERR_INVALID_ARG, where("rows < 0", i));
    if (cols < 1 || cols > kMaxCols)
        return fail(DS_ERR_INVALID_ARG, where("cols outside [1, 2^31 - 1]", i));
    if (ld < cols)
        return fail(DS_ERR_INVALID_ARG, where("leading dimension < cols", i));
    if (rows > 0 && ld > (int64_t(1) << 40))
        return fail(DS_ERR_INVALID_ARG, where("leading dimension too large", i));
    if (rows > (int64_t(1) << 40))
        return fail(DS_ERR_INVALID_ARG, where("rows too large", i));
    return DS_OK;
}

ds_status check_matrix(const void *p, int64_t rows, int64_t ld, int esize, const char *name, int i)
{
    if (rows == 0)
        return DS_OK;
    if (!p)
        return fail(DS_ERR_INVALID_ARG, where((std::string(name) + " is NULL").c_str(), i));
    if (!aligned(p, 16) || (ld * esize) % 16 != 0)
        return fail(DS_ERR_ALIGNMENT, where((std::string(name) + " rows are not 16-byte aligned").c_str(), i));
    return DS_OK;
}

// ------------------------------------------------------------- launching --

// Splits, packs and launches.  `make(i, r0, nrows)` returns the device
// segment for rows [r0, r0 + nrows) of segment i.
// Slerp launches whose segments all use one alpha vector let the staged
// kernel keep |alpha| in shared memory (the kernel checks the length of its
// slice of the columns against its own cache).
// The Dory rows do the same with their scale vectors (sa, and sb when every
// segment shares one).
inline void shared_alpha(WParams &p, int)
{
    p.alpha_shared = p.alpha2_shared = nullptr;
    p.alpha_cols = 0;
}
template <class P>
inline void shared_alpha_act(P &p, int n)
{
    p.alpha_shared = p.alpha2_shared = nullptr;
    p.alpha_cols = 0;
    if (n == 0 || !p.seg[0].alpha)
        return;
    for (int i = 1; i < n; ++i)
        if (p.seg[i].alpha != p.seg[0].alpha || p.seg[i].cols != p.seg[0].cols)
            return;
    p.alpha_shared = p.seg[0].alpha;
    p.alpha_cols = p.seg[0].cols;
}
inline void shared_alpha(AParams &p, int n)
{
    shared_alpha_act(p, n);
    if (!p.alpha_shared || n == 0 || !p.seg[0].s2)
        return;
    for (int i = 1; i < n; ++i)
        if (p.seg[i].s2 != p.seg[0].s2)
            return;
    p.alpha2_shared = p.seg[0].s2;
}
inline void shared_alpha(GParams &p, int n) { shared_alpha_act(p, n); }

struct NoPrep {
    template <class P>
    void operator()(P &) const {}
};

// `prep(params)` runs on each packed parameter block just before its launch.
template <class P, class SegK, class Make, class Launch, class Prep = NoPrep>
ds_status launch_all(int nseg, const int64_t *rows, const std::vector<RowClass> &cls, float eps, Make make,
                     Launch launch, void *stream, Prep prep = Prep())
{
    std::vector<char> done(static_cast<size_t>(nseg), 0);

    static thread_local P params; // ~12 KB: kept off the stack
    for (int first = 0; first < nseg; ++first) {
        if (done[first] || rows[first] == 0)
            continue;
        const RowClass rc = cls[first];
        const int64_t unit_cap = kMaxGrid / std::max(1, rc.cluster);
        int n = 0;
        int64_t units = 0;
        auto flush = [&]() -> ds_status {
            if (n == 0)
                return DS_OK;
            params.nseg = n;
            params.unit_start[n] = units;
            params.eps = eps;
            params.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
            shared_alpha(params, n);
            params.ws = nullptr;
            params.ws_ld = 0;
            prep(params);
            const int e = launch(rc, params, units, stream);
            if (e != 0) {
                char buf[160];
                std::snprintf(buf, sizeof(buf), "kernel launch failed (cudaError %d)", e);
                return fail(DS_ERR_CUDA, buf);
            }
            g_launches.fetch_add(1, std::memory_order_relaxed);
            n = 0;
            units = 0;
            return DS_OK;
        };
        for (int i = first; i < nseg; ++i) {
            if (done[i] || rows[i] == 0 || !ds::same_launch(cls[i], rc))
                continue;
            done[i] = 1;
            const RowClass ci = cls[i];
            // rows per piece so that one piece never exceeds a grid
            const int64_t rpu = rows_per_unit(ci);
            for (int64_t r0 = 0; r0 < rows[i];) {
                int64_t room = unit_cap - units;
                if (n == ds::kSegPerLaunch || room <= 0) {
                    if (ds_status s = flush())
                        return s;
                    room = unit_cap;
                }
                const int64_t nr = std::min(rows[i] - r0, room * rpu);
                params.seg[n] = make(i, r0, nr);
                params.seg[n].group = ds::is_staged(ci) ? ci.rps : ci.group;
                params.unit_start[n] = units;
                units += units_for(ci, nr);
                ++n;
                r0 += nr;
            }
        }
        if (ds_status s = flush())
            return s;
    }
    return DS_OK;
}

WSegK wseg_rows(const ds_wseg &s, int64_t r0, int64_t nr, int out_esize, int gy_esize)
{
    WSegK k{};
    k.w = s.w ? s.w + r0 * s.ld : nullptr;
    k.gain = s.gain ? (s.gain_scalar ? s.gain : s.gain + r0) : nullptr;
    k.gain_stride = s.gain_scalar ? 0 : 1;
    k.out = s.w_eff ? static_cast<char *>(s.w_eff) + r0 * s.ld_out * out_esize : nullptr;
    k.gy = s.gy ? static_cast<const char *>(s.gy) + r0 * s.ld_out * gy_esize : nullptr;
    k.grad_w = s.grad_w ? s.grad_w + r0 * s.ld : nullptr;
    k.grad_g = s.grad_g ? s.grad_g + r0 : nullptr;
    k.rows = nr;
    k.ld = s.ld;
    k.ld_out = s.ld_out;
    k.cols = static_cast<int32_t>(s.cols);
    k.nu = static_cast<int32_t>((s.cols + 3) / 4);
    k.radius = s.radius;
    return k;
}

ASegK aseg_rows(const ds_aseg &s, int64_t r0, int64_t nr)
{
    ASegK k{};
    k.x = s.x ? static_cast<const uint16_t *>(s.x) + r0 * s.ld : nullptr;
    k.r = s.r ? static_cast<const uint16_t *>(s.r) + r0 * s.ld : nullptr;
    k.y = s.y ? static_cast<uint16_t *>(s.y) + r0 * s.ld : nullptr;
    k.alpha = s.alpha;
    k.rows = nr;
    k.ld = s.ld;
    k.cols = static_cast<int32_t>(s.cols);
    k.nu = static_cast<int32_t>((s.cols + 7) / 8);
    return k;
}

enum WOp { W_FWD, W_BWD, W_RENORM, W_PROJECT, W_MOMENTUM };

ds_status run_weight(WOp wop, const ds_wseg *segs, int nseg, ds_dtype dt, float eps, void *stream)
{
    g_last_error.clear();
    if (ds_status s = check_common(nseg, segs, eps, stream))
        return s;
    const bool fwd_bwd = wop == W_FWD || wop == W_BWD;
    if (fwd_bwd && dt != DS_F32 && dt != DS_BF16)
        return fail(DS_ERR_UNSUPPORTED_DTYPE, "dtype must be DS_F32 or DS_BF16");
    const int esize = dt == DS_BF16 ? 2 : 4;
    std::vector<Span> spans;
    std::vector<int64_t> rows(static_cast<size_t>(nseg)), cols(static_cast<size_t>(nseg));
    for (int i = 0; i < nseg; ++i) {
        const ds_wseg &s = segs[i];
        if (s.transposed != 0 && s.transposed != 1)
            return fail(DS_ERR_INVALID_ARG, where("transposed must be 0 or 1", i));
        const bool tr = s.transposed != 0;
        if (s.tgroup < 0 || s.tgroup > 256 || (!tr && s.tgroup > 1))
            return fail(DS_ERR_INVALID_ARG, where("tgroup must be 0 or 1, or 1..256 with transposed", i));
        // G stored columns per unit row (ConvTranspose weights; 1 for Conv1D)
        const int64_t G = tr ? std::max<int32_t>(1, s.tgroup) : 1;
        if (tr && s.cols % G != 0)
            return fail(DS_ERR_INVALID_ARG, where("transposed: cols is not a multiple of tgroup", i));
        // the stored matrix: [rows, ld] with cols used per row, or
        // (transposed) [cols / G, ld] with rows * G used per stored row
        const int64_t sr = tr ? s.cols / G : s.rows, sc = tr ? s.rows * G : s.cols;
        if (ds_status st = check_shape(s.rows, s.cols, tr ? std::max<int64_t>(s.ld, s.cols) : s.ld, i))
            return st;
        if (tr && s.ld < sc)
            return fail(DS_ERR_INVALID_ARG, where("transposed: leading dimension < rows * tgroup", i));
        if (tr && sc > (int64_t(1) << 31) - 1)
            return fail(DS_ERR_INVALID_ARG, where("transposed: rows * tgroup above 2^31 - 1", i));
        if (fwd_bwd && s.ld_out < sc)
            return fail(DS_ERR_INVALID_ARG,
                        where(tr ? "transposed: ld_out < rows * tgroup" : "ld_out < cols", i));
        if (!std::isfinite(s.radius))
            return fail(DS_ERR_INVALID_ARG, where("radius is not finite", i));
        rows[i] = tr ? 0 : s.rows; // transposed segments launch on their own
        cols[i] = s.cols;
        if (s.rows == 0)
            continue;
        if (ds_status st = check_matrix(s.w, sr, s.ld, 4, "w", i))
            return st;
        if (fwd_bwd && s.gain && !aligned(s.gain, 4))
            return fail(DS_ERR_ALIGNMENT, where("gain is not 4-byte aligned", i));
        if (fwd_bwd && s.gain_scalar != 0 && s.gain_scalar != 1)
            return fail(DS_ERR_INVALID_ARG, where("gain_scalar must be 0 or 1", i));
        if (fwd_bwd && s.gain_scalar && !s.gain)
            return fail(DS_ERR_INVALID_ARG, where("gain_scalar needs a gain", i));
        // gain: [rows], or [1] for a scalar gain; grad_g: [rows] or [rows + 1]
        const int64_t ng = s.gain_scalar ? 1 : s.rows, ngg = s.gain_scalar ? s.rows + 1 : s.rows;
        if (wop == W_FWD) {
            if (ds_status st = check_matrix(s.w_eff, sr, s.ld_out, esize, "w_eff", i))
                return st;
            spans.push_back(span_of(s.w, sr, sc, s.ld, 4, i, 0, -1));
            if (s.gain)
                spans.push_back(span_of(s.gain, 1, ng, ng, 4, i, 0, -1));
            spans.push_back(span_of(s.w_eff, sr, sc, s.ld_out, esize, i, 1, -1));
        } else if (wop == W_BWD) {
            if (ds_status st = check_matrix(s.gy, sr, s.ld_out, esize, "gy", i))
                return st;
            if (ds_status st = check_matrix(s.grad_w, sr, s.ld, 4, "grad_w", i))
                return st;
            if (s.gain && !s.grad_g)
                return fail(DS_ERR_INVALID_ARG, where("grad_g is NULL while gain is set", i));
            if (s.gain && !aligned(s.grad_g, 4))
                return fail(DS_ERR_ALIGNMENT, where("grad_g is not 4-byte aligned", i));
            spans.push_back(span_of(s.w, sr, sc, s.ld, 4, i, 0, -1));
            spans.push_back(span_of(s.gy, sr, sc, s.ld_out, esize, i, 0, -1));
            spans.push_back(span_of(s.grad_w, sr, sc, s.ld, 4, i, 1, -1));
            if (s.gain) {
                spans.push_back(span_of(s.gain, 1, ng, ng, 4, i, 0, -1));
                spans.push_back(span_of(s.grad_g, 1, ngg, ngg, 4, i, 1, -1));
            }
        } else if (wop == W_PROJECT || wop == W_MOMENTUM) {
            if (ds_status st = check_matrix(s.grad_w, sr, s.ld, 4,
                                            wop == W_PROJECT ? "grad_w (the gradient)" : "grad_w (the momentum)", i))
                return st;
            // the gradient / momentum is updated in place; w is read (project)
            // or updated in place (momentum); the two must not overlap
            spans.push_back(span_of(s.w, sr, sc, s.ld, 4, i, wop == W_MOMENTUM ? 1 : 0, -1));
            spans.push_back(span_of(s.grad_w, sr, sc, s.ld, 4, i, 1, -1));
        } else {
            spans.push_back(span_of(s.w, sr, sc, s.ld, 4, i, 1, -1));
        }
    }
    if (ds_status st = check_overlaps(spans))
        return st;

    const ds_op op = wop == W_FWD ? DS_OP_WN_FORWARD
                   : wop == W_BWD ? DS_OP_WN_BACKWARD
                   : wop == W_RENORM ? DS_OP_ROW_RENORM
                   : wop == W_PROJECT ? DS_OP_GRAD_PROJECT : DS_OP_RENORM_MOMENTUM;
    const int forced = g_force_path.load(std::memory_order_relaxed);
    std::vector<RowClass> cls(static_cast<size_t>(nseg));
    for (int i = 0; i < nseg; ++i) {
        cls[i] = classify(op, cols[i], forced);
        if (ds::is_staged(cls[i]))
            cls[i].rps = tile_rows_per_slot(op, slice_units(op, cols[i], cls[i]), esize, true, cls[i].slot);
    }
    auto make = [&](int i, int64_t r0, int64_t nr) {
        WSegK k = wseg_rows(segs[i], r0, nr, esize, esize);
        if (wop == W_RENORM)
            k.out = k.w ? const_cast<float *>(k.w) : nullptr;
        if (wop == W_PROJECT || wop == W_MOMENTUM) {
            // the kernels read the gradient / momentum as their second input
            // (fp32, the rows' ld) and write it back in place; momentum also
            // writes the rescaled rows over w
            k.gy = k.grad_w;
            k.ld_out = k.ld;
            k.gain = nullptr;
            k.grad_g = nullptr;
            k.out = (wop == W_MOMENTUM && k.w) ? const_cast<float *>(k.w) : nullptr;
        }
        return k;
    };
    const bool bf16 = dt == DS_BF16;
    auto launch = [&](const RowClass &rc, const WParams &p, int64_t units, void *st) -> int {
        if (ds::is_staged(rc)) {
            const int tag = wop == W_FWD ? (bf16 ? 0 : 1)
                          : wop == W_BWD ? (bf16 ? 2 : 3)
                          : wop == W_RENORM ? 4
                          : wop == W_PROJECT ? 7 : 8;
            int used = 0;
            return ds::launch_tile(tag, &p, units, rc.slot, rc.cluster, &used, st);
        }
        switch (wop) {
        case W_FWD: return ds::launch_wn_forward(rc, p, units, bf16, st);
        case W_BWD: return ds::launch_wn_backward(rc, p, units, bf16, st);
        case W_PROJECT: return ds::launch_grad_project(rc, p, units, st);
        case W_MOMENTUM: return ds::launch_renorm_momentum(rc, p, units, st);
        default: return ds::launch_row_renorm(rc, p, units, st);
        }
    };
    if (ds_status st = launch_all<WParams, WSegK>(nseg, rows.data(), cls, eps, make, launch, stream))
        return st;
    // transposed rows: whole column tiles staged over a cluster where they
    // fit shared memory (one launch per tile shape), else the column kernel
    // (one launch over the rest, tiles of col_tile_rows())
    {
        static thread_local WParams tp;
        const int cop = wop == W_FWD ? 0 : wop == W_BWD ? 1 : wop == W_RENORM ? 2 : wop == W_PROJECT ? 3 : 4;
        // bytes per element staged: w, and the second input (GY or the
        // gradient / momentum) where the operation reads one
        const int eb = 4 + (cop == 1 ? esize : (cop == 3 || cop == 4) ? 4 : 0);
        std::vector<int> ct_of(static_cast<size_t>(nseg), 0), cl_of(static_cast<size_t>(nseg), 0);
        // Per segment: the first budget that holds some tile shape, and in it
        // the smallest cluster, then the widest tile (fewer CTAs meeting at
        // each tile's barrier measured faster than wider tiles).
        // G stored columns per unit row: the tiles take G = 1 and powers of
        // two up to 32 (a tile then holds whole unit rows); other G, and
        // grouped rows too tall for the tiles, take the grouped kernel
        auto gsize = [&](int i) { return segs[i].transposed && segs[i].tgroup > 1 ? segs[i].tgroup : 1; };
        auto tile_group = [&](int g) { return g == 1 || (g <= 32 && (g & (g - 1)) == 0); };
        for (int i = 0; i < nseg; ++i) {
            if (!segs[i].transposed || segs[i].rows == 0 || !tile_group(gsize(i)))
                continue;
            const int64_t K = segs[i].cols / gsize(i);   // stored rows
            for (const int budget : ds::kColTileBudgets) {
                for (const int cl : {1, 2, 4, 8}) {
                    for (const int ct : {128, 64, 32, 16})
                        if (ct >= gsize(i) && ds::col_tile_smem(ct, cl, (K + cl - 1) / cl, eb) <= budget) {
                            ct_of[i] = ct;
                            cl_of[i] = cl;
                            break;
                        }
                    if (ct_of[i])
                        break;
                }
                if (ct_of[i])
                    break;
            }
        }
        for (const int ct : {128, 64, 32, 16, 0})
            for (const int cl : {1, 2, 4, 8}) {
                if (ct == 0 && cl != 1)
                    continue;
                int n = 0, smem = 0;
                int64_t units = 0;
                auto flush = [&]() -> ds_status {
                    if (n == 0)
                        return DS_OK;
                    tp.nseg = n;
                    tp.unit_start[n] = units;
                    tp.eps = eps;
                    tp.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
                    const int e = ct ? ds::launch_colt(cop, bf16, ct, cl, smem, tp, units, stream)
                                     : ds::launch_col(cop, bf16, tp, units, stream);
                    if (e != 0) {
                        char buf[160];
                        std::snprintf(buf, sizeof(buf), "kernel launch failed (transposed rows, cudaError %d)", e);
                        return fail(DS_ERR_CUDA, buf);
                    }
                    g_launches.fetch_add(1, std::memory_order_relaxed);
                    n = 0;
                    units = 0;
                    smem = 0;
                    return DS_OK;
                };
                for (int i = 0; i < nseg; ++i) {
                    if (!segs[i].transposed || segs[i].rows == 0 || ct_of[i] != ct || (ct && cl_of[i] != cl) ||
                        (!ct && gsize(i) > 1))
                        continue;
                    if (n == (ct ? ds::col_tile_segments() : ds::kSegPerLaunch))
                        if (ds_status st = flush())
                            return st;
                    const int tile = ct ? ct : ds::col_tile_rows();
                    const int64_t G = gsize(i);
                    tp.seg[n] = make(i, 0, segs[i].rows);
                    tp.seg[n].group = static_cast<int32_t>(G);
                    tp.unit_start[n] = units;
                    units += (segs[i].rows * G + tile - 1) / tile;   // tiles of stored columns
                    if (ct)
                        smem = std::max(smem, ds::col_tile_smem(ct, cl, (segs[i].cols / G + cl - 1) / cl, eb));
                    ++n;
                }
                if (ds_status st = flush())
                    return st;
            }
        // grouped transposed rows (ConvTranspose): blocks of col_group_units(G)
        // unit rows, one launch per table of segments
        int n = 0;
        int64_t units = 0;
        auto flush_g = [&]() -> ds_status {
            if (n == 0)
                return DS_OK;
            tp.nseg = n;
            tp.unit_start[n] = units;
            tp.eps = eps;
            tp.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
            if (const int e = ds::launch_colg(cop, bf16, tp, units, stream)) {
                char buf[160];
                std::snprintf(buf, sizeof(buf), "kernel launch failed (grouped transposed rows, cudaError %d)", e);
                return fail(DS_ERR_CUDA, buf);
            }
            g_launches.fetch_add(1, std::memory_order_relaxed);
            n = 0;
            units = 0;
            return DS_OK;
        };
        for (int i = 0; i < nseg; ++i) {
            if (gsize(i) == 1 || ct_of[i] != 0 || segs[i].rows == 0)
                continue;
            if (n == ds::kSegPerLaunch)
                if (ds_status st = flush_g())
                    return st;
            const int G = segs[i].tgroup, U = ds::col_group_units(G);
            tp.seg[n] = make(i, 0, segs[i].rows);
            tp.seg[n].group = G;
            tp.seg[n].nu = U;
            tp.unit_start[n] = units;
            units += (segs[i].rows + U - 1) / U;
            ++n;
        }
        if (ds_status st = flush_g())
            return st;
    }
    if (wop != W_BWD)
        return DS_OK;
    // scalar gains: dL/dg = the per-row parts summed (fixed order), after them
    static thread_local ds::GainSumParams sums;
    sums.nseg = 0;
    auto flush_sums = [&]() -> ds_status {
        if (sums.nseg == 0)
            return DS_OK;
        if (ds::launch_gain_sums(sums, stream) != 0)
            return fail(DS_ERR_CUDA, "gain-sum launch failed");
        g_launches.fetch_add(1, std::memory_order_relaxed);
        sums.nseg = 0;
        return DS_OK;
    };
    for (int i = 0; i < nseg; ++i) {
        const ds_wseg &s = segs[i];
        if (!s.gain || !s.gain_scalar)
            continue;
        if (sums.nseg == ds::kSegPerLaunch)
            if (ds_status st = flush_sums())
                return st;
        sums.seg[sums.nseg++] = ds::GainSumK{s.grad_g, s.rows};
    }
    return flush_sums();
}

// ------------------------------------------------------------ row lengths --

ds_status run_norms(bool preserve, const ds_wseg *segs, int nseg, float eps, void *stream)
{
    g_last_error.clear();
    if (ds_status s = check_common(nseg, segs, eps, stream))
        return s;
    std::vector<Span> spans;
    for (int i = 0; i < nseg; ++i) {
        const ds_wseg &s = segs[i];
        if (ds_status st = check_shape(s.rows, s.cols, s.ld, i))
            return st;
        if (preserve && !(std::isfinite(s.radius) && s.radius > 0.f))
            return fail(DS_ERR_INVALID_ARG, where("radius must be finite and > 0", i));
        if (s.transposed || s.tgroup > 1)
            return fail(DS_ERR_INVALID_ARG, where("transposed rows are not supported here", i));
        if (s.tgroup < 0)
            return fail(DS_ERR_INVALID_ARG, where("tgroup must be 0 or 1 here", i));
        if (s.rows == 0)
            continue;
        if (ds_status st = check_matrix(s.w, s.rows, s.ld, 4, "w", i))
            return st;
        if (!s.rnorm)
            return fail(DS_ERR_INVALID_ARG, where("rnorm is NULL", i));
        if (!aligned(s.rnorm, 4))
            return fail(DS_ERR_ALIGNMENT, where("rnorm is not 4-byte aligned", i));
        spans.push_back(span_of(s.w, s.rows, s.cols, s.ld, 4, i, 0, -1));
        spans.push_back(span_of(s.rnorm, 1, s.rows, s.rows, 4, i, 1, -1));
    }
    if (ds_status st = check_overlaps(spans))
        return st;
    // rows that a CTA (or a cluster's slices) can stage take the staged
    // kernel, with the forward's row classes (it stages the same rows);
    // longer rows take the warp-per-row kernel
    const int forced = g_force_path.load(std::memory_order_relaxed);
    std::vector<RowClass> cls(static_cast<size_t>(nseg));
    std::vector<int64_t> staged_rows(static_cast<size_t>(nseg), 0);
    for (int i = 0; i < nseg; ++i) {
        cls[i] = classify(DS_OP_WN_FORWARD, segs[i].cols, forced);
        if (ds::is_staged(cls[i])) {
            cls[i].rps = tile_rows_per_slot(DS_OP_WN_FORWARD, slice_units(DS_OP_WN_FORWARD, segs[i].cols, cls[i]), 4,
                                            true, cls[i].slot);
            staged_rows[i] = segs[i].rows;
        }
    }
    auto make = [&](int i, int64_t r0, int64_t nr) {
        WSegK k = wseg_rows(segs[i], r0, nr, 4, 4);
        k.gain = nullptr;
        k.gy = nullptr;
        k.grad_w = nullptr;
        k.grad_g = nullptr;
        k.out = segs[i].rnorm + r0;
        k.radius = preserve ? segs[i].radius : 1.f;
        return k;
    };
    auto launch = [&](const RowClass &rc, const WParams &p, int64_t units, void *st) -> int {
        int used = 0;
        return ds::launch_tile(13, &p, units, rc.slot, rc.cluster, &used, st);
    };
    if (ds_status st = launch_all<WParams, WSegK>(nseg, staged_rows.data(), cls, eps, make, launch, stream))
        return st;
    static thread_local ds::RNParams params;
    int n = 0;
    int64_t units = 0;
    auto flush = [&]() -> ds_status {
        if (n == 0)
            return DS_OK;
        params.nseg = n;
        params.unit_start[n] = units;
        params.eps = eps;
        if (ds::launch_row_norms(params, sm_count(), stream) != 0)
            return fail(DS_ERR_CUDA, "kernel launch failed");
        g_launches.fetch_add(1, std::memory_order_relaxed);
        n = 0;
        units = 0;
        return DS_OK;
    };
    for (int i = 0; i < nseg; ++i) {
        const ds_wseg &s = segs[i];
        if (s.rows == 0 || staged_rows[i] != 0)
            continue;
        if (n == ds::kSegPerLaunch)
            if (ds_status st = flush())
                return st;
        params.seg[n] = ds::RNSegK{s.w, s.rnorm, s.rows, s.ld, static_cast<int32_t>(s.cols),
                                   preserve ? s.radius : 1.f};
        params.unit_start[n] = units;
        units += s.rows;
        ++n;
    }
    return flush();
}

ds_status run_act(bool slerp, const ds_aseg *segs, int nseg, float eps, void *stream)
{
    g_last_error.clear();
    if (ds_status s = check_common(nseg, segs, eps, stream))
        return s;
    std::vector<Span> spans;
    std::vector<int64_t> rows(static_cast<size_t>(nseg)), cols(static_cast<size_t>(nseg));
    for (int i = 0; i < nseg; ++i) {
        const ds_aseg &s = segs[i];
        if (ds_status st = check_shape(s.rows, s.cols, s.ld, i))
            return st;
        rows[i] = s.rows;
        cols[i] = s.cols;
        if (s.rows == 0)
            continue;
        if (ds_status st = check_matrix(s.x, s.rows, s.ld, 2, "x", i))
            return st;
        if (ds_status st = check_matrix(s.y, s.rows, s.ld, 2, "y", i))
            return st;
        if (slerp || s.r)
            if (ds_status st = check_matrix(s.r, s.rows, s.ld, 2, slerp ? "r (out)" : "r", i))
                return st;
        if (slerp) {
            if (!s.alpha)
                return fail(DS_ERR_INVALID_ARG, where("alpha is NULL", i));
            if (!aligned(s.alpha, 16))
                return fail(DS_ERR_ALIGNMENT, where("alpha is not 16-byte aligned", i));
            spans.push_back(span_of(s.alpha, 1, s.cols, s.cols, 4, i, 0, -1));
        }
        // y may be exactly x or exactly r (alias key = segment + 1)
        spans.push_back(span_of(s.x, s.rows, s.cols, s.ld, 2, i, 0, i));
        if (s.r)
            spans.push_back(span_of(s.r, s.rows, s.cols, s.ld, 2, i, 0, i));
        spans.push_back(span_of(s.y, s.rows, s.cols, s.ld, 2, i, 1, i));
    }
    if (ds_status st = check_overlaps(spans))
        return st;
    const ds_op op = slerp ? DS_OP_SLERP_ROWS : DS_OP_L2_ROWS;
    const int forced = g_force_path.load(std::memory_order_relaxed);
    std::vector<RowClass> cls(static_cast<size_t>(nseg));
    for (int i = 0; i < nseg; ++i) {
        cls[i] = classify(op, cols[i], forced);
        if (ds::is_staged(cls[i]))
            cls[i].rps = tile_rows_per_slot(op, slice_units(op, cols[i], cls[i]), 2, segs[i].r != nullptr,
                                            cls[i].slot);
    }
    auto make = [&](int i, int64_t r0, int64_t nr) { return aseg_rows(segs[i], r0, nr); };
    auto launch = [&](const RowClass &rc, const AParams &p, int64_t units, void *st) -> int {
        if (ds::is_staged(rc)) {
            int used = 0;
            return ds::launch_tile(slerp ? 6 : 5, &p, units, rc.slot, rc.cluster, &used, st);
        }
        return slerp ? ds::launch_slerp_rows(rc, p, units, st) : ds::launch_l2_rows(rc, p, units, st);
    };
    return launch_all<AParams, ASegK>(nseg, rows.data(), cls, eps, make, launch, stream);
}

ds_status run_fused(bool swiglu, const ds_fseg *segs, int nseg, float eps, void *stream)
{
    g_last_error.clear();
    if (ds_status s = check_common(nseg, segs, eps, stream))
        return s;
    const ds_op op = swiglu ? DS_OP_SWIGLU_L2_ROWS : DS_OP_GATE_L2_ROWS;
    const int forced = g_force_path.load(std::memory_order_relaxed);
    std::vector<Span> spans;
    std::vector<int64_t> rows(static_cast<size_t>(nseg)), cols(static_cast<size_t>(nseg));
    std::vector<RowClass> cls(static_cast<size_t>(nseg));
    for (int i = 0; i < nseg; ++i) {
        const ds_fseg &s = segs[i];
        if (ds_status st = check_shape(s.rows, s.cols, s.ld, i))
            return st;
        rows[i] = s.rows;
        cols[i] = s.cols;
        cls[i] = classify(op, s.cols, forced);
        if (cls[i].path == 0)
            return fail(DS_ERR_INVALID_ARG, where("row too long (more than 8 staged slices of 64 KB)", i));
        cls[i].rps = tile_rows_per_slot(op, slice_units(op, s.cols, cls[i]), 2, true, cls[i].slot);
        if (s.rows == 0)
            continue;
        if (ds_status st = check_matrix(s.a, s.rows, s.ld, 2, "a", i))
            return st;
        if (ds_status st = check_matrix(s.b, s.rows, s.ld, 2, "b", i))
            return st;
        if (ds_status st = check_matrix(s.y, s.rows, s.ld, 2, "y", i))
            return st;
        for (int k = 0; k < (swiglu ? 2 : 1); ++k) {
            const float *v = k == 0 ? s.sa : s.sb;
            if (!v)
                return fail(DS_ERR_INVALID_ARG, where(k == 0 ? "sa is NULL" : "sb is NULL", i));
            if (!aligned(v, 16))
                return fail(DS_ERR_ALIGNMENT, where(k == 0 ? "sa is not 16-byte aligned" : "sb is not 16-byte aligned", i));
            spans.push_back(span_of(v, 1, s.cols, s.cols, 4, i, 0, -1));
        }
        // y may be exactly a or exactly b (alias key = the segment)
        spans.push_back(span_of(s.a, s.rows, s.cols, s.ld, 2, i, 0, i));
        spans.push_back(span_of(s.b, s.rows, s.cols, s.ld, 2, i, 0, i));
        spans.push_back(span_of(s.y, s.rows, s.cols, s.ld, 2, i, 1, i));
    }
    if (ds_status st = check_overlaps(spans))
        return st;
    auto make = [&](int i, int64_t r0, int64_t nr) {
        const ds_fseg &s = segs[i];
        ASegK k{};
        k.x = s.a ? static_cast<const uint16_t *>(s.a) + r0 * s.ld : nullptr;
        k.r = s.b ? static_cast<const uint16_t *>(s.b) + r0 * s.ld : nullptr;
        k.y = s.y ? static_cast<uint16_t *>(s.y) + r0 * s.ld : nullptr;
        k.alpha = s.sa;
        k.s2 = swiglu ? s.sb : nullptr;
        k.rows = nr;
        k.ld = s.ld;
        k.cols = static_cast<int32_t>(s.cols);
        k.nu = static_cast<int32_t>((s.cols + 7) / 8);
        return k;
    };
    auto launch = [&](const RowClass &rc, const AParams &p, int64_t units, void *st) -> int {
        int used = 0;
        return ds::launch_tile(swiglu ? 12 : 11, &p, units, rc.slot, rc.cluster, &used, st);
    };
    return launch_all<AParams, ASegK>(nseg, rows.data(), cls, eps, make, launch, stream);
}

// ------------------------------------------------------- Dory's q/k rows --

bool qk_head_dim_ok(int32_t d)
{
    return d == 16 || d == 32 || d == 64 || d == 128 || d == 256 || d == 512;
}

ds_status run_qk(const ds_qkseg *segs, int nseg, float eps, void *stream)
{
    g_last_error.clear();
    if (ds_status s = check_common(nseg, segs, eps, stream))
        return s;
    std::vector<Span> spans;
    std::vector<int32_t> rb(static_cast<size_t>(nseg), 1);
    for (int i = 0; i < nseg; ++i) {
        const ds_qkseg &s = segs[i];
        const int32_t D = s.head_dim;
        if (s.rows < 0 || s.rows > (int64_t(1) << 40))
            return fail(DS_ERR_INVALID_ARG, where("rows outside [0, 2^40]", i));
        if (!qk_head_dim_ok(D))
            return fail(DS_ERR_INVALID_ARG, where("head_dim must be 16, 32, 64, 128, 256 or 512", i));
        if (s.hq < 0 || s.hk < 0 || s.hq + s.hk < 1 || s.hq > 4096 || s.hk > 4096)
            return fail(DS_ERR_INVALID_ARG, where("hq, hk must be in [0, 4096] with hq + hk >= 1", i));
        if (s.v && s.hk == 0)
            return fail(DS_ERR_INVALID_ARG, where("v needs hk >= 1", i));
        const int hw = 32 / (D / 16);
        const int tpr = (s.hq + hw - 1) / hw + (s.hk + hw - 1) / hw * (s.v ? 2 : 1);
        // rows per block iteration: as many as give each warp kQkTasks tasks
        rb[i] = std::max(1, std::min(ds::kQkWarps * ds::kQkTasks / tpr, ds::kQkTable / (D / 2)));
        if (s.rows == 0)
            continue;
        const int64_t wq = int64_t(s.hq) * D, wk = int64_t(s.hk) * D;
        if (!s.pos)
            return fail(DS_ERR_INVALID_ARG, where("pos is NULL", i));
        if (!s.inv_freq)
            return fail(DS_ERR_INVALID_ARG, where("inv_freq is NULL", i));
        if (!aligned(s.pos, 4) || !aligned(s.inv_freq, 4) || (s.slot && !aligned(s.slot, 4)))
            return fail(DS_ERR_ALIGNMENT, where("pos, slot and inv_freq must be 4-byte aligned", i));
        spans.push_back(span_of(s.pos, 1, s.rows, s.rows, 4, i, 0, -1));
        spans.push_back(span_of(s.inv_freq, 1, D / 2, D / 2, 4, i, 0, -1));
        if (s.slot)
            spans.push_back(span_of(s.slot, 1, s.rows, s.rows, 4, i, 0, -1));
        if (s.hq > 0) {
            if (s.ld_q < wq || s.ld_q > (int64_t(1) << 40))
                return fail(DS_ERR_INVALID_ARG, where("ld_q below hq * head_dim (or too large)", i));
            if (ds_status st = check_matrix(s.q, s.rows, s.ld_q, 2, "q", i))
                return st;
            if (ds_status st = check_matrix(s.q_out, s.rows, s.ld_q, 2, "q_out", i))
                return st;
            if (s.q_scale) {
                if (!aligned(s.q_scale, 16))
                    return fail(DS_ERR_ALIGNMENT, where("q_scale is not 16-byte aligned", i));
                spans.push_back(span_of(s.q_scale, 1, wq, wq, 4, i, 0, -1));
            }
            spans.push_back(span_of(s.q, s.rows, wq, s.ld_q, 2, i, 0, 3 * i));
            spans.push_back(span_of(s.q_out, s.rows, wq, s.ld_q, 2, i, 1, 3 * i));
        }
        if (s.hk > 0) {
            if (s.ld_kv < wk || s.ld_kv > (int64_t(1) << 40) || s.ld_cache < wk || s.ld_cache > (int64_t(1) << 40))
                return fail(DS_ERR_INVALID_ARG, where("ld_kv or ld_cache below hk * head_dim (or too large)", i));
            if (s.cache_rows < 1 || s.cache_rows > (int64_t(1) << 40) || (!s.slot && s.cache_rows < s.rows))
                return fail(DS_ERR_INVALID_ARG, where("cache_rows below rows (no slot) or outside [1, 2^40]", i));
            if (ds_status st = check_matrix(s.k, s.rows, s.ld_kv, 2, "k", i))
                return st;
            if (ds_status st = check_matrix(s.k_cache, s.cache_rows, s.ld_cache, 2, "k_cache", i))
                return st;
            // in place only row for row (no slots) over the same matrix
            const int key_k = s.slot ? -1 : 3 * i + 1, key_v = s.slot ? -1 : 3 * i + 2;
            spans.push_back(span_of(s.k, s.rows, wk, s.ld_kv, 2, i, 0, key_k));
            spans.push_back(span_of(s.k_cache, s.cache_rows, wk, s.ld_cache, 2, i, 1, key_k));
            if (s.v) {
                if (ds_status st = check_matrix(s.v, s.rows, s.ld_kv, 2, "v", i))
                    return st;
                if (ds_status st = check_matrix(s.v_cache, s.cache_rows, s.ld_cache, 2, "v_cache", i))
                    return st;
                spans.push_back(span_of(s.v, s.rows, wk, s.ld_kv, 2, i, 0, key_v));
                spans.push_back(span_of(s.v_cache, s.cache_rows, wk, s.ld_cache, 2, i, 1, key_v));
            }
        }
    }
    if (ds_status st = check_overlaps(spans))
        return st;

    static thread_local ds::QKParams params; // ~20 KB: kept off the stack
    // one launch per head size present
    for (int pass = 0; pass < 6; ++pass) {
        const int32_t head_dim = 16 << pass;
        int n = 0;
        int64_t units = 0;
        auto flush = [&]() -> ds_status {
            if (n == 0)
                return DS_OK;
            params.nseg = n;
            params.unit_start[n] = units;
            params.eps = eps;
            const int grid = static_cast<int>(std::min<int64_t>(int64_t(sm_count()) * 3, units));
            const int e = ds::launch_qk(params, grid, stream);
            if (e != 0) {
                char buf[160];
                std::snprintf(buf, sizeof(buf), "kernel launch failed (cudaError %d)", e);
                return fail(DS_ERR_CUDA, buf);
            }
            g_launches.fetch_add(1, std::memory_order_relaxed);
            n = 0;
            units = 0;
            return DS_OK;
        };
        for (int i = 0; i < nseg; ++i) {
            const ds_qkseg &s = segs[i];
            if (s.rows == 0 || s.head_dim != head_dim)
                continue;
            if (n == ds::kSegPerLaunch)
                if (ds_status st = flush())
                    return st;
            ds::QKSegK &k = params.seg[n];
            k = ds::QKSegK{};
            k.q = static_cast<const uint16_t *>(s.q);
            k.k = static_cast<const uint16_t *>(s.k);
            k.v = static_cast<const uint16_t *>(s.v);
            k.q_out = static_cast<uint16_t *>(s.q_out);
            k.k_cache = static_cast<uint16_t *>(s.k_cache);
            k.v_cache = s.v ? static_cast<uint16_t *>(s.v_cache) : nullptr;
            k.pos = s.pos;
            k.slot = s.slot;
            k.inv = s.inv_freq;
            k.q_scale = s.hq > 0 ? s.q_scale : nullptr;
            k.rows = s.rows;
            k.cache_rows = s.cache_rows;
            k.ld_q = s.ld_q;
            k.ld_kv = s.ld_kv;
            k.ld_cache = s.ld_cache;
            k.D = s.head_dim;
            k.hq = s.hq;
            k.hk = s.hk;
            k.rb = rb[i];
            params.unit_start[n] = units;
            units += (s.rows + rb[i] - 1) / rb[i];
            ++n;
        }
        if (ds_status st = flush())
            return st;
    }
    return DS_OK;
}

AGSegK agseg_rows(const ds_agseg &s, int64_t r0, int64_t nr)
{
    AGSegK k{};
    k.x = s.x ? static_cast<const uint16_t *>(s.x) + r0 * s.ld : nullptr;
    k.r = s.r ? static_cast<const uint16_t *>(s.r) + r0 * s.ld : nullptr;
    k.dy = s.dy ? static_cast<const uint16_t *>(s.dy) + r0 * s.ld : nullptr;
    k.dx = s.dx ? s.dx + r0 * s.ld_d : nullptr;
    k.dr = s.dr ? s.dr + r0 * s.ld_d : nullptr;
    k.alpha = s.alpha;
    k.rows = nr;
    k.ld = s.ld;
    k.ld_d = s.ld_d;
    k.cols = static_cast<int32_t>(s.cols);
    k.nu = static_cast<int32_t>((s.cols + 7) / 8);
    return k;
}

// Floats per dalpha workspace line: the row's octets, 8 floats each.
int64_t dalpha_ws_ld(int64_t cols) { return (cols + 7) / 8 * 8; }

uint64_t dalpha_ws_bytes(int64_t cols)
{
    return static_cast<uint64_t>(sm_count()) * ds::kTileMaxGroups * static_cast<uint64_t>(dalpha_ws_ld(cols)) * 4u;
}

ds_status run_act_bwd(bool slerp, const ds_agseg *segs, int nseg, float eps, float *dalpha, void *ws,
                      uint64_t ws_bytes, void *stream)
{
    g_last_error.clear();
    if (ds_status s = check_common(nseg, segs, eps, stream))
        return s;
    const ds_op op = slerp ? DS_OP_SLERP_ROWS_BACKWARD : DS_OP_L2_ROWS_BACKWARD;
    const int forced = g_force_path.load(std::memory_order_relaxed);
    std::vector<Span> spans;
    std::vector<int64_t> rows(static_cast<size_t>(nseg)), cols(static_cast<size_t>(nseg));
    std::vector<RowClass> cls(static_cast<size_t>(nseg));
    int64_t total_rows = 0;
    for (int i = 0; i < nseg; ++i) {
        const ds_agseg &s = segs[i];
        if (ds_status st = check_shape(s.rows, s.cols, s.ld, i))
            return st;
        if (s.ld_d < s.cols)
            return fail(DS_ERR_INVALID_ARG, where("ld_d < cols", i));
        rows[i] = s.rows;
        cols[i] = s.cols;
        cls[i] = classify(op, s.cols, forced, slerp || s.r != nullptr);
        if (cls[i].path == 0)
            return fail(DS_ERR_INVALID_ARG, where("row too long for the backward (more than 8 staged slices of 64 KB)", i));
        if (s.rows == 0)
            continue;
        total_rows += s.rows;
        if (ds_status st = check_matrix(s.x, s.rows, s.ld, 2, slerp ? "x (res)" : "x", i))
            return st;
        if (ds_status st = check_matrix(s.dy, s.rows, s.ld, 2, "dy", i))
            return st;
        if (ds_status st = check_matrix(s.dx, s.rows, s.ld_d, 4, "dx", i))
            return st;
        if (slerp || s.r)
            if (ds_status st = check_matrix(s.r, s.rows, s.ld, 2, slerp ? "r (out)" : "r", i))
                return st;
        spans.push_back(span_of(s.x, s.rows, s.cols, s.ld, 2, i, 0, -1));
        if (s.r)
            spans.push_back(span_of(s.r, s.rows, s.cols, s.ld, 2, i, 0, -1));
        spans.push_back(span_of(s.dy, s.rows, s.cols, s.ld, 2, i, 0, -1));
        spans.push_back(span_of(s.dx, s.rows, s.cols, s.ld_d, 4, i, 1, -1));
        if (slerp) {
            if (ds_status st = check_matrix(s.dr, s.rows, s.ld_d, 4, "dr", i))
                return st;
            if (!s.alpha)
                return fail(DS_ERR_INVALID_ARG, where("alpha is NULL", i));
            if (!aligned(s.alpha, 16))
                return fail(DS_ERR_ALIGNMENT, where("alpha is not 16-byte aligned", i));
            spans.push_back(span_of(s.alpha, 1, s.cols, s.cols, 4, i, 0, -1));
            spans.push_back(span_of(s.dr, s.rows, s.cols, s.ld_d, 4, i, 1, -1));
        }
    }
    int64_t dcols = 0;
    if (slerp && dalpha) {
        // every segment shares alpha and cols, one launch covers them all
        for (int i = 0; i < nseg; ++i)
            if (segs[i].alpha != segs[0].alpha || segs[i].cols != segs[0].cols || !ds::same_launch(cls[i], cls[0]))
                return fail(DS_ERR_INVALID_ARG, where("dalpha needs one alpha, one cols and one row class", i));
        if (nseg > ds::kSegPerLaunch)
            return fail(DS_ERR_INVALID_ARG, "dalpha: at most 128 segments");
        dcols = nseg ? segs[0].cols : 0;
        if (dcols > 0) {
            if (!aligned(dalpha, 4))
                return fail(DS_ERR_ALIGNMENT, "dalpha is not 4-byte aligned");
            if (!ws || !aligned(ws, 256))
                return fail(ws ? DS_ERR_ALIGNMENT : DS_ERR_INVALID_ARG, "workspace NULL or not 256-byte aligned");
            if (ws_bytes < dalpha_ws_bytes(dcols))
                return fail(DS_ERR_INVALID_ARG, "workspace smaller than ds_slerp_rows_backward_workspace(cols)");
            spans.push_back(span_of(dalpha, 1, dcols, dcols, 4, -2, 1, -1));
            spans.push_back({reinterpret_cast<uintptr_t>(ws), reinterpret_cast<uintptr_t>(ws) + ws_bytes, -3, 1, -1});
        }
    }
    if (ds_status st = check_overlaps(spans))
        return st;
    for (int i = 0; i < nseg; ++i)
        cls[i].rps = tile_rows_per_slot(op, slice_units(op, cols[i], cls[i]), 2, segs[i].r != nullptr,
                                        cls[i].slot);
    const int tag = slerp ? 10 : 9;
    int grid_used = 0, groups_used = 0;
    int64_t units_used = 0;
    auto make = [&](int i, int64_t r0, int64_t nr) { return agseg_rows(segs[i], r0, nr); };
    auto launch = [&](const RowClass &rc, const GParams &p, int64_t units, void *st) -> int {
        groups_used = ds::tile_groups(tag, rc.slot);
        units_used = units;
        return ds::launch_tile(tag, &p, units, rc.slot, rc.cluster, &grid_used, st);
    };
    const bool want_dalpha = slerp && dalpha && dcols > 0;
    auto prep = [&](GParams &p) {
        if (want_dalpha) {
            p.ws = static_cast<float *>(ws);
            p.ws_ld = static_cast<int32_t>(dalpha_ws_ld(dcols));
        }
    };
    const uint64_t before = g_launches.load(std::memory_order_relaxed);
    if (ds_status st = launch_all<GParams, AGSegK>(nseg, rows.data(), cls, eps, make, launch, stream, prep))
        return st;
    if (want_dalpha) {
        if (g_launches.load(std::memory_order_relaxed) - before > 1)
            return fail(DS_ERR_INVALID_ARG, "dalpha: the rows need more than one launch");
        if (total_rows == 0) {
            // no rows: dalpha is zero
            const cudaError_t e = cudaMemsetAsync(dalpha, 0, static_cast<size_t>(dcols) * 4,
                                                  static_cast<cudaStream_t>(stream));
            if (e != cudaSuccess)
                return fail(DS_ERR_CUDA, "cudaMemsetAsync failed");
            return DS_OK;
        }
        const int e = ds::launch_dalpha_reduce(static_cast<const float *>(ws), static_cast<int>(dalpha_ws_ld(dcols)),
                                              grid_used, groups_used, units_used, static_cast<int>(dcols), dalpha,
                                              stream);
        if (e != 0)
            return fail(DS_ERR_CUDA, "dalpha reduction launch failed");
        g_launches.fetch_add(1, std::memory_order_relaxed);
    }
    return DS_OK;
}

} // namespace

extern "C" {

ds_status ds_wn_forward(const ds_wseg *segs, int nseg, ds_dtype out_dtype, float eps, ds_stream stream)
{
    return run_weight(W_FWD, segs, nseg, out_dtype, eps, stream);
}

ds_status ds_wn_backward(const ds_wseg *segs, int nseg, ds_dtype gy_dtype, float eps, ds_stream stream)
{
    return run_weight(W_BWD, segs, nseg, gy_dtype, eps, stream);
}

ds_status ds_row_renorm(const ds_wseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_weight(W_RENORM, segs, nseg, DS_F32, eps, stream);
}

ds_status ds_grad_project(const ds_wseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_weight(W_PROJECT, segs, nseg, DS_F32, eps, stream);
}

ds_status ds_renorm_momentum(const ds_wseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_weight(W_MOMENTUM, segs, nseg, DS_F32, eps, stream);
}

ds_status ds_gate_l2_rows(const ds_fseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_fused(false, segs, nseg, eps, stream);
}

ds_status ds_swiglu_l2_rows(const ds_fseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_fused(true, segs, nseg, eps, stream);
}

ds_status ds_row_norms(const ds_wseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_norms(false, segs, nseg, eps, stream);
}

ds_status ds_gain_preserve(const ds_wseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_norms(true, segs, nseg, eps, stream);
}

ds_status ds_qk_rows_l2(const ds_qkseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_qk(segs, nseg, eps, stream);
}

ds_status ds_l2_rows_backward(const ds_agseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_act_bwd(false, segs, nseg, eps, nullptr, nullptr, 0, stream);
}

ds_status ds_slerp_rows_backward(const ds_agseg *segs, int nseg, float eps, float *dalpha, void *workspace,
                                 uint64_t workspace_bytes, ds_stream stream)
{
    return run_act_bwd(true, segs, nseg, eps, dalpha, workspace, workspace_bytes, stream);
}

ds_status ds_slerp_rows_backward_noalloc(const ds_agseg *segs, int nseg, float eps, float *dalpha, ds_stream stream)
{
    void *ws = nullptr;
    uint64_t bytes = 0;
    if (dalpha) {
        g_last_error.clear();
        if (nseg > 0 && segs && segs[0].cols >= 1 && segs[0].cols <= kMaxCols &&
            dalpha_ws_bytes(segs[0].cols) > static_cast<uint64_t>(ds::kBuiltinScratchFloats) * 4u) {
            char buf[200];
            std::snprintf(buf, sizeof(buf),
                          "rows of %lld columns need %llu bytes of dalpha scratch; the built-in scratch holds %llu "
                          "(use ds_slerp_rows_backward with a workspace)",
                          static_cast<long long>(segs[0].cols),
                          static_cast<unsigned long long>(dalpha_ws_bytes(segs[0].cols)),
                          static_cast<unsigned long long>(ds::kBuiltinScratchFloats) * 4u);
            return fail(DS_ERR_INVALID_ARG, buf);
        }
        if (const int e = ds::builtin_scratch(&ws, &bytes)) {
            char buf[96];
            std::snprintf(buf, sizeof(buf), "built-in scratch address lookup failed (cudaError %d)", e);
            return fail(DS_ERR_CUDA, buf);
        }
    }
    return run_act_bwd(true, segs, nseg, eps, dalpha, ws, bytes, stream);
}

uint64_t ds_slerp_rows_backward_workspace(int64_t cols)
{
    if (cols < 1 || cols > kMaxCols)
        return 0;
    return dalpha_ws_bytes(cols);
}

ds_status ds_l2_rows(const ds_aseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_act(false, segs, nseg, eps, stream);
}

ds_status ds_slerp_rows(const ds_aseg *segs, int nseg, float eps, ds_stream stream)
{
    return run_act(true, segs, nseg, eps, stream);
}

const char *ds_status_string(ds_status status)
{
    switch (status) {
    case DS_OK: return "ok";
    case DS_ERR_INVALID_ARG: return "invalid argument";
    case DS_ERR_ALIGNMENT: return "row start not 16-byte aligned";
    case DS_ERR_UNSUPPORTED_DTYPE: return "unsupported dtype";
    case DS_ERR_TOO_MANY_SEGMENTS: return "too many segments";
    case DS_ERR_CUDA: return "CUDA error";
    case DS_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case DS_ERR_OVERLAP: return "output overlaps another buffer";
    }
    return "unknown status";
}

const char *ds_last_error(void) { return g_last_error.c_str(); }

ds_status ds_get_device_status(ds_stream stream)
{
    uint32_t code = 0, site = 0;
    const int e = ds::read_and_clear_device_error(&code, &site, stream);
    if (e != 0) {
        char buf[96];
        std::snprintf(buf, sizeof(buf), "device status read failed (cudaError %d)", e);
        return fail(DS_ERR_CUDA, buf);
    }
    if (code == 0)
        return DS_OK;
    char buf[96];
    std::snprintf(buf, sizeof(buf), "device error %u at site %u", code, site);
    // codes the kernels record: a wait that ran out, an argument only the
    // device could check (a cache slot out of range)
    const bool known = code == DS_ERR_DEVICE_TIMEOUT || code == DS_ERR_INVALID_ARG;
    return fail(known ? static_cast<ds_status>(code) : DS_ERR_CUDA, buf);
}

uint64_t ds_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int ds_version(void) { return 100; }

ds_status ds_row_class(ds_op op, int64_t cols, int *path, int *group_threads, int *cluster_ctas)
{
    if (op < DS_OP_WN_FORWARD || op > DS_OP_SWIGLU_L2_ROWS)
        return fail(DS_ERR_INVALID_ARG, "unknown op");
    if (cols < 1 || cols > kMaxCols)
        return fail(DS_ERR_INVALID_ARG, "cols outside [1, 2^31 - 1]");
    const RowClass rc = classify(op, cols, g_force_path.load(std::memory_order_relaxed));
    if (rc.path == 0)
        return fail(DS_ERR_INVALID_ARG, "row too long for this operation (more than 8 staged slices of 64 KB)");
    if (path)
        *path = rc.path;
    if (group_threads)
        *group_threads = rc.group;
    if (cluster_ctas)
        *cluster_ctas = rc.cluster;
    return DS_OK;
}

ds_status ds_debug_force_path(ds_path path)
{
    if (path < DS_PATH_AUTO || path > DS_PATH_TWO_PASS)
        return fail(DS_ERR_INVALID_ARG, "unknown path");
    g_force_path.store(path, std::memory_order_relaxed);
    return DS_OK;
}

ds_status ds_debug_set_wait_limit_ns(uint64_t limit_ns)
{
    g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
    return DS_OK;
}

ds_status ds_debug_wait_timeout_selftest(uint64_t limit_ns, ds_stream stream)
{
    if (limit_ns > 10ull * 1000 * 1000 * 1000)
        return fail(DS_ERR_INVALID_ARG, "limit above 10 s");
    const int e = ds::launch_wait_selftest(limit_ns, stream);
    if (e != 0)
        return fail(DS_ERR_CUDA, "self-test launch failed");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return DS_OK;
}

ds_status ds_debug_division_check(uint64_t *counts, ds_stream stream)
{
    if (!counts)
        return fail(DS_ERR_INVALID_ARG, "counts is NULL");
    if (reinterpret_cast<uintptr_t>(counts) % 8)
        return fail(DS_ERR_ALIGNMENT, "counts must be 8-byte aligned");
    const int e = ds::launch_division_check(reinterpret_cast<unsigned long long *>(counts), stream);
    if (e != 0)
        return fail(DS_ERR_CUDA, "division check launch failed");
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return DS_OK;
}

} // extern "C"
