// ds_qk.cu -- Dory's q and k rows on sm_100a (TensorFold PR #1260,
// tf_qk_rows_l2): rotate-half RoPE on the bf16 q and k heads at the fp32
// angle pos * inv (the tern-tc listing's rope_cache / apply_rope: fp32
// products, cast back to bf16), each head's L2 norm with eps on the sum, q
// times an fp32 scale vector after the normalized head's rounding; k goes to
// its cache row, v is copied to its cache row as is.
//
// Layout.  One head of D bf16 columns is held by L = D/16 lanes: lane j holds
// octet j of the first half (columns 8j..8j+7) and octet j of the second half
// (D/2 + 8j..), so each pair (x_i, x_{i+D/2}) the rotation mixes sits in one
// lane and needs no shuffle.  A warp takes 32/L heads at once (two heads of
// 256).  A block iteration takes `rb` consecutive rows: their cos and sin
// (one per row and pair index, shared by every head of the row) are computed
// once into shared memory while the warps' loads of the rows' heads are in
// flight; the heads are split into warp tasks (a group of 32/L heads of q, k
// or v of one row) dealt round-robin to the 8 warps, up to kQkTasks held in
// registers at once.  Every access is a 16-byte vector.  (Staging the rows
// through shared memory by bulk copies, two iterations ahead, measured
// slower on B200: 121 against 113 us for 16,384 of Dory's rows.)
#include <cuda_runtime.h>

#include "ds_device.cuh"

namespace ds {

namespace {

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 lo2(uint32_t w) { return f2(bf_lo(w), bf_hi(w)); }
__device__ __forceinline__ uint32_t pk(float2 v) { return pack_bf2(v.x, v.y); }
__device__ __forceinline__ uint32_t word4(const uint4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }
__device__ __forceinline__ float2 neg2(float2 v) { return f2(-v.x, -v.y); }

// Reductions over the L lanes of one head (L a power of two; the groups are
// aligned, so xor offsets below L stay inside the head).  `any` is
// warp-wide: the rescale branch of row_scale stays uniform in the warp.
template <int L>
struct HeadRed {
    __device__ __forceinline__ bool any(bool b) const { return __any_sync(0xffffffffu, b); }
    __device__ __forceinline__ float max(float v) const
    {
#pragma unroll
        for (int o = L >> 1; o > 0; o >>= 1)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        return v;
    }
    template <int N>
    __device__ __forceinline__ void sum(float (&v)[N]) const
    {
#pragma unroll
        for (int o = L >> 1; o > 0; o >>= 1)
#pragma unroll
            for (int i = 0; i < N; ++i)
                v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
    }
};

// bf16(v * pre * inv) for the 8 values of an octet (pre = 1 on all but the
// rescaled rows of subnormals, see row_scale).
__device__ __forceinline__ uint4 scale_octet(uint4 v, RowScale rs)
{
    const float2 s = f2(rs.inv, rs.inv);
    uint32_t w[4];
    if (rs.pre == 1.f) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = pk(__fmul2_rn(lo2(word4(v, i)), s));
    } else {
        const float2 p = f2(rs.pre, rs.pre);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = pk(__fmul2_rn(__fmul2_rn(lo2(word4(v, i)), p), s));
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// bf16(y_j * scale_j) for an octet of q's normalized head.
__device__ __forceinline__ uint4 q_scale_octet(uint4 y, const float *sc)
{
    const float4 a = ld16_cached(sc), b = ld16_cached(sc + 4);
    return make_uint4(pk(__fmul2_rn(lo2(y.x), f2(a.x, a.y))), pk(__fmul2_rn(lo2(y.y), f2(a.z, a.w))),
                      pk(__fmul2_rn(lo2(y.z), f2(b.x, b.y))), pk(__fmul2_rn(lo2(y.w), f2(b.z, b.w))));
}

// One warp task: a group of 32/L heads of q, k or v of one row of the block
// iteration.  Tasks are numbered row by row (tpr per row: q groups, k
// groups, v groups), and a warp walks its tasks t = warp, warp + 8, ...
// keeping (row, index within the row) incrementally.
struct TaskWalk {
    int rib, tr;
    __device__ __forceinline__ void start(int t, int tpr)
    {
        rib = t / tpr;
        tr = t - rib * tpr;
    }
    __device__ __forceinline__ void step(int tpr)
    {
        tr += kQkWarps;
        while (tr >= tpr) {
            tr -= tpr;
            ++rib;
        }
    }
};

struct Task {
    int kind; // 0 q, 1 k, 2 v
    int head; // this lane's head
    bool valid;
};

template <int D>
__device__ __forceinline__ Task task_of(const QKSegK &sg, int tr, int nq, int nk, int lane_head, bool row_ok)
{
    constexpr int hw = 32 / (D / 16);
    Task k;
    int group, H;
    if (tr < nq) {
        k.kind = 0;
        group = tr;
        H = sg.hq;
    } else if (tr < nq + nk) {
        k.kind = 1;
        group = tr - nq;
        H = sg.hk;
    } else {
        k.kind = 2;
        group = tr - nq - nk;
        H = sg.hk;
    }
    k.head = group * hw + lane_head;
    k.valid = row_ok && k.head < H;
    return k;
}

// Everything of one warp task after its two octets (this lane's first-half
// and second-half columns) are in registers: the v copy, or the rotation,
// the head's norm and the stores.  Uniform in the warp up to `tk.valid` (the
// head reduction and row_scale's vote need every lane).
template <int D>
__device__ __forceinline__ void qk_task(const QKSegK &sg, const Task &tk, int rib, uint4 xa, uint4 xb, int64_t row0,
                                        const float *s_cos, const float *s_sin, int j, float eps)
{
    constexpr int H2 = D / 2, L = D / 16;
    const int64_t row = row0 + rib;
    int64_t dst = row;
    if (tk.kind != 0 && tk.valid && sg.slot) {
        dst = sg.slot[row];
        if (dst < 0 || dst >= sg.cache_rows) {
            raise_device_error(DS_ERR_INVALID_ARG, kSiteQkSlot);
            dst = -1;
        }
    }
    const bool store = tk.valid && dst >= 0;
    const int64_t col = static_cast<int64_t>(tk.head) * D + 8 * j;
    if (tk.kind == 2) { // v: as is
        if (store) {
            uint16_t *o = sg.v_cache + dst * sg.ld_cache + col;
            st16(o, xa);
            st16(o + H2, xb);
        }
        return;
    }
    // rotate-half: (x_i cos - x_{i+h} sin, x_i sin + x_{i+h} cos) as
    // separate fp32 products and one fp32 add, then bf16
    const float *cs = s_cos + rib * H2 + 8 * j, *sn = s_sin + rib * H2 + 8 * j;
    const float4 c0 = *reinterpret_cast<const float4 *>(cs), c1 = *reinterpret_cast<const float4 *>(cs + 4);
    const float4 n0 = *reinterpret_cast<const float4 *>(sn), n1 = *reinterpret_cast<const float4 *>(sn + 4);
    const float2 cc[4] = {f2(c0.x, c0.y), f2(c0.z, c0.w), f2(c1.x, c1.y), f2(c1.z, c1.w)};
    const float2 ss[4] = {f2(n0.x, n0.y), f2(n0.z, n0.w), f2(n1.x, n1.y), f2(n1.z, n1.w)};
    uint32_t w1[4], w2[4];
    float2 acc = f2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = lo2(word4(xa, i)), b = lo2(word4(xb, i));
        w1[i] = pk(__fadd2_rn(__fmul2_rn(a, cc[i]), neg2(__fmul2_rn(b, ss[i]))));
        w2[i] = pk(__fadd2_rn(__fmul2_rn(a, ss[i]), __fmul2_rn(b, cc[i])));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = lo2(w1[i]);
        acc = __ffma2_rn(v, v, acc);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = lo2(w2[i]);
        acc = __ffma2_rn(v, v, acc);
    }
    const HeadRed<L> red;
    float S[1] = {acc.x + acc.y};
    red.sum(S);
    const RowScale rs = row_scale(S[0], eps, red, [&](auto f) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 v = lo2(w1[i]);
            f(v.x);
            f(v.y);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 v = lo2(w2[i]);
            f(v.x);
            f(v.y);
        }
    });
    uint4 y1 = scale_octet(make_uint4(w1[0], w1[1], w1[2], w1[3]), rs);
    uint4 y2 = scale_octet(make_uint4(w2[0], w2[1], w2[2], w2[3]), rs);
    if (!store)
        return;
    if (tk.kind == 0) {
        if (sg.q_scale) {
            y1 = q_scale_octet(y1, sg.q_scale + col);
            y2 = q_scale_octet(y2, sg.q_scale + col + H2);
        }
        uint16_t *o = sg.q_out + row * sg.ld_q + col;
        st16(o, y1);
        st16(o + H2, y2);
    } else {
        uint16_t *o = sg.k_cache + dst * sg.ld_cache + col;
        st16(o, y1);
        st16(o + H2, y2);
    }
}

// cos and sin of the fp32 angle fp32(pos) * inv_i for rows row0.. of an
// iteration (every thread of the block takes a share; one range reduction
// for both).
template <int D>
__device__ __forceinline__ void qk_table(const QKSegK &sg, int64_t row0, int nrows_blk, float *s_cos, float *s_sin)
{
    constexpr int H2 = D / 2;
    for (int e = threadIdx.x; e < sg.rb * H2; e += kQkThreads) {
        const int r = e / H2, i = e % H2;
        if (r < nrows_blk) {
            const float th = __fmul_rn(__int2float_rn(sg.pos[row0 + r]), __ldg(sg.inv + i));
            sincosf(th, &s_sin[e], &s_cos[e]);
        }
    }
}

struct IterGeom {
    int seg;
    int64_t row0;
    int nrows_blk, nq, nk, tpr, ntask;
};

template <int D>
__device__ __forceinline__ IterGeom iter_geom(const QKParams &p, int64_t u)
{
    constexpr int hw = 32 / (D / 16);
    IterGeom g;
    g.seg = find_segment(p, u);
    const QKSegK &sg = p.seg[g.seg];
    g.row0 = (u - p.unit_start[g.seg]) * sg.rb;
    g.nrows_blk = sg.rows - g.row0 < sg.rb ? static_cast<int>(sg.rows - g.row0) : sg.rb;
    g.nq = (sg.hq + hw - 1) / hw;
    g.nk = (sg.hk + hw - 1) / hw;
    g.tpr = g.nq + g.nk + (sg.v ? g.nk : 0);
    g.ntask = sg.rb * g.tpr;
    return g;
}

// A block iteration's warps load their tasks' octets straight from global
// memory (up to kQkTasks per warp at once) while the table is computed.
// The table is double-buffered: iteration k writes buffer k % 2, whose last
// readers (iteration k - 2) all passed iteration k - 1's barrier, so one
// barrier per iteration (table written) is enough.
template <int D>
__global__ void __launch_bounds__(kQkThreads, 3) k_qk(const __grid_constant__ QKParams p)
{
    constexpr int H2 = D / 2, L = D / 16;
    __shared__ __align__(16) float s_cos2[2][kQkTable];
    __shared__ __align__(16) float s_sin2[2][kQkTable];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = lane & (L - 1), lane_head = lane / L;
    const int64_t total = p.unit_start[p.nseg];

    int parity = 0;
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x, parity ^= 1) {
        const IterGeom g = iter_geom<D>(p, u);
        const QKSegK &sg = p.seg[g.seg];
        float *s_cos = s_cos2[parity], *s_sin = s_sin2[parity];
        for (int base = 0; base < g.ntask; base += kQkWarps * kQkTasks) {
            uint4 xa[kQkTasks], xb[kQkTasks];
            TaskWalk wk;
            wk.start(base + warp, g.tpr);
            TaskWalk w0 = wk;
#pragma unroll
            for (int m = 0; m < kQkTasks; ++m) {
                xa[m] = xb[m] = make_uint4(0, 0, 0, 0);
                if (base + warp + kQkWarps * m < g.ntask) {
                    const Task tk = task_of<D>(sg, wk.tr, g.nq, g.nk, lane_head, wk.rib < g.nrows_blk);
                    if (tk.valid) {
                        const int64_t row = g.row0 + wk.rib;
                        const uint16_t *src = tk.kind == 0 ? sg.q + row * sg.ld_q
                                              : tk.kind == 1 ? sg.k + row * sg.ld_kv
                                                             : sg.v + row * sg.ld_kv;
                        src += static_cast<int64_t>(tk.head) * D + 8 * j;
                        xa[m] = ld16(src);
                        xb[m] = ld16(src + H2);
                    }
                }
                wk.step(g.tpr);
            }
            if (base == 0) { // while the loads above are in flight
                qk_table<D>(sg, g.row0, g.nrows_blk, s_cos, s_sin);
                __syncthreads();
            }
#pragma unroll
            for (int m = 0; m < kQkTasks; ++m) {
                if (base + warp + kQkWarps * m >= g.ntask) // uniform in the warp
                    break;
                const Task tk = task_of<D>(sg, w0.tr, g.nq, g.nk, lane_head, w0.rib < g.nrows_blk);
                qk_task<D>(sg, tk, w0.rib, xa[m], xb[m], g.row0, s_cos, s_sin, j, p.eps);
                w0.step(g.tpr);
            }
        }
    }
}

template <int D>
cudaError_t launch_qk_d(const QKParams &p, int grid, cudaStream_t st)
{
    k_qk<D><<<grid, kQkThreads, 0, st>>>(p);
    return cudaGetLastError();
}

} // namespace

int launch_qk(const QKParams &p, int grid, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (p.seg[0].D) { // every segment of a launch has the same head size
    case 16: return launch_qk_d<16>(p, grid, st);
    case 32: return launch_qk_d<32>(p, grid, st);
    case 64: return launch_qk_d<64>(p, grid, st);
    case 128: return launch_qk_d<128>(p, grid, st);
    case 256: return launch_qk_d<256>(p, grid, st);
    case 512: return launch_qk_d<512>(p, grid, st);
    default: return cudaErrorInvalidValue;
    }
}

int qk_read_and_clear_error(uint32_t *code, uint32_t *site) { return module_read_and_clear_error(code, site); }

} // namespace ds
