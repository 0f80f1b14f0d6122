// ds_tile.cu -- the staged path: a persistent, bulk-copy (TMA) fed kernel
// for every row whose input fits a shared-memory slot of 16, 32 or 64 KB.
//
// One CTA per SM.  The last warp is the producer: it walks the CTA's slots
// (slot = a run of consecutive rows of one segment, at most the slot size of
// input) in order, waits until the slot's ring position is free, and fills
// it with one cp.async.bulk per array (or per row when rows are padded)
// completing on that position's "full" mbarrier.  The other warps own the
// ring positions, a team of warps each (one or two warps at 16 KB, more for
// larger slots): slot j of the CTA goes to position j % positions, whose
// team waits on "full", normalises its rows out of shared memory, stores the
// results straight to global memory, and arrives on "empty".  Because a
// position is consumed by its own team, in order, no barrier is ever waited
// on more than one phase ahead of its current phase.  Every wait is bounded.
//
// Per row a team sums in a fixed order -- each thread its units u = t,
// t + G, ... in order (G threads in the team), two packed fp32 accumulators
// (even and odd elements) added at the end, an xor butterfly over the lanes,
// then the warps' partials as a balanced tree -- so a row's bits depend on
// its length and the operation only.
#include <algorithm>
#include <atomic>

#include <cuda_runtime.h>

#include "ds_device.cuh"

namespace ds {

// ds_kernels.cu's tags, repeated (the two files share this numbering).
enum TileTag {
    tFwdBf16, tFwdF32, tBwdBf16, tBwdF32, tRenorm, tL2, tSlerp, tProject, tMomentum, tL2Bwd, tSlerpBwd, tGateL2,
    tSwigluL2, tNorms
};

__host__ __device__ constexpr bool is_weight_tag(int T)
{
    return T <= tRenorm || T == tProject || T == tMomentum || T == tNorms;
}
__host__ __device__ constexpr bool is_act_bwd_tag(int T) { return T == tL2Bwd || T == tSlerpBwd; }
__host__ __device__ constexpr bool is_fused_tag(int T) { return T == tGateL2 || T == tSwigluL2; }
__host__ __device__ constexpr bool is_act_tag(int T)
{
    return T == tL2 || T == tSlerp || is_act_bwd_tag(T) || is_fused_tag(T);
}

namespace {


struct SlotHdr {
    int32_t seg;
    int32_t nrows;
    int64_t row0;
};

// ------------------------------------------------------------- helpers --

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 lo2(uint32_t w) { return f2(bf_lo(w), bf_hi(w)); }

__device__ __forceinline__ uint32_t pk(float2 v) { return pack_bf2(v.x, v.y); }

__device__ __forceinline__ float warp_sum1(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max1(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ void sq2(float2 &acc, float2 v) { acc = __ffma2_rn(v, v, acc); }

template <class F>
__device__ __forceinline__ void each4_(float4 v, F &&f)
{
    f(v.x);
    f(v.y);
    f(v.z);
    f(v.w);
}

__device__ __forceinline__ float2 fneg2(float2 v) { return f2(-v.x, -v.y); }

__device__ __forceinline__ void named_sync(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Distributed shared memory helpers for rows split over a cluster: the
// address of a variable of this CTA as seen in peer `rank`'s shared memory,
// a store and an mbarrier arrival there (release at cluster scope: the
// values written before it are visible to whoever acquires the phase).
__device__ __forceinline__ uint32_t peer_addr(const void *local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
    return r;
}

__device__ __forceinline__ void peer_store_u32(uint32_t addr, uint32_t v)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// Two floats to peer `rank`'s shared memory at `addr`, completing 8 bytes of
// the transaction count of its mbarrier at `bar` (an asynchronous store: no
// fence on this thread's earlier global stores is needed, and the peer sees
// the values once it observes the barrier's phase complete).
__device__ __forceinline__ void peer_store2_tx(uint32_t addr, float a, float b, uint32_t bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(addr),
                 "f"(a), "f"(b), "r"(bar)
                 : "memory");
}

// Exchange area of one team when its rows are split over a cluster: two
// alternating buffers of [kMaxCluster CTAs][2 values] and their mbarriers
// (one arrival per exchange, the team's own, with the transaction bytes of
// the cluster's ncta asynchronous stores).
constexpr int kXchgFloats = 2 * kMaxCluster * 2;
constexpr int kXchgBytesPerTeam = kXchgFloats * 4 + 2 * 8;

// The cluster context of a CTA: its rank, the cluster's size, the CTA-wide
// abort flag (set here, and in every peer, by the first wait that gives up)
// and the bound of every wait.
struct ClusterCtx {
    uint32_t rank, ncta;
    volatile int *abort_flag;
    uint64_t limit_ns;

    __device__ void abort_all() const
    {
        *abort_flag = 1;
        for (uint32_t k = 0; k < ncta; ++k)
            if (k != rank)
                peer_store_u32(peer_addr(const_cast<int *>(abort_flag), k), 1u);
    }
};

// The threads that normalise one row: one warp (weight calls) or the team
// of WP warps that share a group of ring positions (activation calls), in
// each CTA of the row's cluster.  A sum comes back to every thread of every
// CTA with the same bits: the xor butterfly in each warp, then the warps'
// partials through shared memory and the group's named barrier, added as a
// balanced tree in warp order ((w0 + w1) + (w2 + w3) ...), then -- rows split
// over a cluster -- the CTAs' totals through distributed shared memory,
// added in rank order.  Two alternating slots make back-to-back reductions
// safe with one barrier each (all warps of a team run the same sequence of
// reductions; all CTAs of a cluster the same sequence of exchanges, and a
// CTA writes exchange k + 2 only after every peer's part of exchange k + 1
// arrived, which each peer sends after reading exchange k).
template <int N>
__device__ __forceinline__ float tree_sum(const float *r, int i)
{
    if constexpr (N == 1)
        return r[i];
    else
        return tree_sum<N / 2>(r, i) + tree_sum<N / 2>(r + N, i);
}

template <int N>
__device__ __forceinline__ float tree_max(const float *r)
{
    if constexpr (N == 1)
        return r[0];
    else
        return fmaxf(tree_max<N / 2>(r), tree_max<N / 2>(r + N));
}

template <int WP, bool SPLIT = false>
struct Team {
    static constexpr int G = 32 * WP; // threads per row in this CTA
    static constexpr int kRed = 4 * WP; // floats of `red`: [2 slots][WP warps][2 values]
    int t;                            // this thread's index in the team
    int bar;                          // named barrier (teams of several warps)
    float *red;
    int slot = 0;
    // rows split over a cluster (SPLIT): this team's exchange area (unused,
    // and dropped by the compiler, with one CTA per row)
    const ClusterCtx *ctx = nullptr;
    uint32_t xrank = 0, xn = 1;       // this CTA's rank, the cluster's CTAs (ctx's, in registers)
    float *xbuf = nullptr;            // [2][kMaxCluster][2]
    uint64_t *xbar = nullptr;         // [2]
    uint32_t xuse = 0;                // exchanges so far
    bool failed = false;              // an exchange gave up: store nothing more

    __device__ __forceinline__ uint32_t rank() const
    {
        if constexpr (SPLIT)
            return xrank;
        else
            return 0u;
    }
    __device__ __forceinline__ bool good() const
    {
        if constexpr (SPLIT)
            return !failed;
        else
            return true;
    }

    // The bounded wait for an exchange's phase, out of line (rarely taken
    // long); gives up at the limit or when this CTA or a peer aborted.
    __device__ __noinline__ bool wait_slow(uint64_t *bb, uint32_t parity) const
    {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bb, parity)) {
            if (*ctx->abort_flag || global_timer_ns() - t0 > ctx->limit_ns)
                return false;
        }
        return true;
    }

    // The CTAs' totals v[0..N) through the cluster, combined in rank order.
    // Thread 0 sends this CTA's totals to slot [rank] of every CTA's buffer
    // (its own included) with asynchronous stores that complete bytes on
    // that CTA's barrier, and arms its own barrier for the ncta stores it
    // will receive (the transaction count may run ahead of the arming);
    // every thread waits for the phase and adds the slots in rank order.
    template <int N, class Op>
    __device__ __forceinline__ void exchange(float (&v)[N], Op op)
    {
        static_assert(N <= 2, "two values at most");
        const int b = static_cast<int>(xuse & 1u);
        const uint32_t parity = (xuse >> 1) & 1u;
        ++xuse;
        float *buf = xbuf + b * (kMaxCluster * 2);
        uint64_t *bb = xbar + b;
        const uint32_t n = xn, me = xrank;
        __syncwarp();
        if (t == 0 && !failed) {
            const float v1 = N > 1 ? v[N > 1 ? 1 : 0] : 0.f;
            for (uint32_t k = 0; k < n; ++k)
                peer_store2_tx(peer_addr(buf + me * 2, k), v[0], v1, peer_addr(bb, k));
            mbar_arrive_expect_tx(bb, 8u * n);
        }
        bool ok = !failed;
        if (ok && !mbar_try_wait(bb, parity))
            ok = wait_slow(bb, parity);
        if (!ok) {
            if (!failed)
                ctx->abort_all();
            failed = true;
            return;
        }
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float a = buf[i];
            for (uint32_t k = 1; k < n; ++k)
                a = op(a, buf[k * 2 + i]);
            v[i] = a;
        }
    }

    template <int N>
    __device__ __forceinline__ void sum(float (&v)[N])
    {
#pragma unroll
        for (int i = 0; i < N; ++i)
            v[i] = warp_sum1(v[i]);
        if constexpr (WP > 1) {
            static_assert(N <= 2, "two values at most");
            float *r = red + slot * 2 * WP;
            if ((t & 31) == 0)
#pragma unroll
                for (int i = 0; i < N; ++i)
                    r[(t >> 5) * 2 + i] = v[i];
            named_sync(bar, G);
#pragma unroll
            for (int i = 0; i < N; ++i)
                v[i] = tree_sum<WP>(r, i);
            slot ^= 1;
        }
        if constexpr (SPLIT)
            exchange(v, [](float a, float b) { return a + b; });
    }

    __device__ __forceinline__ float sum1(float v)
    {
        float a[1] = {v};
        sum(a);
        return a[0];
    }

    __device__ __forceinline__ float max(float v)
    {
        v = warp_max1(v);
        if constexpr (WP > 1) {
            float *r = red + slot * 2 * WP;
            if ((t & 31) == 0)
                r[(t >> 5) * 2] = v;
            named_sync(bar, G);
            v = tree_max<WP>(r);
            slot ^= 1;
        }
        if constexpr (SPLIT) {
            float a[1] = {v};
            exchange(a, [](float x, float y) { return fmaxf(x, y); });
            v = a[0];
        }
        return v;
    }
};

// Factor of a row from its team-summed S (see RowScale).  The rescale path
// re-sums with exactly the fast path's structure -- the same pairs, in the
// same order, into two packed accumulators -- so that a row scaled by 2^k
// gives the same bits whichever path it takes.  `gen(f)` calls f(pair) on
// every pair the thread summed, in order.  The branch is uniform over the team.
template <class Red, class Gen>
__device__ __forceinline__ RowScale tile_scale(Red &red, float S, float eps, Gen &&gen)
{
    if (!needs_rescale(S, eps))
        return {1.0f / sqrtf(S + eps), 1.f};
    float M = 0.f;
    gen([&](float2 v) { M = fmaxf(M, fmaxf(fabsf(v.x), fabsf(v.y))); });
    M = red.max(M);
    if (!(M > 0.f && M < __int_as_float(0x7f800000)))
        return {1.0f / sqrtf(S + eps), 1.f};
    const int m = 48 - ilogbf(M);
    float2 acc = f2(0.f, 0.f);
    gen([&](float2 v) {
        const float2 u = f2(scalbnf(v.x, m), scalbnf(v.y, m));
        acc = __ffma2_rn(u, u, acc);
    });
    const float Ss = red.sum1(acc.x + acc.y);
    const float inv = 1.0f / sqrtf(Ss + scalbnf(eps, 2 * m));
    if (m > 100)
        return {scalbnf(inv, 100), scalbnf(1.f, m - 100)};
    return {scalbnf(inv, m), 1.f};
}

// |alpha| for the 8 elements of unit u, as four pairs, 0 past cols (the
// float4 holding the last valid element may extend past cols inside its
// 16-byte block; what it holds there is dropped).
__device__ __forceinline__ void alpha_pairs(const float *alpha, int u, int cols, float2 (&m)[4])
{
    const int e0 = 8 * u;
    const float4 a = e0 < cols ? __ldg(reinterpret_cast<const float4 *>(alpha + e0)) : make_float4(0, 0, 0, 0);
    const float4 b = e0 + 4 < cols ? __ldg(reinterpret_cast<const float4 *>(alpha + e0 + 4)) : make_float4(0, 0, 0, 0);
    m[0] = f2(fabsf(a.x), fabsf(a.y));
    m[1] = f2(fabsf(a.z), fabsf(a.w));
    m[2] = f2(fabsf(b.x), fabsf(b.y));
    m[3] = f2(fabsf(b.z), fabsf(b.w));
    if (e0 + 8 > cols) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            m[i] = f2(e0 + 2 * i < cols ? m[i].x : 0.f, e0 + 2 * i + 1 < cols ? m[i].y : 0.f);
    }
}

// ------------------------------------------------------- layout per op ---
//
// Arrays staged per row and their bytes per 16-byte unit of the row.

template <int T>
struct TileLayout {
    static constexpr int kArrays = (T == tFwdBf16 || T == tFwdF32 || T == tRenorm || T == tNorms) ? 1
                                   : is_act_bwd_tag(T)                                          ? 3
                                                                                                : 2;
    // bytes per unit of array a (the activation backward: x, r, dy)
    static __device__ __forceinline__ int ub(int a, bool has_r)
    {
        if (a == 0)
            return 16;
        if (T == tBwdBf16)
            return 8;
        if (T == tL2 || (T == tL2Bwd && a == 1))
            return has_r ? 16 : 0;
        return 16;
    }
};

// Source row pointers of array a.
template <int T>
__device__ __forceinline__ const char *tile_src(const WSegK &sg, int a, int64_t row)
{
    if (a == 0)
        return reinterpret_cast<const char *>(sg.w + row * sg.ld);
    return static_cast<const char *>(sg.gy) + row * sg.ld_out * (T == tBwdBf16 ? 2 : 4);
}

template <int T>
__device__ __forceinline__ const char *tile_src(const ASegK &sg, int a, int64_t row)
{
    return reinterpret_cast<const char *>((a == 0 ? sg.x : sg.r) + row * sg.ld);
}

template <int T>
__device__ __forceinline__ const char *tile_src(const AGSegK &sg, int a, int64_t row)
{
    return reinterpret_cast<const char *>((a == 0 ? sg.x : a == 1 ? sg.r : sg.dy) + row * sg.ld);
}

__device__ __forceinline__ bool seg_has_r(const WSegK &) { return true; }
__device__ __forceinline__ bool seg_has_r(const ASegK &s) { return s.r != nullptr; }
__device__ __forceinline__ bool seg_has_r(const AGSegK &s) { return s.r != nullptr; }

// Row pitch in global memory (bytes) of array a.
template <int T>
__device__ __forceinline__ int64_t tile_src_pitch(const WSegK &sg, int a)
{
    return a == 0 ? sg.ld * 4 : sg.ld_out * (T == tBwdBf16 ? 2 : 4);
}

template <int T>
__device__ __forceinline__ int64_t tile_src_pitch(const ASegK &sg, int)
{
    return sg.ld * 2;
}

template <int T>
__device__ __forceinline__ int64_t tile_src_pitch(const AGSegK &sg, int)
{
    return sg.ld * 2;
}

// ============================================================ row bodies ==
//
// `s0`, `s1`: this row's units of array 0 and 1 in shared memory (unit
// stride 16 or 8 bytes).  nfull = units with every element valid; `tail` =
// valid elements of unit nfull (0 if none), handled by lane nfull % 32 after
// its full units, so every lane's units are summed in increasing order.

template <bool OUT_BF16, bool RENORM, int WP, bool SPLIT>
__device__ __forceinline__ void tile_scale_row(Team<WP, SPLIT> &tm, const WSegK &sg, int64_t row, float g,
                                               const unsigned char *s0, int nfull, int tail, float eps, bool store)
{
    constexpr int G = Team<WP>::G;
    const int lane = tm.t;
    const float4 *w = reinterpret_cast<const float4 *>(s0);
    float2 acc = f2(0.f, 0.f);
#pragma unroll 4
    for (int u = lane; u < nfull; u += G) {
        const float4 v = w[u];
        sq2(acc, f2(v.x, v.y));
        sq2(acc, f2(v.z, v.w));
    }
    const bool tl = tail && lane == nfull % G;
    float4 vt = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tl) {
        vt = mask_quad(w[nfull], tail);
        sq2(acc, f2(vt.x, vt.y));
        sq2(acc, f2(vt.z, vt.w));
    }
    const float S = tm.sum1(acc.x + acc.y);
    const RowScale rs = tile_scale(tm, S, eps, [&](auto f) {
        for (int u = lane; u < nfull; u += G) {
            const float4 v = w[u];
            f(f2(v.x, v.y));
            f(f2(v.z, v.w));
        }
        if (tl) {
            f(f2(vt.x, vt.y));
            f(f2(vt.z, vt.w));
        }
    });
    if (!store || !tm.good())
        return;
    const float sc = (g * sg.radius) * rs.inv;
    const float2 sc2 = f2(sc, sc), pre2 = f2(rs.pre, rs.pre);
    char *out = RENORM ? reinterpret_cast<char *>(const_cast<float *>(sg.w) + row * sg.ld)
                       : static_cast<char *>(sg.out) + row * sg.ld_out * (OUT_BF16 ? 2 : 4);
    const bool plain = rs.pre == 1.f;
#pragma unroll 4
    for (int u = lane; u < nfull; u += G) {
        const float4 v = w[u];
        float2 a = f2(v.x, v.y), b = f2(v.z, v.w);
        if (!plain) {
            a = __fmul2_rn(a, pre2);
            b = __fmul2_rn(b, pre2);
        }
        a = __fmul2_rn(a, sc2);
        b = __fmul2_rn(b, sc2);
        if constexpr (OUT_BF16)
            st8(out + 8 * u, make_uint2(pk(a), pk(b)));
        else
            st16(out + 16 * u, make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x),
                                          __float_as_uint(b.y)));
    }
    if (tl) {
        const float4 y = make_float4((vt.x * rs.pre) * sc, (vt.y * rs.pre) * sc, (vt.z * rs.pre) * sc,
                                     (vt.w * rs.pre) * sc);
        if constexpr (OUT_BF16) {
            uint16_t *o = reinterpret_cast<uint16_t *>(out) + 4 * nfull;
            const float e[4] = {y.x, y.y, y.z, y.w};
            for (int i = 0; i < tail; ++i) {
                __nv_bfloat16 h = __float2bfloat16_rn(e[i]);
                o[i] = *reinterpret_cast<uint16_t *>(&h);
            }
        } else {
            float *o = reinterpret_cast<float *>(out) + 4 * nfull;
            o[0] = y.x;
            if (tail > 1) o[1] = y.y;
            if (tail > 2) o[2] = y.z;
        }
    }
}

// Row lengths (ds_row_norms; ds_gain_preserve with the radius as divisor):
// S summed as the forward sums it, then out[row] = sqrt(S + eps) / radius.
// A row whose fp32 sum overflows (or, at eps = 0, underflows) is summed
// again scaled by 2^m (exact) and its length scaled back.
template <int WP, bool SPLIT>
__device__ __forceinline__ void tile_norm_row(Team<WP, SPLIT> &tm, const WSegK &sg, int64_t row,
                                              const unsigned char *s0, int nfull, int tail, float eps, bool store)
{
    constexpr int G = Team<WP>::G;
    const int lane = tm.t;
    const float4 *w = reinterpret_cast<const float4 *>(s0);
    float2 acc = f2(0.f, 0.f);
#pragma unroll 4
    for (int u = lane; u < nfull; u += G) {
        const float4 v = w[u];
        sq2(acc, f2(v.x, v.y));
        sq2(acc, f2(v.z, v.w));
    }
    const bool tl = tail && lane == nfull % G;
    float4 vt = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tl) {
        vt = mask_quad(w[nfull], tail);
        sq2(acc, f2(vt.x, vt.y));
        sq2(acc, f2(vt.z, vt.w));
    }
    const float S = tm.sum1(acc.x + acc.y);
    float len = sqrtf(S + eps);
    if (needs_rescale(S, eps)) {
        float M = 0.f;
        for (int u = lane; u < nfull; u += G) {
            const float4 v = w[u];
            M = fmaxf(M, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
        M = fmaxf(M, fmaxf(fmaxf(fabsf(vt.x), fabsf(vt.y)), fmaxf(fabsf(vt.z), fabsf(vt.w))));
        M = tm.max(M);
        if (M > 0.f && M < __int_as_float(0x7f800000)) {
            const int m = 48 - ilogbf(M);
            float2 as = f2(0.f, 0.f);
            auto add = [&](float4 v) {
                const float2 a = f2(scalbnf(v.x, m), scalbnf(v.y, m)), b = f2(scalbnf(v.z, m), scalbnf(v.w, m));
                as = __ffma2_rn(a, a, as);
                as = __ffma2_rn(b, b, as);
            };
            for (int u = lane; u < nfull; u += G)
                add(w[u]);
            if (tl)
                add(vt);
            const float Ss = tm.sum1(as.x + as.y);
            len = scalbnf(sqrtf(Ss + scalbnf(eps, 2 * m)), -m);
        }
    }
    if (!store || !tm.good())
        return;
    if (lane == 0 && tm.rank() == 0)
        static_cast<float *>(sg.out)[row] = __fdiv_rn(len, sg.radius);
}

template <bool GY_BF16>
__device__ __forceinline__ float4 gy_unit(const unsigned char *s1, int u)
{
    if constexpr (GY_BF16) {
        const uint2 r = *reinterpret_cast<const uint2 *>(s1 + 8 * u);
        return make_float4(bf_lo(r.x), bf_hi(r.x), bf_lo(r.y), bf_hi(r.y));
    } else {
        return *reinterpret_cast<const float4 *>(s1 + 16 * u);
    }
}

// Epilogues of the two-reduction row (S = sum w^2, D = w . d; d staged as
// array 1): MODE 0 = ds_wn_backward (grad_w, grad_g), 1 = ds_grad_project
// (d <- d - w D/n^2 in place), 2 = ds_renorm_momentum (the same on the
// momentum, and w <- rho w / n in place).  With the power-of-two rescale the
// projection applies the scaled quotient to the scaled row, which stays
// finite where D/n^2 alone would overflow.
template <bool GY_BF16, int MODE, int WP, bool SPLIT>
__device__ __forceinline__ void tile_backward_row(Team<WP, SPLIT> &tm, const WSegK &sg, int64_t row, float g,
                                                  const unsigned char *s0, const unsigned char *s1, int nfull,
                                                  int tail, float eps, bool store)
{
    constexpr int G = Team<WP>::G;
    const int lane = tm.t;
    const float4 *w = reinterpret_cast<const float4 *>(s0);
    float2 as = f2(0.f, 0.f), ad = f2(0.f, 0.f);
#pragma unroll 4
    for (int u = lane; u < nfull; u += G) {
        const float4 x = w[u];
        const float4 d = gy_unit<GY_BF16>(s1, u);
        sq2(as, f2(x.x, x.y));
        sq2(as, f2(x.z, x.w));
        ad = __ffma2_rn(f2(x.x, x.y), f2(d.x, d.y), ad);
        ad = __ffma2_rn(f2(x.z, x.w), f2(d.z, d.w), ad);
    }
    const bool tl = tail && lane == nfull % G;
    float4 xt = make_float4(0.f, 0.f, 0.f, 0.f), dt = xt;
    if (tl) {
        xt = mask_quad(w[nfull], tail);
        dt = mask_quad(gy_unit<GY_BF16>(s1, nfull), tail);
        sq2(as, f2(xt.x, xt.y));
        sq2(as, f2(xt.z, xt.w));
        ad = __ffma2_rn(f2(xt.x, xt.y), f2(dt.x, dt.y), ad);
        ad = __ffma2_rn(f2(xt.z, xt.w), f2(dt.z, dt.w), ad);
    }
    float sd[2] = {as.x + as.y, ad.x + ad.y};
    tm.sum(sd);
    float S = sd[0], D = sd[1];
    // Rows needing the rescale: w scaled by 2^m (exact), S and D re-summed,
    // 2^m carried into the row constants (as the register paths do).
    int m = 0;
    if (needs_rescale(S, eps)) {
        float M = 0.f;
        for (int u = lane; u < nfull; u += G)
            each4_(w[u], [&](float v) { M = fmaxf(M, fabsf(v)); });
        if (tl)
            each4_(xt, [&](float v) { M = fmaxf(M, fabsf(v)); });
        M = tm.max(M);
        if (M > 0.f && M < __int_as_float(0x7f800000)) {
            m = 48 - ilogbf(M);
            float2 bs = f2(0.f, 0.f), bd = f2(0.f, 0.f);
            auto add = [&](float4 x, float4 d) {
                const float2 p = f2(scalbnf(x.x, m), scalbnf(x.y, m)), q = f2(scalbnf(x.z, m), scalbnf(x.w, m));
                sq2(bs, p);
                sq2(bs, q);
                bd = __ffma2_rn(p, f2(d.x, d.y), bd);
                bd = __ffma2_rn(q, f2(d.z, d.w), bd);
            };
            for (int u = lane; u < nfull; u += G)
                add(w[u], gy_unit<GY_BF16>(s1, u));
            if (tl)
                add(xt, dt);
            float sd2[2] = {bs.x + bs.y, bd.x + bd.y};
            tm.sum(sd2);
            S = sd2[0];
            D = sd2[1];
        }
    }
    if (!store || !tm.good())
        return;
    const float n2 = S + (m == 0 ? eps : scalbnf(eps, 2 * m));
    const float inv = 1.0f / sqrtf(n2);
    if constexpr (MODE != 0) {
        const float2 nqs = f2(-D / n2, -D / n2);      // -D/(S+eps) times 2^-m
        const float sc = sg.radius * inv;             // rho / n times 2^-m
        const float2 sc2 = f2(sc, sc);
        float *dd = sg.grad_w + row * sg.ld;
        float *wo = static_cast<float *>(sg.out) + row * sg.ld;
        auto scaled = [&](float4 x) {
            return m == 0 ? x : make_float4(scalbnf(x.x, m), scalbnf(x.y, m), scalbnf(x.z, m), scalbnf(x.w, m));
        };
#pragma unroll 4
        for (int u = lane; u < nfull; u += G) {
            const float4 x = scaled(w[u]);
            const float4 d = gy_unit<GY_BF16>(s1, u);
            const float2 a = __ffma2_rn(f2(x.x, x.y), nqs, f2(d.x, d.y));
            const float2 b = __ffma2_rn(f2(x.z, x.w), nqs, f2(d.z, d.w));
            st16(dd + 4 * u, make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x),
                                        __float_as_uint(b.y)));
            if constexpr (MODE == 2) {
                const float2 p = __fmul2_rn(f2(x.x, x.y), sc2), q = __fmul2_rn(f2(x.z, x.w), sc2);
                st16(wo + 4 * u, make_uint4(__float_as_uint(p.x), __float_as_uint(p.y), __float_as_uint(q.x),
                                            __float_as_uint(q.y)));
            }
        }
        if (tl) {
            const float4 x = scaled(xt);
            const float e[3] = {x.x, x.y, x.z}, dv[3] = {dt.x, dt.y, dt.z};
            for (int i = 0; i < tail; ++i) {
                dd[4 * nfull + i] = fmaf(e[i], nqs.x, dv[i]);
                if constexpr (MODE == 2)
                    wo[4 * nfull + i] = e[i] * sc;
            }
        }
        return;
    }
    const float q = m == 0 ? D / n2 : scalbnf(D / n2, m);
    const float pre = (g * sg.radius) * (m == 0 ? inv : scalbnf(inv, m));
    if (lane == 0 && sg.gain && tm.rank() == 0)
        sg.grad_g[row] = sg.radius * D * inv;
    const float2 nq = f2(-q, -q), pre2 = f2(pre, pre);
    char *out = reinterpret_cast<char *>(sg.grad_w + row * sg.ld);
#pragma unroll 4
    for (int u = lane; u < nfull; u += G) {
        const float4 x = w[u];
        const float4 d = gy_unit<GY_BF16>(s1, u);
        const float2 a = __fmul2_rn(__ffma2_rn(f2(x.x, x.y), nq, f2(d.x, d.y)), pre2);
        const float2 b = __fmul2_rn(__ffma2_rn(f2(x.z, x.w), nq, f2(d.z, d.w)), pre2);
        st16(out + 16 * u,
             make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x), __float_as_uint(b.y)));
    }
    if (tl) {
        float *o = reinterpret_cast<float *>(out) + 4 * nfull;
        o[0] = pre * fmaf(xt.x, -q, dt.x);
        if (tail > 1) o[1] = pre * fmaf(xt.y, -q, dt.y);
        if (tail > 2) o[2] = pre * fmaf(xt.z, -q, dt.z);
    }
}

// p[0..4) += v at the memory (fp32 adds rounded to nearest), without the
// round trip of reading the line back: the slerp backward's dalpha lines.
// Only the calling thread ever updates these floats, so the additions take
// place in its program order, row after row -- the same sums, in the same
// order, as a read-modify-write.
__device__ __forceinline__ void red_add4(float *p, float4 v)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// Octet helpers: 8 bf16 as four packed pairs.
//
// Squares of a bf16 pair into the (even, odd) accumulators with one fused
// multiply-add per element taken straight from the packed halves: the
// product of two bf16 is exact in fp32, so each step rounds exactly as the
// fp32 fma of the widened values would (the same bits as sq2(acc, lo2(w))).
__device__ __forceinline__ void sq_bf2(float2 &acc, uint32_t w)
{
    asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
        "fma.rn.f32.bf16 %0, l, l, %0;\n\tfma.rn.f32.bf16 %1, h, h, %1;\n\t}"
        : "+f"(acc.x), "+f"(acc.y)
        : "r"(w));
}

// The same sums through widened pairs (packed fp32 fma): the l2 rows use
// this form (with a residual the widened pairs also serve the sum x + r);
// slerp's two-array pass 1 is faster with sq8.
__device__ __forceinline__ void sq8w(float2 &acc, uint4 v)
{
    sq2(acc, lo2(v.x));
    sq2(acc, lo2(v.y));
    sq2(acc, lo2(v.z));
    sq2(acc, lo2(v.w));
}

__device__ __forceinline__ void sq8(float2 &acc, uint4 v)
{
    sq_bf2(acc, v.x);
    sq_bf2(acc, v.y);
    sq_bf2(acc, v.z);
    sq_bf2(acc, v.w);
}

template <class F>
__device__ __forceinline__ void pairs8(uint4 v, F &&f)
{
    f(lo2(v.x));
    f(lo2(v.y));
    f(lo2(v.z));
    f(lo2(v.w));
}

__device__ __forceinline__ uint4 scale8(uint4 v, RowScale r)
{
    const float2 s = f2(r.inv, r.inv);
    if (r.pre == 1.f)
        return make_uint4(pk(__fmul2_rn(lo2(v.x), s)), pk(__fmul2_rn(lo2(v.y), s)), pk(__fmul2_rn(lo2(v.z), s)),
                          pk(__fmul2_rn(lo2(v.w), s)));
    const float2 p = f2(r.pre, r.pre);
    return make_uint4(pk(__fmul2_rn(__fmul2_rn(lo2(v.x), p), s)), pk(__fmul2_rn(__fmul2_rn(lo2(v.y), p), s)),
                      pk(__fmul2_rn(__fmul2_rn(lo2(v.z), p), s)), pk(__fmul2_rn(__fmul2_rn(lo2(v.w), p), s)));
}

// bf16(x + r) for a pair: the fp32 sum, rounded to nearest even.  The fp32
// sum of two bf16 is exact unless their exponents are more than 16 apart,
// and then its error lies far from any bf16 halfway point, so this is the
// exact sum rounded once.
__device__ __forceinline__ uint32_t add_bf2(uint32_t a, uint32_t b)
{
    return pk(__fadd2_rn(lo2(a), lo2(b)));
}

__device__ __forceinline__ void store_tail8(uint16_t *o, uint4 v, int valid)
{
    for (int e = 0; e < valid; ++e) {
        const uint32_t w = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
        o[e] = static_cast<uint16_t>((e & 1) ? (w >> 16) : (w & 0xFFFFu));
    }
}

// l2 rows (a pair of warps per row).  With a residual, pass 1 writes
// s = bf16(x + r) back over x in the slot (each thread its own units), so
// pass 2 reads s directly.  Full units run in the loops; the ragged last
// unit (if any) once, by its owner.
template <bool HAS_R>
__device__ __forceinline__ uint4 l2_unit_s(const uint4 *x, const uint4 *r, int u)
{
    uint4 s = x[u];
    if constexpr (HAS_R) {
        const uint4 b = r[u];
        s = make_uint4(add_bf2(s.x, b.x), add_bf2(s.y, b.y), add_bf2(s.z, b.z), add_bf2(s.w, b.w));
    }
    return s;
}

template <int WP, bool HAS_R, bool SPLIT>
__device__ __forceinline__ void tile_l2_row(Team<WP, SPLIT> &tm, const ASegK &sg, int64_t row, unsigned char *s0,
                                            const unsigned char *s1, int nfull, int tail, float eps, bool store)
{
    constexpr int G = Team<WP>::G;
    const int t = tm.t;
    const bool tl = tail && t == nfull % G;
    uint4 *x = reinterpret_cast<uint4 *>(s0);
    const uint4 *r = reinterpret_cast<const uint4 *>(s1);
    float2 acc = f2(0.f, 0.f);
#pragma unroll 4
    for (int u = t; u < nfull; u += G) {
        const uint4 s = l2_unit_s<HAS_R>(x, r, u);
        if constexpr (HAS_R)
            x[u] = s;
        sq8w(acc, s);
    }
    if (tl) {
        const uint4 s = mask_octet(l2_unit_s<HAS_R>(x, r, nfull), tail);
        x[nfull] = s;
        sq8w(acc, s);
    }
    const float S = tm.sum1(acc.x + acc.y);
    const int nunits = nfull + (tail ? 1 : 0);
    const RowScale rs = tile_scale(tm, S, eps, [&](auto f) {
        for (int u = t; u < nunits; u += G)
            pairs8(x[u], f);
    });
    if (!store || !tm.good())
        return;
    uint16_t *y = sg.y + row * sg.ld;
#pragma unroll 4
    for (int u = t; u < nfull; u += G)
        st16(y + 8 * u, scale8(x[u], rs));
    if (tl)
        store_tail8(y + 8 * nfull, scale8(x[nfull], rs), tail);
}

// slerp rows (a pair of warps per row).  Pass 1 sums res^2 and out^2.
// Pass 2 forms a = bf16(l2(res)), b = bf16(l2(out)) and the lerp
// t = a + |alpha| (b - a) in fp32, sums t^2, and writes t over the row's
// inputs in the slot (t's first four of each unit over res, the last four
// over out; each thread its own units).  Pass 3 scales t and stores h.  The
// full units run in the loops; the ragged last unit (if any) once, by its
// owner, after them.
__device__ __forceinline__ float2 lerp2(float2 a, float2 b, float2 m)
{
    return __ffma2_rn(m, __fadd2_rn(b, fneg2(a)), a);
}

// How much of a launch's per-column vector a CTA holds in shared memory:
// none, all of its columns, or (slerp rows longer than the cache) the first
// columns, with the rest read from global memory.
enum AlphaCache { kAlphaNone = 0, kAlphaAll = 1, kAlphaHead = 2 };

// |alpha| of unit u: from the shared-memory cache (split layout: the first
// four of each unit at abs_alpha[4u], the last four at abs_alpha[half + 4u];
// units below half / 4) or from global memory.
template <int AC>
__device__ __forceinline__ void abs_alpha8(const float *abs_alpha, int half, const float *alpha, int u, int cols,
                                           float2 (&m)[4])
{
    if (AC == kAlphaAll || (AC == kAlphaHead && 4 * u < half)) {
        const float4 m0 = *reinterpret_cast<const float4 *>(abs_alpha + 4 * u);
        const float4 m1 = *reinterpret_cast<const float4 *>(abs_alpha + half + 4 * u);
        m[0] = f2(m0.x, m0.y);
        m[1] = f2(m0.z, m0.w);
        m[2] = f2(m1.x, m1.y);
        m[3] = f2(m1.z, m1.w);
    } else {
        alpha_pairs(alpha, u, cols, m);
    }
}

template <int AC>
__device__ __forceinline__ void slerp_unit_t(uint4 p, uint4 q, RowScale ra, RowScale rb, const float *abs_alpha,
                                             int half, const float *alpha, int u, int cols, float2 &at, float4 &ta,
                                             float4 &tb)
{
    const uint4 a = scale8(p, ra), b = scale8(q, rb);
    float2 m[4];
    abs_alpha8<AC>(abs_alpha, half, alpha, u, cols, m);
    const float2 t0 = lerp2(lo2(a.x), lo2(b.x), m[0]), t1 = lerp2(lo2(a.y), lo2(b.y), m[1]);
    const float2 t2 = lerp2(lo2(a.z), lo2(b.z), m[2]), t3 = lerp2(lo2(a.w), lo2(b.w), m[3]);
    sq2(at, t0);
    sq2(at, t1);
    sq2(at, t2);
    sq2(at, t3);
    ta = make_float4(t0.x, t0.y, t1.x, t1.y);
    tb = make_float4(t2.x, t2.y, t3.x, t3.y);
}

__device__ __forceinline__ uint4 slerp_unit_h(float4 p, float4 q, float2 s)
{
    return make_uint4(pk(__fmul2_rn(f2(p.x, p.y), s)), pk(__fmul2_rn(f2(p.z, p.w), s)),
                      pk(__fmul2_rn(f2(q.x, q.y), s)), pk(__fmul2_rn(f2(q.z, q.w), s)));
}

template <int WP, int AC, bool SPLIT>
__device__ __forceinline__ void tile_slerp_row(Team<WP, SPLIT> &tm, const ASegK &sg, int64_t row, unsigned char *s0,
                                               unsigned char *s1, int nfull, int tail, float eps, bool store,
                                               const float *abs_alpha, int half)
{
    constexpr int G = Team<WP>::G;
    const int t = tm.t;
    const bool tl = tail && t == nfull % G; // owner of the ragged last unit
    uint4 *xa = reinterpret_cast<uint4 *>(s0);
    uint4 *xb = reinterpret_cast<uint4 *>(s1);
    float4 *ta = reinterpret_cast<float4 *>(s0);
    float4 *tb = reinterpret_cast<float4 *>(s1);
    // pass 1
    float2 aa = f2(0.f, 0.f), ab = f2(0.f, 0.f);
#pragma unroll 2
    for (int u = t; u < nfull; u += G) {
        sq8(aa, xa[u]);
        sq8(ab, xb[u]);
    }
    if (tl) {
        const uint4 p = mask_octet(xa[nfull], tail), q = mask_octet(xb[nfull], tail);
        xa[nfull] = p;
        xb[nfull] = q;
        sq8(aa, p);
        sq8(ab, q);
    }
    float sab[2] = {aa.x + aa.y, ab.x + ab.y};
    tm.sum(sab);
    const int nunits = nfull + (tail ? 1 : 0);
    const RowScale ra = tile_scale(tm, sab[0], eps, [&](auto f) {
        for (int u = t; u < nunits; u += G)
            pairs8(xa[u], f);
    });
    const RowScale rb = tile_scale(tm, sab[1], eps, [&](auto f) {
        for (int u = t; u < nunits; u += G)
            pairs8(xb[u], f);
    });
    // pass 2
    float2 at = f2(0.f, 0.f);
#pragma unroll 4
    for (int u = t; u < nfull; u += G) {
        float4 p, q;
        slerp_unit_t<AC>(xa[u], xb[u], ra, rb, abs_alpha, half, sg.alpha, u, sg.cols, at, p, q);
        ta[u] = p;
        tb[u] = q;
    }
    if (tl) {
        float4 p, q;
        slerp_unit_t<AC>(xa[nfull], xb[nfull], ra, rb, abs_alpha, half, sg.alpha, nfull, sg.cols, at, p, q);
        ta[nfull] = p;
        tb[nfull] = q;
    }
    const float St = tm.sum1(at.x + at.y);
    const RowScale rt = tile_scale(tm, St, eps, [&](auto f) {
        for (int u = t; u < nunits; u += G) {
            const float4 p = ta[u], q = tb[u];
            f(f2(p.x, p.y));
            f(f2(p.z, p.w));
            f(f2(q.x, q.y));
            f(f2(q.z, q.w));
        }
    });
    if (!store || !tm.good())
        return;
    // pass 3
    uint16_t *y = sg.y + row * sg.ld;
    const float2 s = f2(rt.inv, rt.inv);
    if (rt.pre == 1.f) {
#pragma unroll 4
        for (int u = t; u < nfull; u += G)
            st16(y + 8 * u, slerp_unit_h(ta[u], tb[u], s));
    } else {
        const float2 pr = f2(rt.pre, rt.pre);
        for (int u = t; u < nfull; u += G) {
            const float4 p = ta[u], q = tb[u];
            const float4 pp = make_float4(p.x * pr.x, p.y * pr.x, p.z * pr.x, p.w * pr.x);
            const float4 qq = make_float4(q.x * pr.x, q.y * pr.x, q.z * pr.x, q.w * pr.x);
            st16(y + 8 * u, slerp_unit_h(pp, qq, s));
        }
    }
    if (tl) {
        float4 p = ta[nfull], q = tb[nfull];
        p = make_float4(p.x * rt.pre, p.y * rt.pre, p.z * rt.pre, p.w * rt.pre);
        q = make_float4(q.x * rt.pre, q.y * rt.pre, q.z * rt.pre, q.w * rt.pre);
        store_tail8(y + 8 * nfull, slerp_unit_h(p, q, s), tail);
    }
}

// ===================================================== activation backward ==
//
// Derived gradients of the two activation calls, straight through their bf16
// rounding points (which keep the rounded values the forward uses).  Inputs
// come from the slot (x, r, dy bf16 as arrays 0, 1, 2); gradients go straight
// to global memory in fp32.

__device__ __forceinline__ void dot8(float2 &acc, uint4 a, uint4 b)
{
    acc = __ffma2_rn(lo2(a.x), lo2(b.x), acc);
    acc = __ffma2_rn(lo2(a.y), lo2(b.y), acc);
    acc = __ffma2_rn(lo2(a.z), lo2(b.z), acc);
    acc = __ffma2_rn(lo2(a.w), lo2(b.w), acc);
}

__device__ __forceinline__ uint32_t word4(uint4 v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// Eight fp32 values of one unit to row `o` at unit u: one 32-byte store
// where the row starts on 32 bytes (a32), so that a warp's store covers its
// 1 KB of the row whole; else two 16-byte stores; or only the first `valid`
// elements.
__device__ __forceinline__ void store8f(float *o, int u, const float2 (&v)[4], int valid, bool a32)
{
    if (valid >= 8) {
        const uint4 lo = make_uint4(__float_as_uint(v[0].x), __float_as_uint(v[0].y), __float_as_uint(v[1].x),
                                    __float_as_uint(v[1].y));
        const uint4 hi = make_uint4(__float_as_uint(v[2].x), __float_as_uint(v[2].y), __float_as_uint(v[3].x),
                                    __float_as_uint(v[3].y));
        if (a32) {
            st32(o + 8 * u, lo, hi);
        } else {
            st16(o + 8 * u, lo);
            st16(o + 8 * u + 4, hi);
        }
    } else {
        // fully unrolled: v stays in registers (a runtime index would put it
        // in local memory)
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (e < valid)
                o[8 * u + e] = (e & 1) ? v[e >> 1].y : v[e >> 1].x;
    }
}

// l2 backward: s = x or bf16(x + r) (written back over x, as in the
// forward), S = sum s^2 and D = sum s dy in one pass, then
// dx = (dy - s D/(S+eps)) / sqrt(S+eps).  Rows needing the power-of-two
// rescale re-sum with s scaled by 2^m and apply the scaled quotient to the
// scaled row (exactly the unscaled product), with 2^m carried into 1/n.
template <int WP, bool HAS_R, bool SPLIT>
__device__ __forceinline__ void tile_l2_bwd_row(Team<WP, SPLIT> &tm, const AGSegK &sg, int64_t row, unsigned char *s0,
                                                const unsigned char *s1, unsigned char *s2, int nfull, int tail,
                                                float eps, bool store)
{
    constexpr int G = Team<WP>::G;
    const int t = tm.t;
    const bool tl = tail && t == nfull % G;
    const int nunits = nfull + (tail ? 1 : 0);
    uint4 *x = reinterpret_cast<uint4 *>(s0);
    const uint4 *r = reinterpret_cast<const uint4 *>(s1);
    uint4 *dy = reinterpret_cast<uint4 *>(s2);
    float2 as = f2(0.f, 0.f), ad = f2(0.f, 0.f);
#pragma unroll 4
    for (int u = t; u < nfull; u += G) {
        const uint4 sv = l2_unit_s<HAS_R>(x, r, u);
        if constexpr (HAS_R)
            x[u] = sv;
        sq8w(as, sv);
        dot8(ad, sv, dy[u]);
    }
    if (tl) {
        const uint4 sv = mask_octet(l2_unit_s<HAS_R>(x, r, nfull), tail);
        const uint4 d = mask_octet(dy[nfull], tail);
        x[nfull] = sv;
        dy[nfull] = d;
        sq8w(as, sv);
        dot8(ad, sv, d);
    }
    float sd[2] = {as.x + as.y, ad.x + ad.y};
    tm.sum(sd);
    float S = sd[0], D = sd[1];
    int m = 0;
    if (needs_rescale(S, eps)) {
        float M = 0.f;
        for (int u = t; u < nunits; u += G)
            pairs8(x[u], [&](float2 v) { M = fmaxf(M, fmaxf(fabsf(v.x), fabsf(v.y))); });
        M = tm.max(M);
        if (M > 0.f && M < __int_as_float(0x7f800000)) {
            m = 48 - ilogbf(M);
            float2 bs = f2(0.f, 0.f), bd = f2(0.f, 0.f);
            for (int u = t; u < nunits; u += G) {
                const uint4 sv = x[u], d = dy[u];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 v = lo2(word4(sv, i));
                    const float2 w2 = f2(scalbnf(v.x, m), scalbnf(v.y, m));
                    sq2(bs, w2);
                    bd = __ffma2_rn(w2, lo2(word4(d, i)), bd);
                }
            }
            float sd2[2] = {bs.x + bs.y, bd.x + bd.y};
            tm.sum(sd2);
            S = sd2[0];
            D = sd2[1];
        }
    }
    if (!store || !tm.good())
        return;
    const float n2 = S + (m == 0 ? eps : scalbnf(eps, 2 * m));
    const float inv = 1.0f / sqrtf(n2);
    const float2 nq = f2(-D / n2, -D / n2);                      // -D/(S+eps) times 2^-m
    const float os = m == 0 ? inv : scalbnf(inv, m);              // 1/n
    const float2 os2 = f2(os, os);
    float *o = sg.dx + row * sg.ld_d;
    const bool a32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
#pragma unroll 2
    for (int u = t; u < nunits; u += G) {
        const uint4 sv = x[u], d = dy[u];
        float2 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 sp = lo2(word4(sv, i));
            if (m != 0)
                sp = f2(scalbnf(sp.x, m), scalbnf(sp.y, m));
            v[i] = __fmul2_rn(__ffma2_rn(sp, nq, lo2(word4(d, i))), os2);
        }
        store8f(o, u, v, u < nfull ? 8 : tail, a32);
    }
}

// alpha of unit u as four pairs, signed: from the cache (split layout) or
// from global memory (0 past cols).
template <bool CACHED>
__device__ __forceinline__ void alpha8_signed(const float *cache, int half, const float *alpha, int u, int cols,
                                              float2 (&m)[4])
{
    if constexpr (CACHED) {
        const float4 m0 = *reinterpret_cast<const float4 *>(cache + 4 * u);
        const float4 m1 = *reinterpret_cast<const float4 *>(cache + half + 4 * u);
        m[0] = f2(m0.x, m0.y);
        m[1] = f2(m0.z, m0.w);
        m[2] = f2(m1.x, m1.y);
        m[3] = f2(m1.z, m1.w);
    } else {
        const int e0 = 8 * u;
        const float4 a = e0 < cols ? __ldg(reinterpret_cast<const float4 *>(alpha + e0)) : make_float4(0, 0, 0, 0);
        const float4 b = e0 + 4 < cols ? __ldg(reinterpret_cast<const float4 *>(alpha + e0 + 4))
                                       : make_float4(0, 0, 0, 0);
        m[0] = f2(a.x, a.y);
        m[1] = f2(a.z, a.w);
        m[2] = f2(b.x, b.y);
        m[3] = f2(b.z, b.w);
        if (e0 + 8 > cols) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                m[i] = f2(e0 + 2 * i < cols ? m[i].x : 0.f, e0 + 2 * i + 1 < cols ? m[i].y : 0.f);
        }
    }
}

__device__ __forceinline__ float2 abs2(float2 v) { return f2(fabsf(v.x), fabsf(v.y)); }
__device__ __forceinline__ float2 sgn2(float2 v)
{
    return f2(v.x > 0.f ? 1.f : v.x < 0.f ? -1.f : 0.f, v.y > 0.f ? 1.f : v.y < 0.f ? -1.f : 0.f);
}

// slerp backward, three passes over the slot.  Pass 1 sums res^2 and
// out^2.  Pass 2 forms a, b and t as the forward does and sums, besides
// St = t . t and Dt = t . dh, the four sums that fold the projections of
// da = (1 - |alpha|) dt and db = |alpha| dt onto ua = res/na and ub = out/nb
// (before their rounding) into the same pass: with q = Dt/(St + eps) and
// it = 1/sqrt(St + eps), dt = (dh - t q) it, so
//   ua . da = it (ua (1-|alpha|) . dh - q  ua (1-|alpha|) . t),
//   ub . db = it (ub |alpha| . dh    - q  ub |alpha| . t).
// Pass 3 forms dt, da, db, stores dres = (da - ua (ua . da))/na and dout
// likewise, and adds this row's sign(alpha) (b - a) dt to the team's dalpha
// line.  The terms of each sum are exact rearrangements of the definition;
// only the fp32 rounding order differs.
template <int WP, bool CACHED, bool SPLIT>
__device__ __forceinline__ void tile_slerp_bwd_row(Team<WP, SPLIT> &tm, const AGSegK &sg, int64_t row, unsigned char *s0,
                                                   unsigned char *s1, unsigned char *s2, int nfull, int tail, float eps,
                                                   bool store, const float *acache, int half, float *wsl,
                                                   bool ws_first)
{
    constexpr int G = Team<WP>::G;
    const int t = tm.t;
    const bool tl = tail && t == nfull % G;
    const int nunits = nfull + (tail ? 1 : 0);
    uint4 *xa = reinterpret_cast<uint4 *>(s0);
    uint4 *xb = reinterpret_cast<uint4 *>(s1);
    uint4 *xd = reinterpret_cast<uint4 *>(s2);
    // pass 1
    float2 aa = f2(0.f, 0.f), ab = f2(0.f, 0.f);
#pragma unroll 2
    for (int u = t; u < nfull; u += G) {
        sq8(aa, xa[u]);
        sq8(ab, xb[u]);
    }
    if (tl) {
        const uint4 p = mask_octet(xa[nfull], tail), q = mask_octet(xb[nfull], tail);
        xa[nfull] = p;
        xb[nfull] = q;
        xd[nfull] = mask_octet(xd[nfull], tail);
        sq8(aa, p);
        sq8(ab, q);
    }
    float sab[2] = {aa.x + aa.y, ab.x + ab.y};
    tm.sum(sab);
    const RowScale ra = tile_scale(tm, sab[0], eps, [&](auto f) {
        for (int u = t; u < nunits; u += G)
            pairs8(xa[u], f);
    });
    const RowScale rb = tile_scale(tm, sab[1], eps, [&](auto f) {
        for (int u = t; u < nunits; u += G)
            pairs8(xb[u], f);
    });
    const float2 pa = f2(ra.pre, ra.pre), ia = f2(ra.inv, ra.inv);
    const float2 pb = f2(rb.pre, rb.pre), ib = f2(rb.inv, rb.inv);
    const bool plain = ra.pre == 1.f && rb.pre == 1.f;
    // per unit: ua, ub (the forward's products before rounding), a, b
    // (bf16), t (fp32) and alpha (signed) as pairs
    auto unit = [&](int u, float2 (&ua)[4], float2 (&ub)[4], float2 (&a)[4], float2 (&b)[4], float2 (&al)[4],
                    float2 (&tv)[4]) {
        const uint4 r = xa[u], o = xb[u];
        alpha8_signed<CACHED>(acache, half, sg.alpha, u, sg.cols, al);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 vr = lo2(word4(r, i)), vo = lo2(word4(o, i));
            ua[i] = plain ? __fmul2_rn(vr, ia) : __fmul2_rn(__fmul2_rn(vr, pa), ia);
            ub[i] = plain ? __fmul2_rn(vo, ib) : __fmul2_rn(__fmul2_rn(vo, pb), ib);
            a[i] = lo2(pk(ua[i]));
            b[i] = lo2(pk(ub[i]));
            tv[i] = lerp2(a[i], b[i], abs2(al[i]));
        }
    };
    const float2 one = f2(1.f, 1.f);
    // pass 2
    float2 st = f2(0.f, 0.f), sd = f2(0.f, 0.f), a_d = f2(0.f, 0.f), a_t = f2(0.f, 0.f), b_d = f2(0.f, 0.f),
           b_t = f2(0.f, 0.f);
#pragma unroll 1
    for (int u = t; u < nunits; u += G) {
        float2 ua[4], ub[4], a[4], b[4], al[4], tv[4];
        unit(u, ua, ub, a, b, al, tv);
        const uint4 d = xd[u];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 dh = lo2(word4(d, i)), m = abs2(al[i]);
            const float2 wa = __fmul2_rn(ua[i], __fadd2_rn(one, fneg2(m))), wb = __fmul2_rn(ub[i], m);
            sq2(st, tv[i]);
            sd = __ffma2_rn(tv[i], dh, sd);
            a_d = __ffma2_rn(wa, dh, a_d);
            a_t = __ffma2_rn(wa, tv[i], a_t);
            b_d = __ffma2_rn(wb, dh, b_d);
            b_t = __ffma2_rn(wb, tv[i], b_t);
        }
    }
    float s1v[2] = {st.x + st.y, sd.x + sd.y};
    tm.sum(s1v);
    float s2v[2] = {a_d.x + a_d.y, a_t.x + a_t.y};
    tm.sum(s2v);
    float s3v[2] = {b_d.x + b_d.y, b_t.x + b_t.y};
    tm.sum(s3v);
    if (!store || !tm.good())
        return;
    const float nt2 = s1v[0] + eps;
    const float it = 1.0f / sqrtf(nt2);
    const float q = s1v[1] / nt2;
    const float Sa = it * (s2v[0] - q * s2v[1]);   // ua . da
    const float Sb = it * (s3v[0] - q * s3v[1]);   // ub . db
    const float2 nq = f2(-q, -q), it2 = f2(it, it);
    const float2 nDa = f2(-Sa, -Sa), nDb = f2(-Sb, -Sb);
    const float ra_n = ra.inv * ra.pre, rb_n = rb.inv * rb.pre;      // 1/na, 1/nb
    const float2 ra2 = f2(ra_n, ra_n), rb2 = f2(rb_n, rb_n);
    float *odx = sg.dx + row * sg.ld_d;
    float *odr = sg.dr + row * sg.ld_d;
    const bool a32 = ((reinterpret_cast<uintptr_t>(odx) | reinterpret_cast<uintptr_t>(odr)) & 31u) == 0;
    // pass 3
#pragma unroll 1
    for (int u = t; u < nunits; u += G) {
        float2 ua[4], ub[4], a[4], b[4], al[4], tv[4];
        unit(u, ua, ub, a, b, al, tv);
        const uint4 d = xd[u];
        float2 gx[4], gr[4], part[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 m = abs2(al[i]);
            const float2 dt = __fmul2_rn(__ffma2_rn(tv[i], nq, lo2(word4(d, i))), it2);
            const float2 da = __fmul2_rn(__fadd2_rn(one, fneg2(m)), dt), db = __fmul2_rn(m, dt);
            gx[i] = __fmul2_rn(__ffma2_rn(ua[i], nDa, da), ra2);
            gr[i] = __fmul2_rn(__ffma2_rn(ub[i], nDb, db), rb2);
            part[i] = __fmul2_rn(__fmul2_rn(sgn2(al[i]), __fadd2_rn(b[i], fneg2(a[i]))), dt);
        }
        const int valid = u < nfull ? 8 : tail;
        store8f(odx, u, gx, valid, a32);
        store8f(odr, u, gr, valid, a32);
        if (wsl != nullptr) {
            float *l = wsl + 8 * u;
            const float4 p0 = make_float4(part[0].x, part[0].y, part[1].x, part[1].y);
            const float4 p1 = make_float4(part[2].x, part[2].y, part[3].x, part[3].y);
            if (ws_first) {
                st16(l, as_u4(p0));
                st16(l + 4, as_u4(p1));
            } else {
                red_add4(l, p0);
                red_add4(l + 4, p1);
            }
        }
    }
}

// ============================================================ Dory rows ==
//
// Gated and SwiGLU rows, then their l2 over the whole row (a pair of warps
// per row, as tile_l2_row).  Pass 1 forms the row's bf16 value s from the
// two staged inputs (a, b) and the scale vectors, writes it back over a in
// the slot and sums s^2; pass 2 is l2's.  Every fp32 step is the one the
// definition names, in its order, with no contraction:
//   gate:   z = b sa, e = expf(-z), sig = 1 / (1 + e), s = bf16(a sig)
//   swiglu: gs = bf16(a sa), us = bf16(b sb), sl = gs / (1 + expf(-gs)),
//           s = bf16(sl us)
//
// The IEEE reciprocal and quotient come from Markstein's fused multiply-add
// iteration (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990): from y0,
// the hardware's approximate reciprocal of d, y = y0 + y0 (1 - d y0) is 1/d
// rounded to nearest, and with q = RN(x y), q + y (x - d q) is x/d rounded to
// nearest; the quotient takes x's sign, so that -0 stays -0.  This runs where
// every d of the unit lies in [1, 2^126) (no subnormal reciprocal) and, for
// silu, no x is +inf; any other unit takes __frcp_rn / __fdiv_rn.  On that
// range both agree with IEEE division for every fp32 input, which
// ds_debug_division_check counts on the device.
__device__ __forceinline__ float2 rcp_approx2(float2 d)
{
    float2 y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.x) : "f"(d.x));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.y) : "f"(d.y));
    return y;
}

__device__ __forceinline__ float2 neg2(float2 v) { return f2(-v.x, -v.y); }

// 1/d, d in [1, 2^126)
__device__ __forceinline__ float2 rcp_fast2(float2 d)
{
    const float2 y0 = rcp_approx2(d);
    const float2 e = __ffma2_rn(neg2(d), y0, f2(1.f, 1.f));
    return __ffma2_rn(e, y0, y0);
}

__device__ __forceinline__ float copy_sign_bit(float q, float x)
{
    return __int_as_float((__float_as_int(q) & 0x7fffffff) | (__float_as_int(x) & int(0x80000000u)));
}

// x/d from y = RN(1/d), d in [1, 2^126), x finite
__device__ __forceinline__ float2 div_fast2(float2 x, float2 d, float2 y)
{
    const float2 q = __fmul2_rn(x, y);
    const float2 r = __ffma2_rn(neg2(d), q, x);
    const float2 v = __ffma2_rn(r, y, q);
    return f2(copy_sign_bit(v.x, x.x), copy_sign_bit(v.y, x.y));
}

constexpr uint32_t kFastDLimit = 0x7E800000u; // bits of 2^126

// Words (pairs of columns) that share one range check: fewer keep fewer
// values live across the check.
constexpr int kFusedCheckWords = 4;

template <int PRO>
__device__ __forceinline__ uint4 fused_unit(uint4 a, uint4 b, const float2 (&sa)[4], const float2 (&sb)[4])
{
    constexpr int H = kFusedCheckWords;
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; h += H) {
        float2 x[H], d[H], m[H]; // gate: m = a; swiglu: x = gs, m = us
        uint32_t dmax = 0;
        int xmax = int(0x80000000u);
#pragma unroll
        for (int k = 0; k < H; ++k) {
            const int i = h + k;
            if constexpr (PRO == 0) {
                const float2 z = __fmul2_rn(lo2(word4(b, i)), sa[i]);
                d[k] = __fadd2_rn(f2(1.f, 1.f), f2(expf(-z.x), expf(-z.y)));
                m[k] = lo2(word4(a, i));
            } else {
                x[k] = lo2(pk(__fmul2_rn(lo2(word4(a, i)), sa[i])));
                m[k] = lo2(pk(__fmul2_rn(lo2(word4(b, i)), sb[i])));
                d[k] = __fadd2_rn(f2(1.f, 1.f), f2(expf(-x[k].x), expf(-x[k].y)));
                xmax = max(xmax, max(__float_as_int(x[k].x), __float_as_int(x[k].y)));
            }
            dmax = max(dmax, max(__float_as_uint(d[k].x), __float_as_uint(d[k].y)));
        }
        // unsigned bits order d >= 1 and put NaN past every finite d; signed
        // bits put +inf past every other x
        const bool fast = dmax < kFastDLimit && (PRO == 0 || xmax < 0x7F800000);
        if (fast) {
#pragma unroll
            for (int k = 0; k < H; ++k) {
                const float2 y = rcp_fast2(d[k]);
                if constexpr (PRO == 0)
                    w[h + k] = pk(__fmul2_rn(m[k], y));
                else
                    w[h + k] = pk(__fmul2_rn(div_fast2(x[k], d[k], y), m[k]));
            }
        } else {
#pragma unroll
            for (int k = 0; k < H; ++k) {
                if constexpr (PRO == 0)
                    w[h + k] = pack_bf2(__fmul_rn(m[k].x, __frcp_rn(d[k].x)), __fmul_rn(m[k].y, __frcp_rn(d[k].y)));
                else
                    w[h + k] = pack_bf2(__fmul_rn(__fdiv_rn(x[k].x, d[k].x), m[k].x),
                                        __fmul_rn(__fdiv_rn(x[k].y, d[k].y), m[k].y));
            }
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Every fp32 bit pattern v as the gate argument z = v and as silu's x = v:
// counts[0] / counts[1] = inputs where the fast reciprocal / quotient runs
// and its bits differ from __frcp_rn / __fdiv_rn; counts[2] / counts[3] =
// inputs where it runs.
__global__ void __launch_bounds__(256) k_division_check(unsigned long long *counts)
{
    unsigned long long bad_r = 0, bad_q = 0, n_r = 0, n_q = 0;
    const uint64_t step = uint64_t(gridDim.x) * blockDim.x;
    for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < (uint64_t(1) << 32); i += 2 * step) {
        // two inputs per iteration through the packed forms
        const uint64_t j = i + step < (uint64_t(1) << 32) ? i + step : i;
        const float2 v = f2(__uint_as_float(uint32_t(i)), __uint_as_float(uint32_t(j)));
        const float2 d = __fadd2_rn(f2(1.f, 1.f), f2(expf(-v.x), expf(-v.y)));
        const float2 y = rcp_fast2(d);
        const float2 q = div_fast2(v, d, y);
        const float dd[2] = {d.x, d.y}, yy[2] = {y.x, y.y}, qq[2] = {q.x, q.y}, vv[2] = {v.x, v.y};
        const int nk = j == i ? 1 : 2;
        for (int k = 0; k < nk; ++k) {
            if (__float_as_uint(dd[k]) >= kFastDLimit)
                continue;
            ++n_r;
            bad_r += __float_as_uint(yy[k]) != __float_as_uint(__frcp_rn(dd[k]));
            if (__float_as_int(vv[k]) >= 0x7F800000)
                continue;
            ++n_q;
            bad_q += __float_as_uint(qq[k]) != __float_as_uint(__fdiv_rn(vv[k], dd[k]));
        }
    }
    atomicAdd(&counts[0], bad_r);
    atomicAdd(&counts[1], bad_q);
    atomicAdd(&counts[2], n_r);
    atomicAdd(&counts[3], n_q);
}

template <int WP, int PRO, bool CACHED, bool SPLIT>
__device__ __forceinline__ void tile_fused_row(Team<WP, SPLIT> &tm, const ASegK &sg, int64_t row, unsigned char *s0,
                                               const unsigned char *s1, int nfull, int tail, float eps, bool store,
                                               const float *ca, const float *cb, int half)
{
    constexpr int G = Team<WP>::G;
    const int t = tm.t;
    const bool tl = tail && t == nfull % G;
    const int nunits = nfull + (tail ? 1 : 0);
    uint4 *x = reinterpret_cast<uint4 *>(s0);
    const uint4 *r = reinterpret_cast<const uint4 *>(s1);
    float2 acc = f2(0.f, 0.f);
#pragma unroll 1
    for (int u = t; u < nunits; u += G) {
        float2 va[4], vb[4];
        alpha8_signed<CACHED>(ca, half, sg.alpha, u, sg.cols, va);
        if constexpr (PRO == 1)
            alpha8_signed<CACHED>(cb, half, sg.s2, u, sg.cols, vb);
        else
#pragma unroll
            for (int i = 0; i < 4; ++i)
                vb[i] = f2(0.f, 0.f);
        uint4 sv = fused_unit<PRO>(x[u], r[u], va, vb);
        if (u == nfull && tl)
            sv = mask_octet(sv, tail);
        x[u] = sv;
        sq8w(acc, sv);
    }
    const float S = tm.sum1(acc.x + acc.y);
    const RowScale rs = tile_scale(tm, S, eps, [&](auto f) {
        for (int u = t; u < nunits; u += G)
            pairs8(x[u], f);
    });
    if (!store || !tm.good())
        return;
    uint16_t *y = sg.y + row * sg.ld;
#pragma unroll 4
    for (int u = t; u < nfull; u += G)
        st16(y + 8 * u, scale8(x[u], rs));
    if (tl)
        store_tail8(y + 8 * nfull, scale8(x[nfull], rs), tail);
}

// =============================================================== kernel ==

template <int T>
using TParams = typename std::conditional<is_weight_tag(T), WParams,
                                          typename std::conditional<is_act_bwd_tag(T), GParams, AParams>::type>::type;

// Ring shape per operation and slot size SB (16, 32 or 64 KB of staged
// input per slot; 112 KB for weight rows).  A position is owned by a team
// of warps that reduce each row together: one warp (weight calls) or a pair
// (activation calls, more work per byte) at 16 KB, and proportionally more
// warps for the larger slots, so that every thread holds about the same
// number of units per row.  The ring keeps ~200 KB in flight: 13, 6, 3 or 2
// positions.  slerp caches |alpha|
// in the shared memory left over (4,096 columns at 16 KB, 8,192 otherwise).
template <int T, int SB>
struct TileCfg {
    static_assert(SB == 16384 || SB == 32768 || SB == 65536 || SB == 114688, "slot size");
    static_assert(SB != 114688 || is_weight_tag(T), "112 KB slots: weight rows only");
    static constexpr int kSlotBytes = SB;
    static constexpr int kScale = SB == 114688 ? 8 : SB / 16384;    // 1, 2, 4; 8 for 112 KB
    static constexpr int kWP = (is_act_tag(T) ? 2 : 1) * kScale;
    // SwiGLU rows keep two scale vectors in shared memory: one position fewer;
    // the slerp backward in 32 KB slots takes one fewer too, so that its
    // 672 threads get 80 registers each (800 threads get 72 and spill)
    static constexpr int kGroups = SB == 16384 ? (T == tSwigluL2 ? 12 : 13)
                                   : SB == 32768 ? ((T == tSwigluL2 || T == tSlerpBwd) ? 5 : 6)
                                   : SB == 65536 ? 3 : 2;
    static constexpr int kSlots = kGroups;                          // one position per team
    static constexpr int kConsumers = kWP * kGroups;
    static constexpr int kThreads = (kConsumers + 1) * 32;
    // Columns of each per-column vector held in shared memory after the ring
    // (slerp: alpha; Dory rows: the scale vectors, none in 64 KB slots)
    static constexpr int kAlphaCache = (T == tSlerp || T == tSlerpBwd) ? (SB == 16384 ? 4096 : 8192)
                                       : (T == tGateL2 || T == tSwigluL2) ? (SB == 16384 ? 4096 : SB == 32768 ? 8192 : 0)
                                                                         : 0;
    static constexpr int kVecs = T == tSwigluL2 ? 2 : 1;
    // Refill pacing: the producer sleeps this long after each refill.  For
    // the operations below a paced read stream ran faster on B200 (l2 rows
    // with a residual 74 -> 67 us, the momentum projection + renorm 274 ->
    // 250 us, backward in 32 KB slots 97 -> 91 us on the benchmark shapes);
    // for the others it only slowed them, so they refill at once.
    static constexpr unsigned kPaceNs =
        ((SB == 16384 && (T == tL2 || T == tMomentum)) || (SB == 32768 && (T == tBwdBf16 || T == tBwdF32))) ? 300
                                                                                                           : 0;
    static_assert(kSlots <= kMaxTileSlots && kConsumers + 1 <= 32, "ring shape");
    static constexpr int kSmem = SB * kSlots + 4 * kAlphaCache * kVecs;
    static_assert(kSmem <= 229376, "ring and vector caches fit 224 KB");
};

// The rows of one slot, each through its operation's row body.  `sg` is
// the segment, or with a row split over a cluster the view of this CTA's
// slice; `wsl` the team's dalpha line (slerp backward) at the slice's
// first column.
template <int T, int SB, bool SPLIT, int WP, class Seg>
__device__ __forceinline__ void tile_rows(Team<WP, SPLIT> &tm, const Seg &sg, const TParams<T> &p, const SlotHdr &h,
                                          unsigned char *base, unsigned char *a1, unsigned char *a2p, int pitch0,
                                          int pitch1, int pitch2, int nfull, int tail, bool store, bool &ws_first,
                                          float *s_alpha, int acache, float *wsl)
{
    using Cfg = TileCfg<T, SB>;
    const int lane = threadIdx.x & 31;
    const bool has_r = seg_has_r(sg);
    float g_lane = 1.f;
            for (int r = 0; r < h.nrows; ++r) {
                const int64_t row = h.row0 + r;
                unsigned char *s0 = base + r * pitch0;
                unsigned char *s1 = a1 + r * pitch1;
                unsigned char *s2 = a2p + r * pitch2;
                if constexpr (T == tFwdBf16 || T == tFwdF32 || T == tBwdBf16 || T == tBwdF32) {
                    // gains of the next 32 rows, one per lane
                    if ((r & 31) == 0)
                        g_lane = (sg.gain && r + lane < h.nrows) ? __ldg(sg.gain + (row + lane) * sg.gain_stride) : 1.f;
                }
                const float g = __shfl_sync(0xffffffffu, g_lane, r & 31);
                if constexpr (T == tFwdBf16)
                    tile_scale_row<true, false>(tm, sg, row, g, s0, nfull, tail, p.eps, store);
                else if constexpr (T == tFwdF32)
                    tile_scale_row<false, false>(tm, sg, row, g, s0, nfull, tail, p.eps, store);
                else if constexpr (T == tRenorm)
                    tile_scale_row<false, true>(tm, sg, row, 1.f, s0, nfull, tail, p.eps, store);
                else if constexpr (T == tNorms)
                    tile_norm_row(tm, sg, row, s0, nfull, tail, p.eps, store);
                else if constexpr (T == tBwdBf16)
                    tile_backward_row<true, 0>(tm, sg, row, g, s0, s1, nfull, tail, p.eps, store);
                else if constexpr (T == tBwdF32)
                    tile_backward_row<false, 0>(tm, sg, row, g, s0, s1, nfull, tail, p.eps, store);
                else if constexpr (T == tProject)
                    tile_backward_row<false, 1>(tm, sg, row, 1.f, s0, s1, nfull, tail, p.eps, store);
                else if constexpr (T == tMomentum)
                    tile_backward_row<false, 2>(tm, sg, row, 1.f, s0, s1, nfull, tail, p.eps, store);
                else if constexpr (T == tL2) {
                    if (has_r)
                        tile_l2_row<WP, true>(tm, sg, row, s0, s1, nfull, tail, p.eps, store);
                    else
                        tile_l2_row<WP, false>(tm, sg, row, s0, s1, nfull, tail, p.eps, store);
                } else if constexpr (T == tGateL2 || T == tSwigluL2) {
                    constexpr int PRO = T == tGateL2 ? 0 : 1;
                    constexpr int H = Cfg::kAlphaCache / 2;
                    if (acache == kAlphaAll && (PRO == 0 || p.alpha2_shared))
                        tile_fused_row<WP, PRO, true>(tm, sg, row, s0, s1, nfull, tail, p.eps, store, s_alpha,
                                                      s_alpha + Cfg::kAlphaCache, H);
                    else
                        tile_fused_row<WP, PRO, false>(tm, sg, row, s0, s1, nfull, tail, p.eps, store, nullptr,
                                                       nullptr, 0);
                } else if constexpr (T == tL2Bwd) {
                    if (has_r)
                        tile_l2_bwd_row<WP, true>(tm, sg, row, s0, s1, s2, nfull, tail, p.eps, store);
                    else
                        tile_l2_bwd_row<WP, false>(tm, sg, row, s0, s1, s2, nfull, tail, p.eps, store);
                } else if constexpr (T == tSlerpBwd) {
                    if (acache == kAlphaAll)
                        tile_slerp_bwd_row<WP, true>(tm, sg, row, s0, s1, s2, nfull, tail, p.eps, store, s_alpha,
                                                     Cfg::kAlphaCache / 2, wsl, ws_first);
                    else
                        tile_slerp_bwd_row<WP, false>(tm, sg, row, s0, s1, s2, nfull, tail, p.eps, store, nullptr, 0,
                                                      wsl, ws_first);
                    ws_first = false;
                } else if (acache == kAlphaAll) {
                    tile_slerp_row<WP, kAlphaAll>(tm, sg, row, s0, s1, nfull, tail, p.eps, store, s_alpha,
                                                  Cfg::kAlphaCache / 2);
                } else if (acache == kAlphaHead) {
                    tile_slerp_row<WP, kAlphaHead>(tm, sg, row, s0, s1, nfull, tail, p.eps, store, s_alpha,
                                                   Cfg::kAlphaCache / 2);
                } else {
                    tile_slerp_row<WP, kAlphaNone>(tm, sg, row, s0, s1, nfull, tail, p.eps, store, nullptr, 0);
                }
            }
}

// Segment view of CTA `rank`'s slice of every row: the row pointers (and
// the per-column vectors) moved to column c0 and the row length cut to the
// slice's `cols` columns in `nu` units (per-row vectors -- gains, grad_g --
// stay), so that a row body sees the slice as a row of its own; the
// per-column vectors are then read only up to the slice's end.
template <int T>
__device__ __forceinline__ WSegK shifted(const WSegK &s, int c0, int cols, int nu)
{
    WSegK k = s;
    k.cols = cols;
    k.nu = nu;
    constexpr int oe = (T == tFwdBf16 || T == tBwdBf16) ? 2 : 4; // bytes of an element of out / gy
    k.w = s.w + c0;
    if (s.out)
        k.out = static_cast<char *>(s.out) + static_cast<int64_t>(c0) * (T == tRenorm || T == tProject ||
                                                                        T == tMomentum ? 4 : oe);
    if (s.gy)
        k.gy = static_cast<const char *>(s.gy) + static_cast<int64_t>(c0) * (T == tBwdBf16 ? 2 : 4);
    if (s.grad_w)
        k.grad_w = s.grad_w + c0;
    return k;
}

template <int T>
__device__ __forceinline__ ASegK shifted(const ASegK &s, int c0, int cols, int nu)
{
    ASegK k = s;
    k.cols = cols;
    k.nu = nu;
    k.x = s.x + c0;
    if (s.r)
        k.r = s.r + c0;
    k.y = s.y + c0;
    if (s.alpha)
        k.alpha = s.alpha + c0;
    if (s.s2)
        k.s2 = s.s2 + c0;
    return k;
}

template <int T>
__device__ __forceinline__ AGSegK shifted(const AGSegK &s, int c0, int cols, int nu)
{
    AGSegK k = s;
    k.cols = cols;
    k.nu = nu;
    k.x = s.x + c0;
    if (s.r)
        k.r = s.r + c0;
    k.dy = s.dy + c0;
    k.dx = s.dx + c0;
    if (s.dr)
        k.dr = s.dr + c0;
    if (s.alpha)
        k.alpha = s.alpha + c0;
    return k;
}

// Exchange area bytes of a staged launch whose rows are split over a
// cluster (after the ring and the vector caches); none for one CTA per row.
template <int T, int SB>
constexpr int tile_xchg_bytes()
{
    return TileCfg<T, SB>::kGroups * kXchgBytesPerTeam;
}

// The staged kernel.  One CTA per SM; with a cluster launch (2, 4 or 8 CTAs
// per cluster) the cluster's CTAs walk the same slots, each staging and
// normalising its slice of the rows (slice_per), and the teams' reductions
// meet through distributed shared memory.
template <int T, int SB, bool SPLIT>
__global__ void __launch_bounds__(TileCfg<T, SB>::kThreads, 1)
    k_tile(const __grid_constant__ TParams<T> p)
{
    using Cfg = TileCfg<T, SB>;
    constexpr int slot_bytes = SB;
    constexpr int WP = Cfg::kWP;
    constexpr int nslots = Cfg::kSlots;
    constexpr int E = is_weight_tag(T) ? 4 : 8;   // elements per 16-byte unit of array 0
    extern __shared__ __align__(128) unsigned char ring[];
    __shared__ __align__(8) uint64_t full[nslots];
    __shared__ __align__(8) uint64_t empty[nslots];
    __shared__ SlotHdr hdr[nslots];
    __shared__ float red[Cfg::kGroups * Team<WP>::kRed]; // team reductions
    __shared__ int vote[Cfg::kGroups * 2 * WP];           // team agreement on a wait: [team][2][warp]
    __shared__ volatile int abort_flag;                    // set by the first wait that runs out (or by a peer)
    // slerp: |alpha| of the launch's (single) alpha vector, after the ring
    float *s_alpha = reinterpret_cast<float *>(ring + static_cast<size_t>(nslots) * slot_bytes);
    // rows split over a cluster: the teams' exchange areas after the caches
    unsigned char *xarea = ring + Cfg::kSmem;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t ncta = SPLIT ? cluster_nctarank() : 1u, rank = SPLIT ? cluster_ctarank() : 0u;
    constexpr bool split = SPLIT;
    const int64_t cid = blockIdx.x / ncta, ncl = gridDim.x / ncta;   // this cluster, the clusters
    const int64_t total = p.unit_start[p.nseg];
    // this cluster's slots: cid, cid + ncl, ...
    const int64_t mine = total > cid ? (total - 1 - cid) / ncl + 1 : 0;
    const ClusterCtx ctx{rank, ncta, &abort_flag, p.wait_limit_ns};

    if (threadIdx.x == 0) {
        for (int s = 0; s < nslots; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], WP); // every warp of the owning team arrives
        }
        if (split)
            for (int q = 0; q < Cfg::kGroups; ++q) {
                uint64_t *xb = reinterpret_cast<uint64_t *>(xarea + q * kXchgBytesPerTeam + kXchgFloats * 4);
                mbar_init(&xb[0], 1); // the team's own arrival, with the peers' store bytes
                mbar_init(&xb[1], 1);
            }
        abort_flag = 0;
        mbar_init_fence();
    }
    // |alpha| (slerp), alpha (slerp backward) or the scale vectors (Dory
    // rows) of this CTA's slice of the columns, when every segment of the
    // launch shares them and the slice fits the cache
    int acols = p.alpha_cols, ac0 = 0;
    if (SPLIT && p.alpha_shared) {
        const int anu = (p.alpha_cols + 7) / 8, aper = slice_per(anu, static_cast<int>(ncta));
        const int au0 = min(anu, static_cast<int>(rank) * aper), au1 = min(anu, au0 + aper);
        ac0 = 8 * au0;
        acols = max(0, min(p.alpha_cols - ac0, 8 * (au1 - au0)));
    }
    // (one CTA per row: read from the parameters where it is used).  The
    // slerp forward caches the head of a longer |alpha| and reads the rest.
    auto cached = [&]() {
        if (p.alpha_shared == nullptr || Cfg::kAlphaCache == 0)
            return static_cast<int>(kAlphaNone);
        if ((SPLIT ? acols : p.alpha_cols) <= Cfg::kAlphaCache)
            return static_cast<int>(kAlphaAll);
        return static_cast<int>(T == tSlerp ? kAlphaHead : kAlphaNone);
    };
    const int acache = cached();
    if constexpr (T == tSlerp || T == tSlerpBwd) {
        // |alpha| split by halves of each 8-element unit: unit u's first four
        // at [4u], its last four at [half + 4u], so that a warp reading one
        // float4 per lane touches consecutive 16-byte words (no bank conflict)
        if (acache != kAlphaNone) {
            const int nu = min((acols + 7) / 8, Cfg::kAlphaCache / 8), half = Cfg::kAlphaCache / 2;
            for (int i = threadIdx.x; i < 8 * nu; i += blockDim.x) {
                const int u = i >> 3, e = i & 7;
                // the backward keeps the sign (dalpha needs it); the forward |alpha|
                const float a = i < acols ? __ldg(p.alpha_shared + ac0 + i) : 0.f;
                const float v = T == tSlerpBwd ? a : fabsf(a);
                s_alpha[(e < 4 ? 0 : half) + 4 * u + (e & 3)] = v;
            }
        }
    }
    if constexpr (T == tGateL2 || T == tSwigluL2) {
        // the scale vectors in the same split layout, sb after sa
        if (acache == kAlphaAll && (T == tGateL2 || p.alpha2_shared)) {
            const int nu = (acols + 7) / 8, half = Cfg::kAlphaCache / 2;
            for (int i = threadIdx.x; i < 8 * nu; i += blockDim.x) {
                const int u = i >> 3, e = i & 7, at = (e < 4 ? 0 : half) + 4 * u + (e & 3);
                s_alpha[at] = i < acols ? __ldg(p.alpha_shared + ac0 + i) : 0.f;
                if constexpr (T == tSwigluL2)
                    s_alpha[Cfg::kAlphaCache + at] = i < acols ? __ldg(p.alpha2_shared + ac0 + i) : 0.f;
            }
        }
    }
    __syncthreads();
    if (split) {
        // every CTA of the cluster has initialised its barriers before any
        // peer arrives on them
        cluster_arrive();
        cluster_wait();
    }

    using Layout = TileLayout<T>;
    bool ok = true;

    if (warp == Cfg::kConsumers) {
        // ------------------------------------------------------ producer --
        // One thread.  Its per-slot work sits between a consumer's release
        // and the refill it waits for, so it is kept short: position,
        // phase and slot advance incrementally, and the current segment's
        // copy geometry is cached in registers until the walk leaves it.
        // (The consumers fence their generic-proxy writes to a slot before
        // releasing it, so the refill needs no fence here.)
        if (lane == 0) {
            int si = -1;
            int64_t seg_begin = 0, seg_end = 0, seg_rows = 0;
            int rps = 1;
            constexpr int NA = Layout::kArrays;
            uint32_t pitch[NA], off[NA];
            const char *src[NA];
            int64_t spitch[NA];
            bool contig[NA];
#pragma unroll
            for (int a2 = 0; a2 < NA; ++a2) {
                pitch[a2] = off[a2] = 0u;
                src[a2] = nullptr;
                spitch[a2] = 0;
                contig[a2] = false;
            }
            int s = 0;
            uint32_t phase = 0;             // parity of the release a refill of position s waits for
            int64_t slot = cid;
            for (int64_t j = 0; j < mine; ++j, slot += ncl) {
                if (j >= nslots && (abort_flag || !mbar_wait_bounded(&empty[s], phase, p.wait_limit_ns))) {
                    ok = false;
                    if (split && !abort_flag)
                        ctx.abort_all();
                    abort_flag = 1;
                    break;
                }
                if (slot >= seg_end) {      // slots increase: walk forward to the slot's segment
                    do {
                        ++si;
                        seg_end = p.unit_start[si + 1];
                    } while (seg_end <= slot);
                    seg_begin = p.unit_start[si];
                    const auto &sg = p.seg[si];
                    seg_rows = sg.rows;
                    rps = sg.group;         // rows per slot for this segment
                    const bool has_r = seg_has_r(sg);
                    // this CTA's slice of the row: units [u0, u0 + nuk)
                    const int per = slice_per(sg.nu, static_cast<int>(ncta));
                    const int u0 = min(sg.nu, static_cast<int>(rank) * per);
                    const int nuk = min(sg.nu, u0 + per) - u0;
                    uint32_t o = 0u;
#pragma unroll
                    for (int a2 = 0; a2 < NA; ++a2) {
                        const int u = Layout::ub(a2, has_r);
                        pitch[a2] = (static_cast<uint32_t>(nuk) * u + 15u) & ~15u;
                        src[a2] = pitch[a2] ? tile_src<T>(sg, a2, 0) + static_cast<int64_t>(u0) * u : nullptr;
                        spitch[a2] = tile_src_pitch<T>(sg, a2);
                        contig[a2] = !split && spitch[a2] == static_cast<int64_t>(pitch[a2]);
                        off[a2] = o;
                        o += pitch[a2] * rps;
                    }
                }
                const int64_t row0 = (slot - seg_begin) * rps;
                const int nrows = static_cast<int>(seg_rows - row0 < rps ? seg_rows - row0 : rps);
                hdr[s] = SlotHdr{si, nrows, row0};
                unsigned char *dst = ring + static_cast<size_t>(s) * slot_bytes;
                uint32_t row_bytes = 0u;
#pragma unroll
                for (int a2 = 0; a2 < NA; ++a2)
                    row_bytes += pitch[a2];
                mbar_arrive_expect_tx(&full[s], row_bytes * nrows);
#pragma unroll
                for (int a2 = 0; a2 < NA; ++a2) {
                    if (!pitch[a2])
                        continue;
                    unsigned char *d = dst + off[a2];
                    const char *g = src[a2] + row0 * spitch[a2];
                    if (contig[a2]) {
                        bulk_g2s(d, g, pitch[a2] * nrows, &full[s]);
                    } else {
                        for (int r = 0; r < nrows; ++r)
                            bulk_g2s(d + r * pitch[a2], g + r * spitch[a2], pitch[a2], &full[s]);
                    }
                }
                if constexpr (Cfg::kPaceNs != 0)
                    __nanosleep(Cfg::kPaceNs);
                if (++s == nslots) {        // a round of the ring ends; rounds 2, 3, ...
                    s = 0;                  // wait for releases of parity 0, 1, 0, ...
                    if (j >= 2 * nslots - 1)
                        phase ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------------ consumers --
        // team q (one warp, or WP warps) owns ring positions q, q + kGroups,
        // ...; the CTA's slot j sits at position j % nslots, so the team
        // takes slots j = q, q + kGroups, ... in order
        constexpr int NG = Cfg::kGroups;
        const int q = warp / WP, wi = warp % WP;
        Team<WP, SPLIT> tm{wi * 32 + lane, 1 + q, red + q * Team<WP>::kRed};
        if constexpr (SPLIT) {
            tm.ctx = &ctx;
            tm.xrank = rank;
            tm.xn = ncta;
            tm.xbuf = reinterpret_cast<float *>(xarea + q * kXchgBytesPerTeam);
            tm.xbar = reinterpret_cast<uint64_t *>(xarea + q * kXchgBytesPerTeam + kXchgFloats * 4);
        }
        bool store = true;
        bool ws_first = true; // slerp backward: this team's dalpha line not yet written
        int vb = 0;
        for (int64_t j = q; j < mine; j += NG, vb ^= 1) {
            const int s = static_cast<int>(j % nslots);
            const uint32_t phase = static_cast<uint32_t>((j / nslots) & 1);
            bool got = !abort_flag && !tm.failed && mbar_wait_bounded(&full[s], phase, p.wait_limit_ns);
            got = __all_sync(0xffffffffu, got);
            if constexpr (WP > 1) {
                // all warps of the team take the same decision (their row
                // barriers need each other)
                int *v = vote + (q * 2 + vb) * WP;
                if (lane == 0)
                    v[wi] = got;
                named_sync(tm.bar, Team<WP>::G);
#pragma unroll
                for (int w = 0; w < WP; ++w)
                    got = got && v[w];
            }
            if (!got) {
                // nothing more will arrive: store nothing from here on, but
                // keep releasing positions so that every wait ends; the
                // peers of a cluster are told, so that none waits for this
                // CTA's part of an exchange
                ok = false;
                if (split && !abort_flag && tm.t == 0)
                    ctx.abort_all();
                abort_flag = 1;
                store = false;
            }
            const SlotHdr h = got ? hdr[s] : SlotHdr{0, 0, 0};
            const auto &sg0 = p.seg[h.seg];
            const bool has_r = seg_has_r(sg0);
            const int rps = sg0.group;
            // this CTA's slice of the rows
            int nuk = sg0.nu, c0 = 0, colsk = sg0.cols;
            if constexpr (SPLIT) {
                const int per = slice_per(sg0.nu, static_cast<int>(ncta));
                const int ub0 = min(sg0.nu, static_cast<int>(rank) * per);
                nuk = min(sg0.nu, ub0 + per) - ub0;
                c0 = E * ub0;
                colsk = max(0, min(sg0.cols - c0, E * nuk));
            }
            unsigned char *base = ring + static_cast<size_t>(s) * slot_bytes;
            const int u0 = Layout::ub(0, has_r), u1 = Layout::kArrays > 1 ? Layout::ub(1, has_r) : 0;
            const int u2 = Layout::kArrays > 2 ? Layout::ub(2, has_r) : 0;
            const int pitch0 = (nuk * u0 + 15) & ~15;
            const int pitch1 = (nuk * u1 + 15) & ~15;
            const int pitch2 = (nuk * u2 + 15) & ~15;
            unsigned char *a1 = base + pitch0 * rps;
            unsigned char *a2p = a1 + pitch1 * rps;
            const int nfull = colsk / E, tail = colsk % E;
            // hand the position back: the slot may hold this warp's
            // generic-proxy writes (s, t, masked tails), so order them
            // before the next bulk copy into it
            bool released = false;
            auto release = [&]() {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&empty[s]);
                released = true;
            };
            // the rows, through the segment itself or (a slice per CTA) a
            // view of it moved to the slice's first column
            if constexpr (SPLIT)
                tile_rows<T, SB, SPLIT>(tm, shifted<T>(sg0, c0, colsk, nuk), p, h, base, a1, a2p, pitch0, pitch1,
                                        pitch2, nfull, tail, store, ws_first, s_alpha, acache,
                                        p.ws ? p.ws + (cid * NG + q) * p.ws_ld + c0 : nullptr);
            else
                tile_rows<T, SB, SPLIT>(tm, sg0, p, h, base, a1, a2p, pitch0, pitch1, pitch2, nfull, tail, store,
                                        ws_first, s_alpha, acache,
                                        p.ws ? p.ws + (static_cast<int64_t>(blockIdx.x) * NG + q) * p.ws_ld : nullptr);
            if (!released)
                release();
        }
        if (tm.failed)
            ok = false;
    }
    if (!ok)
        raise_device_error(DS_ERR_DEVICE_TIMEOUT, kSiteTileWait);
    if (split) {
        // no CTA leaves while a peer may still write into its shared memory
        __syncwarp();
        cluster_arrive();
        cluster_wait();
    }
}

} // namespace

// Clusters of `cluster` CTAs of k_tile<T, SB> that fit the device at once,
// looked up once per device and cluster size.
template <int T, int SB>
static cudaError_t resident_clusters(int cluster, int smem, int *n)
{
    static std::atomic<int> cache[64][4];
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    const int ci = cluster == 2 ? 0 : cluster == 4 ? 1 : cluster == 8 ? 2 : 3;
    if (dev >= 0 && dev < 64 && ci < 3) {
        const int c = cache[dev][ci].load(std::memory_order_relaxed);
        if (c > 0) {
            *n = c;
            return cudaSuccess;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cluster), 1, 1);
    cfg.blockDim = dim3(TileCfg<T, SB>::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    e = cudaOccupancyMaxActiveClusters(&c, k_tile<T, SB, true>, &cfg);
    if (e != cudaSuccess)
        return e;
    if (c <= 0)
        return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64 && ci < 3)
        cache[dev][ci].store(c, std::memory_order_relaxed);
    *n = c;
    return cudaSuccess;
}

static int device_sms()
{
    static std::atomic<int> cache[64];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int T, int SB>
static cudaError_t launch_tile_sb(const TParams<T> &p, int64_t units, int cluster, int *used, void *stream)
{
    using Cfg = TileCfg<T, SB>;
    if (cluster == 1) {
        constexpr int smem = Cfg::kSmem;
        static DeviceFlags attr_set;
        if (const cudaError_t e = enable_dynamic_smem(k_tile<T, SB, false>, smem, attr_set))
            return e;
        const int grid = static_cast<int>(std::min<int64_t>(device_sms(), units));
        *used = grid;
        k_tile<T, SB, false><<<grid, Cfg::kThreads, smem, static_cast<cudaStream_t>(stream)>>>(p);
        return cudaGetLastError();
    }
    if constexpr (SB > kTileSlotMaxBytes) {
        return cudaErrorInvalidValue;   // slices of a row split over a cluster take at most 64 KB
    } else {
        constexpr int smem = Cfg::kSmem + tile_xchg_bytes<T, SB>();
        static DeviceFlags attr_set;
        if (const cudaError_t e = enable_dynamic_smem(k_tile<T, SB, true>, smem, attr_set))
            return e;
        int resident = 0;
        if (const cudaError_t e = resident_clusters<T, SB>(cluster, smem, &resident))
            return e;
        const int64_t ncl = std::min<int64_t>(resident, units);
        *used = static_cast<int>(ncl);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(ncl * cluster), 1, 1);
        cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cfg.stream = static_cast<cudaStream_t>(stream);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, k_tile<T, SB, true>, p);
    }
}

template <int T>
static cudaError_t launch_tile_t(const void *params, int64_t units, int slot_bytes, int cluster, int *used,
                                 void *stream)
{
    const TParams<T> &p = *static_cast<const TParams<T> *>(params);
    if (cluster != 1 && cluster != 2 && cluster != 4 && cluster != 8)
        return cudaErrorInvalidValue;
    switch (slot_bytes) {
    case 16384: return launch_tile_sb<T, 16384>(p, units, cluster, used, stream);
    case 32768: return launch_tile_sb<T, 32768>(p, units, cluster, used, stream);
    case 65536: return launch_tile_sb<T, 65536>(p, units, cluster, used, stream);
    case 114688:
        if constexpr (is_weight_tag(T))
            return launch_tile_sb<T, 114688>(p, units, cluster, used, stream);
        else
            return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
    }
}

int launch_tile(int tag, const void *params, int64_t units, int slot_bytes, int cluster, int *used, void *stream)
{
    switch (tag) {
    case tFwdBf16: return launch_tile_t<tFwdBf16>(params, units, slot_bytes, cluster, used, stream);
    case tFwdF32: return launch_tile_t<tFwdF32>(params, units, slot_bytes, cluster, used, stream);
    case tBwdBf16: return launch_tile_t<tBwdBf16>(params, units, slot_bytes, cluster, used, stream);
    case tBwdF32: return launch_tile_t<tBwdF32>(params, units, slot_bytes, cluster, used, stream);
    case tRenorm: return launch_tile_t<tRenorm>(params, units, slot_bytes, cluster, used, stream);
    case tL2: return launch_tile_t<tL2>(params, units, slot_bytes, cluster, used, stream);
    case tSlerp: return launch_tile_t<tSlerp>(params, units, slot_bytes, cluster, used, stream);
    case tProject: return launch_tile_t<tProject>(params, units, slot_bytes, cluster, used, stream);
    case tMomentum: return launch_tile_t<tMomentum>(params, units, slot_bytes, cluster, used, stream);
    case tL2Bwd: return launch_tile_t<tL2Bwd>(params, units, slot_bytes, cluster, used, stream);
    case tSlerpBwd: return launch_tile_t<tSlerpBwd>(params, units, slot_bytes, cluster, used, stream);
    case tGateL2: return launch_tile_t<tGateL2>(params, units, slot_bytes, cluster, used, stream);
    case tSwigluL2: return launch_tile_t<tSwigluL2>(params, units, slot_bytes, cluster, used, stream);
    case tNorms: return launch_tile_t<tNorms>(params, units, slot_bytes, cluster, used, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <int T>
static int tile_groups_t(int slot_bytes)
{
    switch (slot_bytes) {
    case 16384: return TileCfg<T, 16384>::kGroups;
    case 32768: return TileCfg<T, 32768>::kGroups;
    case 65536: return TileCfg<T, 65536>::kGroups;
    default: return 0;
    }
}

int tile_read_and_clear_error(uint32_t *code, uint32_t *site) { return module_read_and_clear_error(code, site); }

int launch_division_check(unsigned long long *counts, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(counts, 0, 4 * sizeof(unsigned long long), st);
    if (e != cudaSuccess)
        return e;
    k_division_check<<<148 * 8, 256, 0, st>>>(counts);
    return cudaGetLastError();
}

int tile_groups(int tag, int slot_bytes)
{
    switch (tag) {
    case tL2Bwd: return tile_groups_t<tL2Bwd>(slot_bytes);
    case tSlerpBwd: return tile_groups_t<tSlerpBwd>(slot_bytes);
    case tGateL2: return tile_groups_t<tGateL2>(slot_bytes);
    case tSwigluL2: return tile_groups_t<tSwigluL2>(slot_bytes);
    default: return 0;
    }
}

namespace {

// dalpha of the slerp backward: the used teams' lines (line L = CTA *
// groups + team; a CTA's team q was used iff q < the CTA's slot count) are
// summed per column in a fixed order: thread row lg of a block adds lines
// lg, lg + 32, ... in increasing order, then the 32 partial sums meet in a
// fixed tree.  32 columns per block (one 128-byte segment of a line per
// warp), so a 4,096-column alpha spreads over 128 blocks of 1,024 threads.
__global__ void __launch_bounds__(1024) k_dalpha_reduce(const float *ws, int ws_ld, int grid, int groups,
                                                        int64_t total_units, int cols, float *dalpha)
{
    __shared__ float part[32][33];
    const int cg = threadIdx.x & 31, lg = threadIdx.x >> 5;
    const int c = blockIdx.x * 32 + cg;
    float acc = 0.f;
    if (c < cols) {
        const int nlines = grid * groups;
        for (int L = lg; L < nlines; L += 32) {
            const int cta = L / groups, q = L - cta * groups;
            const int64_t mine = total_units > cta ? (total_units - 1 - cta) / grid + 1 : 0;
            if (q < mine)
                acc += ws[static_cast<int64_t>(L) * ws_ld + c];
        }
    }
    part[lg][cg] = acc;
    __syncthreads();
    for (int o = 16; o > 0; o >>= 1) {
        if (lg < o)
            part[lg][cg] += part[lg + o][cg];
        __syncthreads();
    }
    if (lg == 0 && c < cols)
        dalpha[c] = part[0][cg];
}

} // namespace

// Built-in scratch for the no-alloc slerp backward entry point: one
// module-level device array (64 MB, enough for the dalpha lines of rows up to
// 8,712 columns on 148 SMs), present on every device that loads the library
// until the process exits.  Host code cannot use the array's name as a
// device address, so its address is looked up once per device, with that
// device current, and cached.  Calls that use it must not overlap in time.
static __device__ __align__(256) float g_builtin_scratch[kBuiltinScratchFloats];

int builtin_scratch(void **ptr, uint64_t *bytes)
{
    static DeviceFlags looked_up;
    static void *addr[64] = {};
    *ptr = nullptr;
    *bytes = static_cast<uint64_t>(kBuiltinScratchFloats) * sizeof(float);
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (looked_up.has(dev)) {
        *ptr = addr[dev];
        return cudaSuccess;
    }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_builtin_scratch);
    if (e != cudaSuccess)
        return e;
    if (dev >= 0 && dev < 64) {
        addr[dev] = p;     // written before the flag is published
        looked_up.set(dev);
    }
    *ptr = p;
    return cudaSuccess;
}

int launch_dalpha_reduce(const float *ws, int ws_ld, int grid, int groups, int64_t total_units, int cols,
                         float *dalpha, void *stream)
{
    k_dalpha_reduce<<<(cols + 31) / 32, 1024, 0, static_cast<cudaStream_t>(stream)>>>(ws, ws_ld, grid, groups,
                                                                                   total_units, cols, dalpha);
    return cudaGetLastError();
}

} // namespace ds
