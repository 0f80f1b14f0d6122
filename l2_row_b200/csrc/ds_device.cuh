// ds_device.cuh -- device building blocks for the row kernels (sm_100a):
// 16-byte loads and stores, bf16 packing, fixed-order reductions inside a
// warp, a CTA and a thread-block cluster (DSMEM), and bounded mbarrier waits
// for bulk (TMA) copies.
#pragma once

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ds_internal.h"

namespace ds {

// The device error word.  Without relocatable device code every .cu file
// that includes this header is a module of its own with its own copy, so
// each module exports a reader (module_read_and_clear_error) and the host
// reads them all.
__device__ uint32_t g_device_error[4]; // [0] status code, [1] site, [2] block

__device__ __forceinline__ void raise_device_error(uint32_t code, uint32_t site)
{
    if (atomicCAS(&g_device_error[0], 0u, code) == 0u) {
        g_device_error[1] = site;
        g_device_error[2] = blockIdx.x;
    }
}

// This module's word, read and cleared (the caller has synchronised).
static inline int module_read_and_clear_error(uint32_t *code, uint32_t *site)
{
    uint32_t h[4] = {0, 0, 0, 0};
    cudaError_t e = cudaMemcpyFromSymbol(h, g_device_error, sizeof(h));
    if (e != cudaSuccess)
        return e;
    const uint32_t zero[4] = {0, 0, 0, 0};
    e = cudaMemcpyToSymbol(g_device_error, zero, sizeof(zero));
    if (e != cudaSuccess)
        return e;
    *code = h[0];
    *site = h[1];
    return cudaSuccess;
}

// Kernels with more than 48 KB of dynamic shared memory must opt in, per
// device: the attribute is set the first time the kernel launches with each
// device current (a process may drive several GPUs).
template <class K>
inline cudaError_t enable_dynamic_smem(K kernel, int bytes, DeviceFlags &done)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (done.has(dev))
        return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        done.set(dev);
    return e;
}

// ---------------------------------------------------------------- memory --

// Streaming 16-byte load through the read-only path.  Safe with the exact
// aliasing the ABI allows: every element is read once, by the thread that
// later writes it, before that write.
__device__ __forceinline__ uint4 ld16(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld8(const void *p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p));
    return v;
}

// Small vectors reused across rows (slerp's alpha): keep them in L1.
__device__ __forceinline__ float4 ld16_cached(const float *p)
{
    return __ldg(reinterpret_cast<const float4 *>(p));
}

__device__ __forceinline__ void st16(void *p, uint4 v)
{
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// One 32-byte store (sm_100's 256-bit vector store); p 32-byte aligned.
__device__ __forceinline__ void st32(void *p, uint4 a, uint4 b)
{
    asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
                 "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

__device__ __forceinline__ void st8(void *p, uint2 v)
{
    asm volatile("st.global.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ float4 as_f4(uint4 v)
{
    return make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                       __uint_as_float(v.w));
}

__device__ __forceinline__ uint4 as_u4(float4 v)
{
    return make_uint4(__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
                      __float_as_uint(v.w));
}

// ------------------------------------------------------------------ bf16 --

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two floats -> one word of two bf16, round to nearest even (lo in bits 0..15).
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float bf_get(const uint4 &v, int e)
{
    const uint32_t w = e < 2 ? v.x : e < 4 ? v.y : e < 6 ? v.z : v.w;
    return (e & 1) ? bf_hi(w) : bf_lo(w);
}

// Zero the elements of a unit at or past `valid` (0 < valid < elements).
__device__ __forceinline__ uint4 mask_octet(uint4 v, int valid)
{
    uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (2 * i >= valid)
            w[i] = 0u;
        else if (2 * i + 1 >= valid)
            w[i] &= 0x0000FFFFu;
    }
    return v;
}

__device__ __forceinline__ float4 mask_quad(float4 v, int valid)
{
    if (valid <= 1) v.y = 0.f;
    if (valid <= 2) v.z = 0.f;
    if (valid <= 3) v.w = 0.f;
    return v;
}

// ------------------------------------------------------------ reductions --
//
// Every reducer returns the same total, bit for bit, to every thread of the
// row, and sums in an order fixed by the row's class: each thread's own
// values in unit order, then an xor butterfly over the 32 lanes (offsets 16,
// 8, 4, 2, 1; each step adds two equal pairs, so all lanes agree), then the
// warps of the row in index order, then the CTAs of the cluster in rank
// order.  Two alternating shared-memory slots make back-to-back reductions
// safe with one barrier each.

template <int N>
__device__ __forceinline__ void warp_sum(float (&v)[N])
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int i = 0; i < N; ++i)
            v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_arrive()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait()
{
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The CTAs of a cluster per row; each CTA's total goes to every CTA's
// shared memory (DSMEM) slot [rank], then all sum slots 0..n-1 in order.
// The constructor's caller must have arrived on the cluster barrier once
// (cluster_arrive_relaxed at kernel start); the first exchange waits on it
// so that no CTA writes into a peer that has not started.
struct ClusterReducer {
    float *sm;  // [2][kWarps][4] this CTA's warp partials
    float *dsm; // [2][kMaxCluster][4] partials written by the peers
    uint32_t rank, ncta;
    int slot = 0;
    bool first = true;

    __device__ ClusterReducer(float *scratch, float *peer_slots)
        : sm(scratch), dsm(peer_slots), rank(cluster_ctarank()), ncta(cluster_nctarank())
    {
    }

    template <int N, class Op>
    __device__ __forceinline__ void reduce(float (&v)[N], Op op)
    {
        const int warp = threadIdx.x >> 5;
        float *s = sm + slot * (kWarps * 4);
        if ((threadIdx.x & 31) == 0)
#pragma unroll
            for (int i = 0; i < N; ++i)
                s[warp * 4 + i] = v[i];
        __syncthreads();
        float tot[N];
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float t = s[i];
#pragma unroll
            for (int w = 1; w < kWarps; ++w)
                t = op(t, s[w * 4 + i]);
            tot[i] = t;
        }
        if (first) {
            cluster_wait(); // every peer has started (arrival at kernel start)
            first = false;
        }
        float *d = dsm + slot * (kMaxCluster * 4);
        if (threadIdx.x < ncta) {
            namespace cg = cooperative_groups;
            float *remote = cg::this_cluster().map_shared_rank(d + rank * 4, threadIdx.x);
#pragma unroll
            for (int i = 0; i < N; ++i)
                remote[i] = tot[i];
        }
        cluster_arrive();
        cluster_wait();
#pragma unroll
        for (int i = 0; i < N; ++i) {
            float t = d[i];
            for (uint32_t q = 1; q < ncta; ++q)
                t = op(t, d[q * 4 + i]);
            v[i] = t;
        }
        slot ^= 1;
    }

    template <int N>
    __device__ __forceinline__ void sum(float (&v)[N])
    {
        warp_sum(v);
        reduce(v, [](float a, float b) { return a + b; });
    }

    __device__ __forceinline__ float max(float v)
    {
        float a[1] = {warp_max(v)};
        reduce(a, [](float x, float y) { return fmaxf(x, y); });
        return a[0];
    }

    // The whole cluster works on one row: every decision is already uniform.
    __device__ __forceinline__ bool any(bool b) { return b; }

    // Before exit: no CTA may leave while a peer could still write into it.
    // (Every exchange ends with a full cluster barrier, so the last one
    // already guarantees this; kernels that never exchanged still arrived
    // once and must wait once.)
    __device__ __forceinline__ void finish()
    {
        if (first)
            cluster_wait();
    }
};

// ------------------------------------------------- the row's scale factor --
//
// inv = 1 / sqrt(S + eps) in fp32 (IEEE square root and division).  Rows
// whose fp32 sum overflowed (S = inf with finite entries), or, at eps = 0,
// fell below 2^-100 (where squares may have lost bits to underflow, down to
// a sum of exactly 0 for a non-zero row), are
// summed again after scaling every entry by 2^m, m = 48 - exponent of the
// largest |entry| (exact: a power of two), and the factor is scaled back:
// the result equals the unscaled formula evaluated without overflow or
// underflow.  `gen(f)` must call f(v) on every value the thread contributed,
// in the order they were summed.  The branch is uniform across a row
// (`red.any` keeps CTA barriers uniform when a CTA holds several rows).

constexpr float kTinySum = 0x1p-100f;

__device__ __forceinline__ bool needs_rescale(float S, float eps)
{
    return S == __int_as_float(0x7f800000) || (eps == 0.f && S < kTinySum);
}

template <class Red, class Gen>
__device__ __forceinline__ int rescale_exponent(float S, float eps, Red &red, Gen &&gen, float &S_scaled)
{
    int m = 0;
    const bool need = needs_rescale(S, eps);
    if (red.any(need)) {
        float M = 0.f;
        gen([&](float v) { M = fmaxf(M, fabsf(v)); });
        M = red.max(M);
        if (need && M > 0.f && M < __int_as_float(0x7f800000))
            m = 48 - ilogbf(M);
        float acc[1] = {0.f};
        gen([&](float v) {
            const float u = scalbnf(v, m);
            acc[0] = fmaf(u, u, acc[0]);
        });
        red.sum(acc);
        S_scaled = acc[0];
    }
    return m;
}

// The row's factor as two parts: result = (entry * pre) * inv.  pre is 1
// except for rows of subnormals at eps = 0 (m > 100), where 2^m / n would
// pass FLT_MAX: 2^(m-100) then rides on the entries (both parts are exact
// powers of two times the rounded inverse, so the product rounds once, as
// 2^m / n would).
struct RowScale {
    float inv;
    float pre;
};

template <class Red, class Gen>
__device__ __forceinline__ RowScale row_scale(float S, float eps, Red &red, Gen &&gen)
{
    float Ss = S;
    const int m = rescale_exponent(S, eps, red, gen, Ss);
    if (m == 0)
        return {1.0f / sqrtf(S + eps), 1.f};
    const float inv = 1.0f / sqrtf(Ss + scalbnf(eps, 2 * m));
    if (m > 100)
        return {scalbnf(inv, 100), scalbnf(1.f, m - 100)};
    return {scalbnf(inv, m), 1.f};
}

// ------------------------------------------------ mbarrier + bulk copies --

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, for at most limit_ns.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns)
            return false;
    }
    return true;
}

// One bulk (non-tensor TMA) copy global -> this CTA's shared memory,
// completing `bytes` on `bar`.  dst, src 16-byte aligned; bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Segment lookup: the segment whose unit range holds `unit`.
template <class P>
__device__ __forceinline__ int find_segment(const P &p, int64_t unit)
{
    int lo = 0, hi = p.nseg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.unit_start[mid] <= unit)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

} // namespace ds
