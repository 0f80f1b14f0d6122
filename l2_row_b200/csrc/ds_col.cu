// ds_col.cu -- the weight calls on transposed rows (sm_100a): GPT-2's Conv1D
// stores its weight as [in, out], so a unit row (one output channel) is a
// COLUMN of the stored matrix: element j of row r sits at w[j * ld + r].
// DragonScale's package description lists transformers' Conv1D among the
// supported layers; the operations are the row calls' (eq. W_eff, eq. dL/dW,
// "Optimizer"), applied to those columns.
//
// One block owns a tile of kColTile consecutive unit rows (the stored
// matrix's columns) over the whole row length.  Its 256 threads are 8 quads
// (32 rows, 128 contiguous bytes of a stored row) by 32 lanes along the row;
// a warp reads 4 stored rows x 128 bytes per step, four steps in flight.
// (Capping the grid at four blocks per SM, so that the tiles in flight fit
// L2 for pass 2's re-read, measured slower: fewer bytes in flight.)  Pass 1 sums w^2 (and
// w . d) per unit row in double -- no fp32 overflow or underflow is
// possible, so no rescale path is needed -- and reduces the 64 lanes in a
// fixed tree; pass 2 re-reads the tile (from L2) and writes each result as
// its double value rounded once.  Every access is a 16-byte (fp32 quad) or
// 8-byte (bf16 quad) vector; the unit rows past `rows` are masked.
#include <algorithm>
#include <cfloat>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "ds_device.cuh"

namespace ds {

namespace {

constexpr int kColQuads = 8;                    // quads of unit rows per block
constexpr int kColTile = 4 * kColQuads;         // unit rows per block
constexpr int kColLanes = kCta / kColQuads;     // lanes along the row

__device__ __forceinline__ float4 col_quad_f32(const float *p) { return as_f4(ld16(p)); }

__device__ __forceinline__ float4 col_quad_bf16(const uint16_t *p)
{
    const uint2 r = ld8(p);
    return make_float4(bf_lo(r.x), bf_hi(r.x), bf_lo(r.y), bf_hi(r.y));
}

__device__ __forceinline__ float comp(const float4 &v, int i) { return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w; }

// Stores of a quad of unit rows (r0 .. r0+3) at one position j, masked to
// the first `valid` of them.
template <bool BF16>
__device__ __forceinline__ void col_store(void *base, float4 v, int valid)
{
    if constexpr (BF16) {
        uint16_t *o = static_cast<uint16_t *>(base);
        if (valid >= 4) {
            st8(o, make_uint2(pack_bf2(v.x, v.y), pack_bf2(v.z, v.w)));
        } else {
            const uint32_t a = pack_bf2(v.x, v.y), b = pack_bf2(v.z, v.w);
            const uint16_t h[4] = {static_cast<uint16_t>(a & 0xFFFFu), static_cast<uint16_t>(a >> 16),
                                   static_cast<uint16_t>(b & 0xFFFFu), static_cast<uint16_t>(b >> 16)};
            for (int i = 0; i < valid; ++i)
                o[i] = h[i];
        }
    } else {
        float *o = static_cast<float *>(base);
        if (valid >= 4) {
            st16(o, as_u4(v));
        } else {
            for (int i = 0; i < valid; ++i)
                o[i] = comp(v, i);
        }
    }
}

// OP: 0 forward (B16: bf16 W_eff), 1 backward (B16: bf16 GY), 2 renorm,
// 3 gradient projection, 4 momentum projection + renorm.
template <int OP, bool B16>
__global__ void __launch_bounds__(kCta) k_col(const __grid_constant__ WParams p)
{
    constexpr bool TWO = OP == 1 || OP == 3 || OP == 4; // sums w . d as well
    __shared__ double red[2][kColLanes][kColTile];
    __shared__ double fac[2][kColTile]; // per unit row: the scale, and D / n^2
    const int q = threadIdx.x % kColQuads, ks = threadIdx.x / kColQuads;
    const int64_t total = p.unit_start[p.nseg];

    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
        const int si = find_segment(p, u);
        const WSegK &sg = p.seg[si];
        const int64_t r0 = (u - p.unit_start[si]) * kColTile + 4 * q; // this thread's first unit row
        const int valid = sg.rows - r0 >= 4 ? 4 : static_cast<int>(sg.rows - r0 > 0 ? sg.rows - r0 : 0);
        const int K = sg.cols;
        // d: the backward's GY (bf16 or fp32, ld_out), or the projections'
        // gradient / momentum (fp32, ld)
        const bool d_bf16 = OP == 1 && B16;
        const int64_t ld_d = OP == 1 ? sg.ld_out : sg.ld;

        double s[4] = {0, 0, 0, 0}, dd[4] = {0, 0, 0, 0};
        if (valid > 0) {
#pragma unroll 4
            for (int j = ks; j < K; j += kColLanes) {
                const float4 w = col_quad_f32(sg.w + j * sg.ld + r0);
                float4 d = make_float4(0.f, 0.f, 0.f, 0.f);
                if constexpr (TWO)
                    d = d_bf16 ? col_quad_bf16(static_cast<const uint16_t *>(sg.gy) + j * ld_d + r0)
                               : col_quad_f32(static_cast<const float *>(sg.gy) + j * ld_d + r0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double wi = comp(w, i);
                    s[i] = fma(wi, wi, s[i]);
                    if constexpr (TWO)
                        dd[i] = fma(wi, static_cast<double>(comp(d, i)), dd[i]);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            red[0][ks][4 * q + i] = s[i];
            if constexpr (TWO)
                red[1][ks][4 * q + i] = dd[i];
        }
        __syncthreads();
        // fixed tree over the lanes
        for (int o = kColLanes / 2; o > 0; o >>= 1) {
            if (ks < o) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    red[0][ks][4 * q + i] += red[0][ks + o][4 * q + i];
                    if constexpr (TWO)
                        red[1][ks][4 * q + i] += red[1][ks + o][4 * q + i];
                }
            }
            __syncthreads();
        }
        if (threadIdx.x < kColTile) {
            const int c = threadIdx.x;
            const int64_t r = (u - p.unit_start[si]) * kColTile + c;
            if (r < sg.rows) {
                const double S = red[0][0][c] + static_cast<double>(p.eps);
                const double n = sqrt(S);
                const double g = (OP <= 1 && sg.gain) ? static_cast<double>(__ldg(sg.gain + r * sg.gain_stride)) : 1.0;
                fac[0][c] = g * static_cast<double>(sg.radius) / n; // g rho / n (renorm, momentum: rho / n)
                if constexpr (TWO)
                    fac[1][c] = red[1][0][c] / S;                    // D / n^2
                if constexpr (OP == 1) {
                    if (sg.gain)
                        sg.grad_g[r] = static_cast<float>(static_cast<double>(sg.radius) * red[1][0][c] / n);
                }
            }
        }
        __syncthreads();
        if (valid > 0) {
            double sc[4], qt[4] = {0, 0, 0, 0};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sc[i] = fac[0][4 * q + i];
                if constexpr (TWO)
                    qt[i] = fac[1][4 * q + i];
            }
#pragma unroll 4
            for (int j = ks; j < K; j += kColLanes) {
                const float4 w = col_quad_f32(sg.w + j * sg.ld + r0);
                float4 d = make_float4(0.f, 0.f, 0.f, 0.f);
                if constexpr (TWO)
                    d = d_bf16 ? col_quad_bf16(static_cast<const uint16_t *>(sg.gy) + j * ld_d + r0)
                               : col_quad_f32(static_cast<const float *>(sg.gy) + j * ld_d + r0);
                // each output is its double value rounded once to fp32 (bf16)
                float y[4], e[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double wi = comp(w, i);
                    y[i] = static_cast<float>(wi * sc[i]);
                    if constexpr (TWO) {
                        const double ei = static_cast<double>(comp(d, i)) - wi * qt[i];
                        e[i] = static_cast<float>(OP == 1 ? sc[i] * ei : ei);
                    }
                }
                const float4 yv = make_float4(y[0], y[1], y[2], y[3]);
                if constexpr (OP == 0) {
                    col_store<B16>(static_cast<char *>(sg.out) + (j * sg.ld_out + r0) * (B16 ? 2 : 4), yv, valid);
                } else if constexpr (OP == 2) {
                    col_store<false>(const_cast<float *>(sg.w) + j * sg.ld + r0, yv, valid);
                } else {
                    col_store<false>(sg.grad_w + j * sg.ld + r0, make_float4(e[0], e[1], e[2], e[3]), valid);
                    if constexpr (OP == 4)
                        col_store<false>(const_cast<float *>(sg.w) + j * sg.ld + r0, yv, valid);
                }
            }
        }
        __syncthreads(); // red and fac are reused by the next tile
    }
}

// ---------------------------------------------------------------------------
// Grouped transposed rows (ConvTranspose weights [in, out, k...] stored as
// [in, out * G], G = the kernel's volume): unit row r is the G consecutive
// stored columns [r G, r G + G) of every stored row, element (j, m) at
// w[j * ld + r G + m].  A block owns U consecutive unit rows (the host
// passes U in nu and G in group), i.e. the W = U G contiguous stored
// columns of every stored row: thread t takes column t % W and the stored
// rows t / W, t / W + S, ... (S = 256 / W lanes down the rows; threads past
// S W idle).  Pass 1 sums w^2 (and w . d) per column in fp32, lane by lane
// in row order, eight rows' loads in flight; each unit row then adds its
// columns' sums in double, lane by lane and column by column.  A block
// holding a unit row whose fp32 sum overflowed (or, at eps = 0, fell below
// 2^-100) sums again in double.  Pass 2 re-reads the block's columns (from
// L2) and writes the fp32 products with the scale rounded once (in double
// for the blocks summed in double, each result rounded once).  Loads are
// scalar: a unit row's G columns need not start on 16 bytes.
template <int OP, bool B16>
__global__ void __launch_bounds__(kCta) k_colg(const __grid_constant__ WParams p)
{
    constexpr bool TWO = OP == 1 || OP == 3 || OP == 4;
    __shared__ double red[2][kCta]; // [lane ks][column c] at ks * W + c
    __shared__ double fac[2][kCta]; // per unit row of the block (U <= 256)
    const int64_t total = p.unit_start[p.nseg];
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
        const int si = find_segment(p, u);
        const WSegK &sg = p.seg[si];
        const int G = sg.group, U = sg.nu;
        const int W = U * G, S = kCta / W;
        const int64_t r0 = (u - p.unit_start[si]) * U;
        const int nur = sg.rows - r0 < U ? static_cast<int>(sg.rows - r0) : U;
        const int c = threadIdx.x % W, ks = threadIdx.x / W;
        const bool act = ks < S && c < nur * G;
        const int K = sg.cols / G;              // stored rows
        const int64_t col = r0 * G + c;         // this thread's stored column
        const bool d_bf16 = OP == 1 && B16;
        const int64_t ld_d = OP == 1 ? sg.ld_out : sg.ld;
        auto dval = [&](int j) -> float {
            if constexpr (TWO) {
                if (d_bf16)
                    return bf_lo(static_cast<const uint16_t *>(sg.gy)[j * ld_d + col]);
                return static_cast<const float *>(sg.gy)[j * ld_d + col];
            } else {
                return 0.f;
            }
        };
        float s = 0.f, dd = 0.f;
        if (act) {
#pragma unroll 8
            for (int j = ks; j < K; j += S) {
                const float w = sg.w[j * sg.ld + col];
                s = fmaf(w, w, s);
                if constexpr (TWO)
                    dd = fmaf(w, dval(j), dd);
            }
        }
        if (threadIdx.x < S * W) {
            red[0][threadIdx.x] = s;
            red[1][threadIdx.x] = dd;
        }
        __syncthreads();
        // each unit row's sums: lane by lane, column by column
        auto unit_sums = [&](int rr, double &Sr, double &Dr) {
            Sr = 0.0;
            Dr = 0.0;
            for (int k = 0; k < S; ++k)
                for (int m = 0; m < G; ++m) {
                    Sr += red[0][k * W + rr * G + m];
                    if constexpr (TWO)
                        Dr += red[1][k * W + rr * G + m];
                }
        };
        bool need = false;
        if (threadIdx.x < nur) {
            double Sr, Dr;
            unit_sums(threadIdx.x, Sr, Dr);
            need = !(Sr <= static_cast<double>(FLT_MAX)) || (p.eps == 0.f && Sr < 0x1p-100);
        }
        const bool exact = __syncthreads_or(need) != 0;
        if (exact) {
            double se = 0.0, de = 0.0;
            if (act) {
                for (int j = ks; j < K; j += S) {
                    const double w = sg.w[j * sg.ld + col];
                    se = fma(w, w, se);
                    if constexpr (TWO)
                        de = fma(w, static_cast<double>(dval(j)), de);
                }
            }
            if (threadIdx.x < S * W) {
                red[0][threadIdx.x] = se;
                red[1][threadIdx.x] = de;
            }
            __syncthreads();
        }
        if (threadIdx.x < nur) {
            const int rr = threadIdx.x;
            const int64_t r = r0 + rr;
            double Sr, Dr;
            unit_sums(rr, Sr, Dr);
            Sr += static_cast<double>(p.eps);
            const double n = sqrt(Sr);
            const double g = (OP <= 1 && sg.gain) ? static_cast<double>(__ldg(sg.gain + r * sg.gain_stride)) : 1.0;
            fac[0][rr] = g * static_cast<double>(sg.radius) / n;
            fac[1][rr] = TWO ? Dr / Sr : 0.0;
            if constexpr (OP == 1) {
                if (sg.gain)
                    sg.grad_g[r] = static_cast<float>(static_cast<double>(sg.radius) * Dr / n);
            }
        }
        __syncthreads();
        auto put = [&](int j, float w, float y, float e) {
            if constexpr (OP == 0) {
                if constexpr (B16)
                    static_cast<uint16_t *>(sg.out)[j * sg.ld_out + col] = static_cast<uint16_t>(pack_bf2(y, 0.f) & 0xFFFFu);
                else
                    static_cast<float *>(sg.out)[j * sg.ld_out + col] = y;
            } else if constexpr (OP == 2) {
                const_cast<float *>(sg.w)[j * sg.ld + col] = y;
            } else {
                sg.grad_w[j * sg.ld + col] = e;
                if constexpr (OP == 4)
                    const_cast<float *>(sg.w)[j * sg.ld + col] = y;
            }
        };
        if (act && !exact) {
            const float sc = static_cast<float>(fac[0][c / G]), qt = static_cast<float>(fac[1][c / G]);
#pragma unroll 8
            for (int j = ks; j < K; j += S) {
                const float w = sg.w[j * sg.ld + col];
                float e = 0.f;
                if constexpr (TWO) {
                    const float ei = fmaf(-w, qt, dval(j));
                    e = OP == 1 ? sc * ei : ei;
                }
                put(j, w, w * sc, e);
            }
        } else if (act) {
            const double sc = fac[0][c / G], qt = fac[1][c / G];
            for (int j = ks; j < K; j += S) {
                const double w = sg.w[j * sg.ld + col];
                float e = 0.f;
                if constexpr (TWO) {
                    const double ei = static_cast<double>(dval(j)) - w * qt;
                    e = static_cast<float>(OP == 1 ? sc * ei : ei);
                }
                put(j, static_cast<float>(w), static_cast<float>(w * sc), e);
            }
        }
        __syncthreads(); // red and fac are reused by the next block of unit rows
    }
}

// ---------------------------------------------------------------------------
// Transposed rows in column tiles staged whole.  A tile is CT consecutive
// unit rows (stored columns c0 .. c0 + CT) over the whole unit-row length K
// (every stored row); a cluster of CL CTAs owns one tile, CTA k staging the
// band of stored rows [k * band, (k + 1) * band) of it in shared memory with
// 2-D TMA boxes of stored rows (CT * 4 contiguous bytes of each, and CT * 2
// or 4 of the second input), so HBM sees whole row pieces, each read once.
// Tiles are sized so that two or three CTAs share an SM: one's loads
// overlap another's stores (persistent clusters holding two or three tiles
// in flight each, one CTA per SM, measured slower: 234 against 187 us
// forward on 12 x [1600, 6400]).  Each CTA sums w^2 (and w . d) per column
// over its band in fp32 (lanes down the band in row order, an xor butterfly
// over a warp's lanes, the warps in order), the CTAs' partials meet through
// distributed shared memory and are added in rank order, and every CTA then
// scales its staged band straight to global memory with fp32 products (the
// row kernels' arithmetic).  A tile holding a column whose fp32 sum
// overflowed (or, at eps = 0, fell below 2^-100) is summed again in double
// and scaled in double, each output its double value rounded once (the
// column kernel's arithmetic).
template <int OP>
__host__ __device__ constexpr bool col_two() { return OP == 1 || OP == 3 || OP == 4; }

// Segments of one tile launch, each with the tensor maps (TMA descriptors)
// of its stored matrix w and of its second input d: 2-D row-major
// [K stored rows][N stored columns], boxes of CT columns by `box_h` rows.
constexpr int kColtSeg = 16;
struct ColtParams {
    CUtensorMap tmw[kColtSeg];
    CUtensorMap tmd[kColtSeg];
    WSegK seg[kColtSeg];
    int64_t unit_start[kColtSeg + 1];   // prefix sums of tiles
    int32_t box_h[kColtSeg];            // rows per box (<= 256)
    int32_t nseg;
    float eps;
    uint64_t wait_limit_ns;
};

// One 2-D tile of a tensor map into this CTA's shared memory (no
// multicast), completing its bytes on `bar`: columns x.., rows y...
// x * element size is a multiple of 16 bytes (x is a multiple of CT).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
                 ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
                 : "memory");
}

template <int OP, bool B16, int CT>
__global__ void __launch_bounds__(kCta) k_colt(const __grid_constant__ ColtParams p)
{
    constexpr bool TWO = col_two<OP>();
    constexpr int Q = CT / 4;                      // column quads of a tile
    constexpr int L = kCta / Q;                    // lanes down the band
    static_assert(Q * L == kCta && Q <= 32, "tile shape");
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full;
    constexpr int NW = kCta / 32;                  // warps
    __shared__ double red[2][NW][CT];              // the warps' partials per column
    __shared__ double fac[2][CT];
    cluster_arrive_relaxed();
    const uint32_t rank = cluster_ctarank(), ncta = cluster_nctarank();
    const int64_t unit = blockIdx.x / ncta;
    const int si = find_segment(p, unit);
    const WSegK &sg = p.seg[si];
    // G stored columns per unit row (ConvTranspose; 1 for Conv1D; a power
    // of two <= 32, so a tile holds whole unit rows)
    const int G = sg.group > 1 ? sg.group : 1;
    const int64_t NC = sg.rows * G;                              // stored columns
    const int64_t c0 = (unit - p.unit_start[si]) * CT;          // first stored column of the tile
    const int ncols = static_cast<int>(NC - c0 < CT ? NC - c0 : CT);
    const int K = sg.cols / G;
    const int band = (K + static_cast<int>(ncta) - 1) / static_cast<int>(ncta);
    const int k0 = min(K, static_cast<int>(rank) * band), nk = min(K, k0 + band) - k0;
    const bool d_bf16 = OP == 1 && B16;
    const int de = d_bf16 ? 2 : 4;
    const int brows = (band + p.box_h[si] - 1) / p.box_h[si] * p.box_h[si];   // band rows rounded to boxes
    float *tw = reinterpret_cast<float *>(smem);                          // [brows][CT]
    unsigned char *td = smem + static_cast<size_t>(brows) * CT * 4;       // [brows][CT] d
    double *xch = reinterpret_cast<double *>(td + (TWO ? static_cast<size_t>(brows) * CT * de : 0));
    // xch: [2][kMaxCluster][CT] the CTAs' partial sums, written by every peer

    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        mbar_init_fence();
    }
    __syncthreads();
    bool ok = true;
    if (threadIdx.x == 0) {
        // the band as boxes of box_h stored rows by CT columns (a box
        // reaching past the matrix is filled with zeros and still counts
        // its full bytes)
        const int bh = p.box_h[si];
        const int nbox = (nk + bh - 1) / bh;
        const uint32_t box_bytes = static_cast<uint32_t>(bh) * CT * (4u + (TWO ? de : 0));
        mbar_arrive_expect_tx(&full, box_bytes * static_cast<uint32_t>(nbox));
        for (int b = 0; b < nbox; ++b) {
            tma_load_2d(tw + static_cast<size_t>(b) * bh * CT, &p.tmw[si], static_cast<int>(c0), k0 + b * bh, &full);
            if constexpr (TWO)
                tma_load_2d(td + static_cast<size_t>(b) * bh * CT * de, &p.tmd[si], static_cast<int>(c0), k0 + b * bh,
                            &full);
        }
    }
    if (!mbar_wait_bounded(&full, 0, p.wait_limit_ns)) {
        ok = false;
        // no copy may still be writing this CTA's shared memory when it
        // leaves: wait (bounded) once more before going on without data
        if (threadIdx.x == 0 && !mbar_wait_bounded(&full, 0, p.wait_limit_ns))
            raise_device_error(DS_ERR_DEVICE_TIMEOUT, kSiteTileWait);
    }
    const int q = threadIdx.x % Q, ln = threadIdx.x / Q;
    const int warp = threadIdx.x >> 5;
    auto dvalf = [&](int i, int e) -> float {
        if constexpr (TWO) {
            if (d_bf16)
                return bf_lo(reinterpret_cast<const uint16_t *>(td)[static_cast<size_t>(i) * CT + 4 * q + e]);
            return reinterpret_cast<const float *>(td)[static_cast<size_t>(i) * CT + 4 * q + e];
        } else {
            return 0.f;
        }
    };
    // The warps' per-column partials (red[.][warp]) summed in warp order,
    // sent to slot [rank] of every CTA of the cluster, and added there in
    // rank order after the cluster barrier: S (and D) per column in fac's
    // place, identical in every CTA.
    auto cluster_sums = [&](double &S, double &D) {
        __syncthreads();
        if (threadIdx.x < CT) {
            const int c = threadIdx.x;
            double a0 = red[0][0][c], a1 = TWO ? red[1][0][c] : 0.0;
#pragma unroll
            for (int w = 1; w < NW; ++w) {
                a0 += red[0][w][c];
                if constexpr (TWO)
                    a1 += red[1][w][c];
            }
            for (uint32_t k = 0; k < ncta; ++k) {
                namespace cg = cooperative_groups;
                double *x0 = cg::this_cluster().map_shared_rank(xch + rank * CT + c, static_cast<int>(k));
                *x0 = a0;
                if constexpr (TWO) {
                    double *x1 = cg::this_cluster().map_shared_rank(xch + (kMaxCluster + rank) * CT + c,
                                                                    static_cast<int>(k));
                    *x1 = a1;
                }
            }
        }
        cluster_arrive();
        cluster_wait();
        S = 0.0;
        D = 0.0;
        if (threadIdx.x < CT) {
            const int c = threadIdx.x;
            S = xch[c];
            for (uint32_t k = 1; k < ncta; ++k)
                S += xch[k * CT + c];
            if constexpr (TWO) {
                D = xch[kMaxCluster * CT + c];
                for (uint32_t k = 1; k < ncta; ++k)
                    D += xch[(kMaxCluster + k) * CT + c];
            }
        }
    };
    // pass 1: this CTA's band, per column, in fp32 (lanes down the band in
    // row order); the lanes of a warp that hold the same columns (32 / Q of
    // them, Q apart) by an xor butterfly
    {
        float s[4] = {0.f, 0.f, 0.f, 0.f}, dd[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i = ln; i < nk; i += L) {
            const float4 w = *reinterpret_cast<const float4 *>(tw + static_cast<size_t>(i) * CT + 4 * q);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float wi = comp(w, e);
                s[e] = fmaf(wi, wi, s[e]);
                if constexpr (TWO)
                    dd[e] = fmaf(wi, dvalf(i, e), dd[e]);
            }
        }
#pragma unroll
        for (int o = Q; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s[e] += __shfl_xor_sync(0xffffffffu, s[e], o);
                if constexpr (TWO)
                    dd[e] += __shfl_xor_sync(0xffffffffu, dd[e], o);
            }
        if ((threadIdx.x & 31) < Q) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                red[0][warp][4 * q + e] = s[e];
                if constexpr (TWO)
                    red[1][warp][4 * q + e] = dd[e];
            }
        }
    }
    // per column S (and D), identical in every CTA; with G > 1 each column
    // then takes its unit row's sums: the G columns added in order
    auto unit_sums = [&](double &Sc, double &Dc) {
        if (G == 1)
            return;
        if (threadIdx.x < CT) {
            fac[0][threadIdx.x] = Sc;
            fac[1][threadIdx.x] = Dc;
        }
        __syncthreads();
        if (threadIdx.x < CT) {
            const int b = threadIdx.x / G * G;
            Sc = 0.0;
            Dc = 0.0;
            for (int m = 0; m < G; ++m) {
                Sc += fac[0][b + m];
                Dc += fac[1][b + m];
            }
        }
        __syncthreads();
    };
    cluster_wait();   // every peer has started (arrival at kernel start)
    double S, D;
    cluster_sums(S, D);
    unit_sums(S, D);
    // A column whose fp32 sum overflowed (or, at eps = 0, fell below
    // 2^-100) takes the tile through an exact pass: the band summed again
    // in double and a second exchange, then double arithmetic in pass 2.
    // S is the same in every CTA, so every CTA takes the same branch.
    const bool need = threadIdx.x < CT && c0 + threadIdx.x < NC &&
                      (!(S <= static_cast<double>(FLT_MAX)) || (p.eps == 0.f && S < 0x1p-100));
    const bool exact = __syncthreads_or(need) != 0;
    if (exact) {
        double s[4] = {0, 0, 0, 0}, dd[4] = {0, 0, 0, 0};
        for (int i = ln; i < nk; i += L) {
            const float4 w = *reinterpret_cast<const float4 *>(tw + static_cast<size_t>(i) * CT + 4 * q);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const double wi = comp(w, e);
                s[e] = fma(wi, wi, s[e]);
                if constexpr (TWO)
                    dd[e] = fma(wi, static_cast<double>(dvalf(i, e)), dd[e]);
            }
        }
#pragma unroll
        for (int o = Q; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                s[e] += __shfl_xor_sync(0xffffffffu, s[e], o);
                if constexpr (TWO)
                    dd[e] += __shfl_xor_sync(0xffffffffu, dd[e], o);
            }
        // every CTA has read the first exchange before any is overwritten
        cluster_arrive();
        cluster_wait();
        if ((threadIdx.x & 31) < Q) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                red[0][warp][4 * q + e] = s[e];
                if constexpr (TWO)
                    red[1][warp][4 * q + e] = dd[e];
            }
        }
        cluster_sums(S, D);
        unit_sums(S, D);
    }
    if (threadIdx.x < CT) {
        const int c = threadIdx.x;
        const int64_t r = (c0 + c) / G;   // the unit row of this column
        if (c0 + c < NC) {
            S += static_cast<double>(p.eps);
            const double n = sqrt(S);
            const double g = (OP <= 1 && sg.gain) ? static_cast<double>(__ldg(sg.gain + r * sg.gain_stride)) : 1.0;
            fac[0][c] = g * static_cast<double>(sg.radius) / n;
            if constexpr (TWO)
                fac[1][c] = D / S;
            if constexpr (OP == 1) {
                if (sg.gain && rank == 0 && ok && (c0 + c) % G == 0)
                    sg.grad_g[r] = static_cast<float>(static_cast<double>(sg.radius) * D / n);
            }
        } else {
            fac[0][c] = 0.0;
            fac[1][c] = 0.0;
        }
    }
    __syncthreads();
    ok = __syncthreads_and(ok) != 0;
    if (!ok) {
        if (threadIdx.x == 0)
            raise_device_error(DS_ERR_DEVICE_TIMEOUT, kSiteTileWait);
        return;
    }
    const int valid = ncols - 4 * q >= 4 ? 4 : (ncols - 4 * q > 0 ? ncols - 4 * q : 0);
    if (valid == 0)
        return;
    const int64_t col = c0 + 4 * q;
    auto store = [&](int64_t j, const float (&y)[4], const float (&ev)[4]) {
        const float4 yv = make_float4(y[0], y[1], y[2], y[3]);
        if constexpr (OP == 0) {
            col_store<B16>(static_cast<char *>(sg.out) + (j * sg.ld_out + col) * (B16 ? 2 : 4), yv, valid);
        } else if constexpr (OP == 2) {
            col_store<false>(const_cast<float *>(sg.w) + j * sg.ld + col, yv, valid);
        } else {
            col_store<false>(sg.grad_w + j * sg.ld + col, make_float4(ev[0], ev[1], ev[2], ev[3]), valid);
            if constexpr (OP == 4)
                col_store<false>(const_cast<float *>(sg.w) + j * sg.ld + col, yv, valid);
        }
    };
    // pass 2: the scale (and D / n^2) rounded once to fp32, fp32 products;
    // the exact pass keeps them in double, each output rounded once
    if (!exact) {
        float sc[4], qt[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sc[e] = static_cast<float>(fac[0][4 * q + e]);
            if constexpr (TWO)
                qt[e] = static_cast<float>(fac[1][4 * q + e]);
        }
        for (int i = ln; i < nk; i += L) {
            const float4 w = *reinterpret_cast<const float4 *>(tw + static_cast<size_t>(i) * CT + 4 * q);
            float y[4], ev[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float wi = comp(w, e);
                y[e] = wi * sc[e];
                if constexpr (TWO) {
                    const float ei = fmaf(-wi, qt[e], dvalf(i, e));
                    ev[e] = OP == 1 ? sc[e] * ei : ei;
                }
            }
            store(k0 + i, y, ev);
        }
    } else {
        double sc[4], qt[4] = {0, 0, 0, 0};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sc[e] = fac[0][4 * q + e];
            if constexpr (TWO)
                qt[e] = fac[1][4 * q + e];
        }
        for (int i = ln; i < nk; i += L) {
            const float4 w = *reinterpret_cast<const float4 *>(tw + static_cast<size_t>(i) * CT + 4 * q);
            float y[4], ev[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const double wi = comp(w, e);
                y[e] = static_cast<float>(wi * sc[e]);
                if constexpr (TWO) {
                    const double ei = static_cast<double>(dvalf(i, e)) - wi * qt[e];
                    ev[e] = static_cast<float>(OP == 1 ? sc[e] * ei : ei);
                }
            }
            store(k0 + i, y, ev);
        }
    }
}

template <int OP, bool B16>
cudaError_t launch_col_t(const WParams &p, int64_t units, cudaStream_t st)
{
    const int grid = static_cast<int>(units < 148 * 8 ? units : 148 * 8);
    k_col<OP, B16><<<grid, kCta, 0, st>>>(p);
    return cudaGetLastError();
}

template <int OP, bool B16>
cudaError_t launch_colg_t(const WParams &p, int64_t units, cudaStream_t st)
{
    const int grid = static_cast<int>(units < 148 * 8 ? units : 148 * 8);
    k_colg<OP, B16><<<grid, kCta, 0, st>>>(p);
    return cudaGetLastError();
}

template <int OP, bool B16, int CT>
cudaError_t launch_colt_t(const ColtParams &p, int64_t units, int cl, int smem, cudaStream_t st)
{
    static DeviceFlags attr_set;
    if (const cudaError_t e = enable_dynamic_smem(k_colt<OP, B16, CT>, kColTileSmemMax, attr_set))
        return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units * cl), 1, 1);
    cfg.blockDim = dim3(kCta, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cl);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_colt<OP, B16, CT>, p);
}

template <int OP, bool B16>
cudaError_t launch_colt_ct(const ColtParams &p, int64_t units, int ct, int cl, int smem, cudaStream_t st)
{
    switch (ct) {
    case 16: return launch_colt_t<OP, B16, 16>(p, units, cl, smem, st);
    case 32: return launch_colt_t<OP, B16, 32>(p, units, cl, smem, st);
    case 64: return launch_colt_t<OP, B16, 64>(p, units, cl, smem, st);
    case 128: return launch_colt_t<OP, B16, 128>(p, units, cl, smem, st);
    default: return cudaErrorInvalidValue;
    }
}

// cuTensorMapEncodeTiled, from the driver through the runtime (the library
// links the runtime only).
PFN_cuTensorMapEncodeTiled_v12000 encode_tiled()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// The map of a row-major [K][N] matrix with row pitch `ld` elements,
// boxes of ct columns by bh rows.
bool encode_map(CUtensorMap *m, const void *base, bool bf16, int64_t K, int64_t N, int64_t ld, int ct, int bh)
{
    const auto fn = encode_tiled();
    if (!fn)
        return false;
    const int es = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * es};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(ct), static_cast<cuuint32_t>(bh)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace

int col_tile_rows() { return kColTile; }

// Rows per box: the band in as few boxes of at most 256 rows (the TMA box
// limit) as possible, all of one height, so that no box reaches far into
// the next band.  A tensor copy's shared-memory destination must start on
// 128 bytes, so the height is a multiple of the rows that fill 128 bytes at
// the narrowest staged row (CT bf16 elements of a bf16 GY): 4 rows at CT =
// 16, 2 at CT = 32; every box of w and of the second input then starts on
// 128 bytes.  (Rows a box takes past the band are ignored.)
int col_tile_box_rows(int64_t band, int ct)
{
    if (band <= 0)
        return 1;
    const int64_t nbox = (band + 255) / 256;
    const int64_t m = ct * 2 >= 128 ? 1 : 128 / (ct * 2);
    const int64_t bh = (band + nbox - 1) / nbox;
    return static_cast<int>((bh + m - 1) / m * m);
}

int col_tile_smem(int ct, int cl, int64_t band, int elem_bytes)
{
    (void)cl;
    const int64_t bh = col_tile_box_rows(band, ct);
    const int64_t rows = band > 0 ? (band + bh - 1) / bh * bh : 0;
    const int64_t tile = rows * ct * elem_bytes;
    const int64_t xch = int64_t(2) * kMaxCluster * ct * 8;
    return static_cast<int>(tile + xch);
}

int col_tile_segments() { return kColtSeg; }

int launch_col(int op, bool b16, const WParams &p, int64_t units, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (op) {
    case 0: return b16 ? launch_col_t<0, true>(p, units, st) : launch_col_t<0, false>(p, units, st);
    case 1: return b16 ? launch_col_t<1, true>(p, units, st) : launch_col_t<1, false>(p, units, st);
    case 2: return launch_col_t<2, false>(p, units, st);
    case 3: return launch_col_t<3, false>(p, units, st);
    case 4: return launch_col_t<4, false>(p, units, st);
    default: return cudaErrorInvalidValue;
    }
}

int col_group_units(int group)
{
    return group >= 64 ? 1 : 64 / group;
}

int launch_colg(int op, bool b16, const WParams &p, int64_t units, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (op) {
    case 0: return b16 ? launch_colg_t<0, true>(p, units, st) : launch_colg_t<0, false>(p, units, st);
    case 1: return b16 ? launch_colg_t<1, true>(p, units, st) : launch_colg_t<1, false>(p, units, st);
    case 2: return launch_colg_t<2, false>(p, units, st);
    case 3: return launch_colg_t<3, false>(p, units, st);
    case 4: return launch_colg_t<4, false>(p, units, st);
    default: return cudaErrorInvalidValue;
    }
}

int launch_colt(int op, bool b16, int ct, int cl, int smem, const WParams &w, int64_t units, void *stream)
{
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (smem > kColTileSmemMax || w.nseg > kColtSeg)
        return cudaErrorInvalidValue;
    static thread_local ColtParams p;
    const bool two = op == 1 || op == 3 || op == 4;
    for (int i = 0; i < w.nseg; ++i) {
        const WSegK &sg = w.seg[i];
        const int64_t G = sg.group > 1 ? sg.group : 1;
        const int64_t K = sg.cols / G, N = sg.rows * G, band = (K + cl - 1) / cl;
        const int bh = col_tile_box_rows(band, ct);
        p.seg[i] = sg;
        p.unit_start[i] = w.unit_start[i];
        p.box_h[i] = bh;
        if (!encode_map(&p.tmw[i], sg.w, false, K, N, sg.ld, ct, bh))
            return cudaErrorInvalidValue;
        if (two) {
            const bool d16 = op == 1 && b16;
            const int64_t ld_d = op == 1 ? sg.ld_out : sg.ld;
            if (!encode_map(&p.tmd[i], sg.gy, d16, K, N, ld_d, ct, bh))
                return cudaErrorInvalidValue;
        }
    }
    p.unit_start[w.nseg] = w.unit_start[w.nseg];
    p.nseg = w.nseg;
    p.eps = w.eps;
    p.wait_limit_ns = w.wait_limit_ns;
    switch (op) {
    case 0: return b16 ? launch_colt_ct<0, true>(p, units, ct, cl, smem, st) : launch_colt_ct<0, false>(p, units, ct, cl, smem, st);
    case 1: return b16 ? launch_colt_ct<1, true>(p, units, ct, cl, smem, st) : launch_colt_ct<1, false>(p, units, ct, cl, smem, st);
    case 2: return launch_colt_ct<2, false>(p, units, ct, cl, smem, st);
    case 3: return launch_colt_ct<3, false>(p, units, ct, cl, smem, st);
    case 4: return launch_colt_ct<4, false>(p, units, ct, cl, smem, st);
    default: return cudaErrorInvalidValue;
    }
}

} // namespace ds
