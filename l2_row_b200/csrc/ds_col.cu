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

template <int OP, bool B16>
cudaError_t launch_col_t(const WParams &p, int64_t units, cudaStream_t st)
{
    const int grid = static_cast<int>(units < 148 * 8 ? units : 148 * 8);
    k_col<OP, B16><<<grid, kCta, 0, st>>>(p);
    return cudaGetLastError();
}

} // namespace

int col_tile_rows() { return kColTile; }

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

} // namespace ds
