// ds_internal.h -- structures shared by the host planner (ds_api.cpp) and the
// sm_100a kernels (ds_kernels.cu).  Not part of the public ABI.
#pragma once

#include <atomic>
#include <cstdint>

#include "ds.h"

#ifdef __CUDACC__
#define DS_HD __host__ __device__
#else
#define DS_HD
#endif

namespace ds {

// A one-time host step per device (a kernel attribute, a symbol address):
// one bit per device id 0..63, set once the step succeeded with that device
// current.  Devices past 63 are never marked, so their callers redo the step
// on every call, which is correct, only slower.
struct DeviceFlags {
    std::atomic<uint64_t> bits{0};
    bool has(int dev) const
    {
        return dev >= 0 && dev < 64 && ((bits.load(std::memory_order_acquire) >> dev) & 1u) != 0;
    }
    void set(int dev)
    {
        if (dev >= 0 && dev < 64)
            bits.fetch_or(uint64_t(1) << dev, std::memory_order_release);
    }
};

// Every kernel runs 256-thread CTAs.
constexpr int kCta = 256;
constexpr int kWarps = kCta / 32;
// Register paths hold at most kmax_of(op) 16-byte units of each input per
// thread: 8 for one input (forward, renorm), 4 where two inputs are held
// (backward: w and GY; l2 with residual; slerp: res and out).
constexpr int kKmaxMax = 8;
DS_HD constexpr int kmax_of(ds_op op) { return (op == DS_OP_WN_FORWARD || op == DS_OP_ROW_RENORM) ? 8 : 4; }
// Largest number of ring positions of any staged launch (16 KB slots).
constexpr int kTileMaxGroups = 13;
// Largest cluster (portable limit).
constexpr int kMaxCluster = 8;
// Segments per launch (kernel parameter block); larger tables are split.
constexpr int kSegPerLaunch = 128;
// Staged paths: a ring of shared-memory slots filled by bulk copies, 16 KB
// (WARP path) or 32 / 64 KB (CTA path) per slot, and 112 KB for weight rows
// (two of them fill a CTA's shared memory).
constexpr int kTileSlotBytes = 16384;          // WARP path
constexpr int kTileSlotMaxBytes = 65536;       // largest CTA-path slot of the activation rows
constexpr int kTileSlotMaxWeightBytes = 114688;
constexpr int kMaxTileSlots = 13;         // 13 x 16 KB = 208 KB of the 227 KB per CTA
constexpr int kTileMaxRowsPerSlot = 64;
// Two-pass path: pipeline stages (the chunk size is per operation).  Three
// stages let four CTAs share an SM where four stages let three; on rows of
// 262,144 columns that took the forward 107 -> 97 us, slerp 384 -> 326 and
// l2 150 -> 127 (two stages: 114, 334, 121).
constexpr int kStages = 3;

// Rows split over a cluster of `ncta` CTAs (staged cluster classes): CTA k
// stages units [k * per, min(nu, (k + 1) * per)) of every row, per =
// ceil(nu / ncta) rounded up to even, so that every slice of an array with
// 8-byte units (bf16 GY quads) still starts on 16 bytes.  One CTA: the row.
DS_HD constexpr int slice_per(int nu, int ncta)
{
    return ncta <= 1 ? nu : (((nu + ncta - 1) / ncta) + 1) & ~1;
}

// Row length in 16-byte units: weight ops work on quads of fp32 (w is fp32),
// activation ops on octets of bf16.
DS_HD constexpr bool is_weight_op(ds_op op)
{
    return op <= DS_OP_ROW_RENORM || op == DS_OP_GRAD_PROJECT || op == DS_OP_RENORM_MOMENTUM;
}
DS_HD constexpr int elems_per_unit(ds_op op) { return is_weight_op(op) ? 4 : 8; }

struct RowClass {
    int path;    // ds_path (never DS_PATH_AUTO)
    int group;   // threads per row in each CTA (staged paths: the team), 0 on the two-pass path
    int cluster; // CTAs per row: 1 on WARP/CTA, 2..8 on CLUSTER (a staged slice each) and TWO_PASS
    int rps;     // staged paths: rows per shared-memory slot for this segment
    int slot;    // staged paths: slot bytes (16, 32, 64 or 112 KB); 0 on the two-pass path
};

// WARP, CTA and CLUSTER rows all run on the staged kernel (a cluster stages
// one slice of each row per CTA); TWO_PASS rows on the streaming kernel.
inline bool is_staged(const RowClass &c)
{
    return c.path == DS_PATH_WARP || c.path == DS_PATH_CTA || c.path == DS_PATH_CLUSTER;
}

// Launch shape: the staged segments of a call share one launch per (slot
// size, cluster size) (each segment carries its own rows per slot); TWO_PASS
// segments one launch per cluster size.
inline bool same_launch(const RowClass &a, const RowClass &b)
{
    if (a.path == DS_PATH_TWO_PASS || b.path == DS_PATH_TWO_PASS)
        return a.path == b.path && a.cluster == b.cluster;
    return is_staged(b) && a.slot == b.slot && a.cluster == b.cluster && a.path == b.path;
}

// Device copy of one weight segment.
struct WSegK {
    const float *w;
    const float *gain;
    void *out;        // forward: w_eff; renorm: w
    const void *gy;
    float *grad_w;
    float *grad_g;
    int64_t rows;
    int64_t ld;
    int64_t ld_out;
    int32_t cols;
    int32_t nu;       // units per row
    float radius;
    int32_t group;    // staged paths: rows per slot
    int32_t gain_stride; // 1: gain[row]; 0: one gain for every row
    int32_t pad_;
};

// Device copy of one activation segment (bf16 carried as raw 16-bit words).
struct ASegK {
    const uint16_t *x;
    const uint16_t *r;
    uint16_t *y;
    const float *alpha;  // slerp: alpha; Dory rows: the first scale vector
    const float *s2;     // SwiGLU rows: the second scale vector
    int64_t rows;
    int64_t ld;
    int32_t cols;
    int32_t nu;
    int32_t group;    // staged paths: rows per slot
    int32_t pad_;
};

// Device copy of one activation segment of a backward call.
struct AGSegK {
    const uint16_t *x;
    const uint16_t *r;
    const uint16_t *dy;
    float *dx;
    float *dr;
    const float *alpha;
    int64_t rows;
    int64_t ld;       // of x, r, dy (elements)
    int64_t ld_d;     // of dx, dr (elements)
    int32_t cols;
    int32_t nu;
    int32_t group;    // staged paths: rows per slot
    int32_t pad_;
};

template <class Seg>
struct LaunchParams {
    Seg seg[kSegPerLaunch];
    int64_t unit_start[kSegPerLaunch + 1]; // prefix sums of work units
    int32_t nseg;
    float eps;
    uint64_t wait_limit_ns;                // bound of every device-side wait
    const float *alpha_shared;             // slerp: alpha of every segment (or NULL if they differ);
                                           // Dory rows: the first scale vector
    const float *alpha2_shared;            // SwiGLU rows: the second scale vector (or NULL)
    int32_t alpha_cols;                    //        their length
    int32_t ws_ld;                         // slerp backward: floats per workspace line
    float *ws;                             //        per-team dalpha partial sums (NULL: no dalpha)
};

using WParams = LaunchParams<WSegK>;
using AParams = LaunchParams<ASegK>;
using GParams = LaunchParams<AGSegK>;

// Dory's q and k rows (ds_qk.cu): one segment after host validation.
constexpr int kQkThreads = 256;
constexpr int kQkWarps = kQkThreads / 32;
constexpr int kQkTasks = 3;     // warp tasks held in registers at once
constexpr int kQkTable = 1024;  // cos (and sin) entries per block iteration: rb * head_dim / 2
struct QKSegK {
    const uint16_t *q, *k, *v;
    uint16_t *q_out, *k_cache, *v_cache;
    const int32_t *pos, *slot;
    const float *inv, *q_scale;
    int64_t rows, cache_rows;
    int64_t ld_q, ld_kv, ld_cache;
    int32_t D, hq, hk, rb; // rb: rows per block iteration
};
struct QKParams {
    QKSegK seg[kSegPerLaunch];
    int64_t unit_start[kSegPerLaunch + 1]; // prefix sums of block iterations
    int32_t nseg;
    float eps;
};

// Row lengths (ds_kernels.cu): out[r] = sqrt(sum w[r,:]^2 + eps) / div.
struct RNSegK {
    const float *w;
    float *out;
    int64_t rows, ld;
    int32_t cols;
    float div;
};
struct RNParams {
    RNSegK seg[kSegPerLaunch];
    int64_t unit_start[kSegPerLaunch + 1]; // prefix sums of rows
    int32_t nseg;
    float eps;
};
// Scalar gains (ds_kernels.cu): parts[rows] = sum of parts[0..rows) in a
// fixed order, for each listed buffer.
struct GainSumK {
    float *parts;
    int64_t rows;
};
struct GainSumParams {
    GainSumK seg[kSegPerLaunch];
    int32_t nseg;
};

// Error word written by kernels (see ds_get_device_status).
enum DeviceErrorSite : uint32_t {
    kSiteStreamWait = 1,
    kSiteStreamDrain = 2,
    kSiteSelftest = 3,
    kSiteTileWait = 4,
    kSiteQkSlot = 5,
};

// Launchers of the cluster paths (ds_kernels.cu).  `units` = rows
// (CLUSTER/TWO_PASS); return cudaError_t as int.
int launch_wn_forward(const RowClass &rc, const WParams &p, int64_t units, bool out_bf16, void *stream);
int launch_wn_backward(const RowClass &rc, const WParams &p, int64_t units, bool gy_bf16, void *stream);
int launch_row_renorm(const RowClass &rc, const WParams &p, int64_t units, void *stream);
int launch_grad_project(const RowClass &rc, const WParams &p, int64_t units, void *stream);
int launch_renorm_momentum(const RowClass &rc, const WParams &p, int64_t units, void *stream);
int launch_l2_rows(const RowClass &rc, const AParams &p, int64_t units, void *stream);
int launch_slerp_rows(const RowClass &rc, const AParams &p, int64_t units, void *stream);
int launch_wait_selftest(uint64_t limit_ns, void *stream);
// `sms`: the device's SM count (the grid holds every CTA at once).
int launch_row_norms(const RNParams &p, int sms, void *stream);
// Transposed rows (ds_col.cu): op 0 forward, 1 backward, 2 renorm,
// 3 gradient projection, 4 momentum projection; b16: bf16 W_eff / GY.
// p's unit_start counts tiles of col_tile_rows() rows.
int launch_col(int op, bool b16, const WParams &p, int64_t units, void *stream);
int col_tile_rows();
// Grouped transposed rows (ds_col.cu, ConvTranspose): each segment's
// `group` = G stored columns per unit row and `nu` = col_group_units(G)
// unit rows per block; p's unit_start counts blocks.
int col_group_units(int group);
int launch_colg(int op, bool b16, const WParams &p, int64_t units, void *stream);
// Transposed rows in whole column tiles (ds_col.cu): tiles of ct unit rows
// (16, 32, 64 or 128) over every stored row, a cluster of cl CTAs per tile
// (bands of ceil(K / cl) stored rows each, loaded as 2-D TMA boxes); p's
// unit_start counts tiles; at most col_tile_segments() segments.
// Dynamic shared memory of a launch: col_tile_smem(ct, cl, largest band,
// bytes of w plus d per element), at most kColTileSmemMax.
constexpr int kColTileSmemMax = 200 * 1024;
// The planner's budgets, tried in order: the first that holds some tile
// shape of a segment decides it (two or more CTAs per SM, else one).
constexpr int kColTileBudgets[2] = {96 * 1024, kColTileSmemMax};
int col_tile_smem(int ct, int cl, int64_t band, int elem_bytes);
int col_tile_segments();   // segments per tile launch (each carries two TMA descriptors)
int launch_colt(int op, bool b16, int ct, int cl, int smem, const WParams &p, int64_t units, void *stream);
int launch_gain_sums(const GainSumParams &p, void *stream);
// Staged paths (ds_tile.cu).  tag: 0 forward bf16, 1 forward f32,
// 2 backward bf16 GY, 3 backward f32 GY, 4 renorm, 5 l2, 6 slerp,
// 7 gradient projection, 8 momentum projection + renorm, 9 l2 backward,
// 10 slerp backward, 11 gated l2 rows, 12 SwiGLU l2 rows, 13 row lengths
// (out: rnorm, radius: the divisor); params is a WParams
// (tags 0-4, 7, 8, 13), AParams (5, 6, 11, 12) or GParams (9, 10) whose segments
// carry rows per slot in `group` and whose
// unit_start counts slots; slot_bytes 16, 32, 64 or (weights) 112 KB.
// cluster: CTAs per row (1, 2, 4 or 8); units: the launch's slots; the
// kernel gets min(units, resident clusters) clusters, returned in
// *clusters_used (lines of the slerp backward's dalpha workspace).
int launch_tile(int tag, const void *params, int64_t units, int slot_bytes, int cluster, int *clusters_used,
                void *stream);
// Ring positions (consumer teams) per CTA of a staged launch.
int tile_groups(int tag, int slot_bytes);
// The built-in device scratch of the no-alloc slerp backward (ds_tile.cu).
constexpr int64_t kBuiltinScratchFloats = int64_t(16) << 20; // 64 MB
int builtin_scratch(void **ptr, uint64_t *bytes);
// dalpha[c] = sum over CTAs c0 < grid and their used teams q of
// ws[(c0 * groups + q) * ws_ld + c] (slerp backward), in a fixed order:
// 32 interleaved partial sums over the lines, then a fixed tree.
int launch_dalpha_reduce(const float *ws, int ws_ld, int grid, int groups, int64_t total_units, int cols,
                         float *dalpha, void *stream);
// Exhaustive check of the Dory rows' fast reciprocal and quotient (ds_tile.cu).
int launch_division_check(unsigned long long *counts, void *stream);
// Every .cu file is its own device module with its own error word: the
// reader syncs the stream, then reads and clears each module's word.
int read_and_clear_device_error(uint32_t *code, uint32_t *site, void *stream);
int tile_read_and_clear_error(uint32_t *code, uint32_t *site);
int qk_read_and_clear_error(uint32_t *code, uint32_t *site);
// Dory's q and k rows (ds_qk.cu): `grid` blocks of kQkThreads; every
// segment of `p` has the same head size.
int launch_qk(const QKParams &p, int grid, void *stream);

} // namespace ds
