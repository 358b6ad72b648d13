// Launch interface of the fused RPBH + quantise kernel (rpbh_quant.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "oq_internal.h"

namespace oq {

struct RpbhParams {
    const void* x;        // [M, d] rows, bf16 or fp32
    int M, d, nb;         // rows, dimension, h-blocks per row (d / h)
    // Work layout.  A warp covers RW rows x (32 / RW) h-blocks (lane = row
    // r * (32 / RW) + block j); a team of `team` warps covers all nb blocks
    // of a set of RW rows; a CTA holds `tpc` teams, each with `slots`
    // staging slots of RW rows.
    int RW, lbw, lrw;     // rows per warp; log2 of the blocks per warp and of RW
    int SPL;              // lanes per h-block: 1, or 2 (each holds half the block's values)
    int contig;           // identity permutation: blocks read contiguously (one lane per block)
    int team, tpc, slots;
    int row_bytes, srow;  // bytes per input row; shared-memory row stride
    int nrs;              // row sets: ceil(M / RW)
    // Warp-group kernel (rpbh_groups.cu): NG groups of G threads per CTA,
    // tiles of R rows, thread (r, b) of a group on row r's h-block b.
    int R, G, NG, ntiles;
    const uint32_t* gtab; // device gather table (see build_gather_table)
    const uint16_t* gtab16; // the same with 16-bit entries (see build_gather_table16)
    const LutEntry* lut;  // device quantiser lookup table
    int lut_n, lut_off;   // entries; index offset = -(magic bits) - kmin
    float G_lut;          // lookup-table bins per unit of v
    int L;                // levels (2^bits)
    uint8_t* idx_out;     // packed indices (or the centroid values)
    int out_row_bytes;
    int st32;             // idx_out and out_row_bytes are 32-byte aligned: 256-bit stores
    float* s_out;         // activations: s (fp32)
    uint16_t* r_out;      // weights: r (bf16)
    float* y_out;         // test hook: x' (fp32)
    float* norm_out;      // test hook: ||x'||
    float rsqrt_h;        // 1/sqrt(h)
    float eps;            // the split's eps
    float s_max;          // FLT_MAX / (2 sqrt(h)): larger row norms take the middle cell
    int starve;           // test hook: issue no copies (the waits run out)
    uint32_t mid_val;     // value outputs: the middle cell's value (bf16 bits or e4m3 byte)
};

constexpr int kMaxWarps = 12;                 // per CTA: the kernel's launch bound is 384 threads
constexpr int kMaxThreads = kMaxWarps * 32;   // (168 registers each)
constexpr int kMaxWarpsSplit = 16;            // with two lanes per block: 512 threads
constexpr int kMaxThreadsSplit = kMaxWarpsSplit * 32;  // (128 registers each)
constexpr int kSmemLimit = 227 * 1024;

int rpbh_smem_bytes(const RpbhParams& p);

// Chooses RW, team, tpc, slots and srow for a shape (the choice depends on d,
// h, the input's element size and the lookup table only, so every output
// mode of one shape takes the same layout and sums the row norm in the same
// order).  Returns false if no layout fits in shared memory.
bool rpbh_choose_layout(RpbhParams& p, int h, int esize);

// Test and tuning hook: force rows per warp, slots per team and lanes per
// block (0: automatic).
void rpbh_force_layout(int rows_per_warp, int slots, int lanes_per_block);

// The warp-group kernel (rpbh_groups.cu) for permuted plans with h <= 128.
// rpbh_choose_groups sets R, G, NG, srow, row_bytes and ntiles (p.M, p.d,
// p.nb and p.lut_n set); false if the shape has no group layout.
constexpr int kMaxGroups = 4;
bool rpbh_choose_groups(RpbhParams& p, int esize);
cudaError_t launch_rpbh_groups(const RpbhParams& p, bool in_bf16, int h, int bits, int mode, int grid,
                               cudaStream_t stream);

// The kernel for blocks of 256 ... 16384 (rht_big.cu): one row per CTA at a
// time; RW, team, tpc, slots and srow are not used.
int rht_big_smem_bytes(const RpbhParams& p);
cudaError_t launch_rht_big(const RpbhParams& p, bool in_bf16, int h, int bits, int mode, int grid,
                           cudaStream_t stream);

// mode 0: activations (s fp32), 1: weights (r bf16), 2: rotation only (x', norm),
// 3 / 4: activations as centroid values, bf16 / e4m3 of c sqrt(d) (s fp32)
cudaError_t launch_rpbh_quant(const RpbhParams& p, bool in_bf16, int h, int bits, int mode, int grid,
                              cudaStream_t stream);

}  // namespace oq
