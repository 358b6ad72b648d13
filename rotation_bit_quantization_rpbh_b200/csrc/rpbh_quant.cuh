// Launch interface of the fused RPBH + quantise kernel (rpbh_quant.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "oq_internal.h"

namespace oq {

struct RpbhParams {
    const void* x;        // [M, d] rows, bf16 or fp32
    int M, d, nb;         // rows, dimension, h-blocks per row (d / h)
    int R, T, G, NG;      // rows per tile (power of two), threads per CTA, threads per warp group, groups (T = NG G)
    int row_bytes, srow;  // bytes per input row; shared-memory row stride
    int ntiles;
    const uint16_t* gtab;  // device gather table (chunked, see host.cpp)
    const LutEntry* lut;   // device quantiser lookup table
    int lut_n, lut_off;    // entries; index offset = -(magic bits) - kmin
    float G_lut;           // lookup-table bins per unit of v
    int L;                 // levels (2^bits)
    uint8_t* idx_out;      // packed indices
    int out_row_bytes;
    float* s_out;          // activations: s (fp32)
    uint16_t* r_out;       // weights: r (bf16)
    float* y_out;          // test hook: x' (fp32)
    float* norm_out;       // test hook: ||x'||
    float rsqrt_h;         // 1/sqrt(h)
    float eps;             // the split's eps
    float s_max;           // FLT_MAX / (2 sqrt(h)): larger row norms take the middle cell
    int starve;            // test hook: issue no row copies (the waits run out)
    uint32_t mid_val;      // value outputs: the middle cell's value (bf16 bits or e4m3 byte)
};

constexpr int kMaxGroups = 4;    // warp groups per CTA (at most 128 threads each)
constexpr int kMaxThreads = 384;  // per CTA: the kernel's launch bound (168 registers each)

int rpbh_smem_bytes(const RpbhParams& p);

// mode 0: activations (s fp32), 1: weights (r bf16), 2: rotation only (x', norm),
// 3 / 4: activations as centroid values, bf16 / e4m3 of c sqrt(d) (s fp32)
cudaError_t launch_rpbh_quant(const RpbhParams& p, bool in_bf16, int h, int bits, int mode, int grid,
                              cudaStream_t stream);

}  // namespace oq
