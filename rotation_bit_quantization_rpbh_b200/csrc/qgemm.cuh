// Launch interface of the codebook-decode tcgen05 GEMM (qgemm.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace oq {

struct QgemmArgs {
    int M, N, K;             // y[M, N] = decode(a_idx)[M, K] . decode(w_idx)[N, K]^T
    int bits_a, bits_w;      // 2, 4 or 6
    const uint8_t* a_idx;    // [M, K*bits_a/8] (bits 6: [M, K])
    const uint8_t* w_idx;    // [N, K*bits_w/8]
    const float* s;          // [M] activation norms
    const uint16_t* w_r;     // [N] bf16 weight row norms
    const uint16_t* bias;    // [N] bf16 or null
    uint16_t* y;             // [M, N] bf16
    const uint16_t* ca_bf16; // activation centroids (2^bits_a), bf16 bits
    const uint16_t* cw_bf16; // weight centroids (2^bits_w)
    bool fp8;                // e4m3 variant: centroids c_j sqrt(d) as e4m3, K % 128 == 0
    const uint8_t* ca_e4m3;  // activation centroids (fp8 variant)
    const uint8_t* cw_e4m3;  // weight centroids (fp8 variant)
    const void* a_val = nullptr;  // instead of a_idx: A as centroid values [M, K] (bf16, or e4m3 in the fp8 variant)
    bool starve = false;     // test hook: the producer issues no loads (the waits run out)
};

cudaError_t launch_qgemm(const QgemmArgs& a, cudaStream_t stream);

// Test and tuning hook: force the tile height of the A-values product
// (256 or 512 rows; 0: chosen per shape).
void qgemm_force_tile_rows(int rows);

}  // namespace oq
