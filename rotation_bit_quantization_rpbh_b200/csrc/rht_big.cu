// Rotate -> split -> quantise for Walsh-Hadamard blocks larger than the
// in-register kernel holds (h = 256 ... 16384), e.g. the rotation ablation's
// Full RHT, h = d.
//
// Method: "OrbitQuant" paper summary (hyper.ai, papers 2607.02461), section
// 方法 (Method), with the block size of the section 实验 (Experiments)
// rotation ablation: Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi (P_pi = I
// for Block-RHT and Full RHT), s = ||x'||, x~' = x' / (s + eps), index =
// #{ t_j <= x~'_k } -- the same definitions, tables and decision as the
// h <= 128 kernel (rpbh_quant.cu); only the butterfly schedule differs.
//
// Design: a CTA of 256 threads takes one row at a time.  The row arrives by
// one bulk copy into a staging buffer (refilled with the CTA's next row as
// soon as this one is gathered, so the copy overlaps the transform), is
// gathered through the plan's table (sign of D applied, fp32) into a work
// buffer, and the log2 h butterfly stages run in passes of at most 5 index
// bits: each thread loads a unit of up to 32 elements spaced by the pass's
// stride into registers, runs its stages and stores them back.  The work
// buffer is XOR-swizzled (element k lives at k ^ ((k >> 5) & 31)) so that the
// 32 lanes of a warp touch 32 different banks in every pass.  The row norm
// is reduced warp by warp and summed in a fixed order (deterministic).
#include <cuda_bf16.h>

#include "device_util.cuh"
#include "oq_internal.h"
#include "rpbh_quant.cuh"

namespace oq {
namespace {

constexpr int kBigThreads = 256;

__host__ __device__ constexpr int big_align(int x, int a) { return (x + a - 1) / a * a; }

struct BigLayout {
    int gtab, lut, stage, work, red, bar, flag, total;
};

// gather table | lookup table | staged row | fp32 work row | 8 warp
// partials | mbarriers (tables, row) | abort flag
__host__ __device__ inline BigLayout big_layout(const RpbhParams& p) {
    BigLayout L;
    L.gtab = 0;
    L.lut = big_align(p.d * 4, 16);
    L.stage = big_align(L.lut + p.lut_n * 8, 128);
    L.work = big_align(L.stage + p.row_bytes, 128);
    L.red = L.work + p.d * 4;
    L.bar = big_align(L.red + (kBigThreads / 32) * 4, 8);
    L.flag = L.bar + 16;
    L.total = L.flag + 16;
    return L;
}

__device__ __forceinline__ int swz(int k) { return k ^ ((k >> 5) & 31); }

__device__ __forceinline__ uint32_t big_prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// One pass: butterflies over index bits b0 .. b0 + log2(U) - 1 of every
// block, units of U elements spaced by S = 2^b0.
template <int U>
__device__ __forceinline__ void big_pass(float* work, int d, int kh, int b0, int tid) {
    const int S = 1 << b0;
    const int hi_n = (1 << kh) / (S * U);  // units per stride group and block
    const int units = d / U;
    for (int u = tid; u < units; u += kBigThreads) {
        const int lo = u & (S - 1);
        const int rest = u >> b0;
        const int hi = rest % hi_n;
        const int blk = rest / hi_n;
        const int base = (blk << kh) + hi * S * U + lo;
        float v[U];
#pragma unroll
        for (int m = 0; m < U; ++m) v[m] = work[swz(base + m * S)];
#pragma unroll
        for (int st = 1; st < U; st <<= 1) {
#pragma unroll
            for (int m = 0; m < U; ++m) {
                if ((m & st) == 0) {
                    const float a = v[m], c = v[m + st];
                    v[m] = a + c;
                    v[m + st] = a - c;
                }
            }
        }
#pragma unroll
        for (int m = 0; m < U; ++m) work[swz(base + m * S)] = v[m];
    }
}

template <typename InT, int BITS, int MODE>
__global__ void __launch_bounds__(kBigThreads) rht_big_kernel(const __grid_constant__ RpbhParams p, int kh) {
    extern __shared__ __align__(128) uint8_t smem[];
    const BigLayout L = big_layout(p);
    const uint32_t* s_gtab = reinterpret_cast<const uint32_t*>(smem + L.gtab);
    const uint8_t* s_stage = smem + L.stage;
    float* work = reinterpret_cast<float*>(smem + L.work);
    float* red = reinterpret_cast<float*>(smem + L.red);
    uint64_t* tab_bar = reinterpret_cast<uint64_t*>(smem + L.bar);
    uint64_t* row_bar = tab_bar + 1;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flag);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = p.d, h = 1 << kh;
    constexpr int ES = sizeof(InT);

    if (tid == 0) grid_launch_dependents();
    grid_dependency_wait();

    auto issue = [&](int row) {
        if (p.starve) return;
        mbar_arrive_expect_tx(row_bar, (uint32_t)p.row_bytes);
        bulk_g2s(smem + L.stage, static_cast<const uint8_t*>(p.x) + (size_t)row * p.row_bytes,
                 (uint32_t)p.row_bytes, row_bar);
    };
    if (tid == 0) {
        mbar_init(tab_bar, 1);
        mbar_init(row_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        if (!p.starve) {
            const uint32_t gbytes = (uint32_t)(d * 4), lbytes = (uint32_t)(p.lut_n * 8);
            mbar_arrive_expect_tx(tab_bar, gbytes + lbytes);
            bulk_g2s(smem + L.gtab, p.gtab, gbytes, tab_bar);
            if (lbytes) bulk_g2s(smem + L.lut, p.lut, lbytes, tab_bar);
        }
        if ((int)blockIdx.x < p.M) issue(blockIdx.x);
    }
    __syncthreads();

    const float G = p.G_lut, MG = kLutMagic;
    const uint32_t lut_addr0 = smem_u32(smem) + (uint32_t)L.lut + (uint32_t)p.lut_off * 8u;
    int it = 0, pending = ((int)blockIdx.x < p.M && !p.starve) ? 1 : 0;
    for (int row = blockIdx.x; row < p.M; row += gridDim.x, ++it) {
        bool ok = true;
        if (it == 0 && !mbar_wait_bounded(tab_bar, 0u)) ok = false;
        if (ok && !mbar_wait_bounded(row_bar, (uint32_t)(it & 1))) ok = false;
        if (!__syncthreads_and(ok)) break;
        pending = 0;

        // ---- A1 + A2: gather sigma_k x[pi(k)] into the fp32 work row ----
        float ss = 0.f;
        for (int k = tid; k < d; k += kBigThreads) {
            const int b = k >> kh, i = k & (h - 1);
            const uint32_t e = s_gtab[((((i >> 2) * p.nb) + b) << 2) + (i & 3)];
            float f;
            if constexpr (ES == 2) {
                const uint32_t rv = *reinterpret_cast<const uint16_t*>(s_stage + (e >> 16));
                f = __uint_as_float((rv + e) << 16);
            } else {
                const uint32_t rv = *reinterpret_cast<const uint32_t*>(s_stage + ((e >> 16) << 1));
                f = __uint_as_float(rv ^ (e << 16));
            }
            work[swz(k)] = f;
            ss = fmaf(f, f, ss);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) red[warp] = ss;
        __syncthreads();  // the staged row is gathered: refill it with the next row
        if (tid == 0 && row + (int)gridDim.x < p.M) {
            issue(row + gridDim.x);
            pending = !p.starve;
        }
        float ssum = 0.f;
        for (int w = 0; w < kBigThreads / 32; ++w) ssum += red[w];
        const float s = __fsqrt_rn(ssum);

        // ---- A3: unnormalised Walsh-Hadamard stages, 5 index bits per pass ----
        for (int b0 = 0; b0 < kh; b0 += 5) {
            const int nbits = kh - b0 < 5 ? kh - b0 : 5;
            if (nbits == 5) big_pass<32>(work, d, kh, b0, tid);
            else if (nbits == 4) big_pass<16>(work, d, kh, b0, tid);
            else if (nbits == 3) big_pass<8>(work, d, kh, b0, tid);
            else if (nbits == 2) big_pass<4>(work, d, kh, b0, tid);
            else big_pass<2>(work, d, kh, b0, tid);
            __syncthreads();
        }

        // ---- A4 + A5: outputs, 16 elements per thread and step ----
        if (tid == 0) {
            if constexpr (MODE == 0 || MODE >= 3) p.s_out[row] = s;
            if constexpr (MODE == 1) p.r_out[row] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
            if constexpr (MODE == 2) p.norm_out[row] = s;
        }
        const bool in_range = s <= p.s_max;
        const float inv = p.rsqrt_h / (s + p.eps);
        for (int g = tid; g < d / 16; g += kBigThreads) {
            float q[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) q[m] = work[swz(16 * g + m)];
            if constexpr (MODE == 2) {
                float4* yo = reinterpret_cast<float4*>(p.y_out + (size_t)row * d + 16 * g);
#pragma unroll
                for (int m = 0; m < 16; m += 4)
                    yo[m >> 2] = make_float4(q[m] * p.rsqrt_h, q[m + 1] * p.rsqrt_h, q[m + 2] * p.rsqrt_h,
                                             q[m + 3] * p.rsqrt_h);
            } else {
                // the same decision as the h <= 128 kernel: bin(v) = rint(v G), then v >= T of the bin.
                // Rows whose norm is out of range (not finite, or where the fp32
                // transform could overflow) take the middle cell and read no table.
                uint32_t w[16];  // table word: base (codes) or the bin's two values
                uint32_t ge[16];
                if (in_range) {
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float v = q[m] * inv;
                        const float z = fmaf(v, G, MG);
                        float T;
                        asm("ld.shared.v2.b32 {%0, %1}, [%2];"
                            : "=f"(T), "=r"(w[m])
                            : "r"(__float_as_uint(z) * 8u + lut_addr0));
                        ge[m] = v >= T ? 1u : 0u;
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < 16; ++m) w[m] = ge[m] = 0u;
                }
                uint8_t* rowo = p.idx_out + (size_t)row * p.out_row_bytes;
                if constexpr (MODE == 3) {  // bf16 values
                    uint32_t o[8];
#pragma unroll
                    for (int m = 0; m < 16; m += 2)
                        o[m >> 1] = in_range ? big_prmt(w[m], w[m + 1], 0x5410u + ge[m] * 0x22u + ge[m + 1] * 0x2200u)
                                             : p.mid_val * 0x10001u;
                    uint4* dst = reinterpret_cast<uint4*>(rowo + (size_t)32 * g);
                    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                } else if constexpr (MODE == 4) {  // e4m3 values
                    uint32_t o[4];
#pragma unroll
                    for (int m = 0; m < 16; m += 4) {
                        const uint32_t lo = big_prmt(w[m], w[m + 1], 0x40u + ge[m] + ge[m + 1] * 0x10u);
                        const uint32_t hi = big_prmt(w[m + 2], w[m + 3], 0x40u + ge[m + 2] + ge[m + 3] * 0x10u);
                        o[m >> 2] = in_range ? big_prmt(lo, hi, 0x5410u) : p.mid_val * 0x01010101u;
                    }
                    *reinterpret_cast<uint4*>(rowo + (size_t)16 * g) = make_uint4(o[0], o[1], o[2], o[3]);
                } else {
                    uint32_t idx[16];
#pragma unroll
                    for (int m = 0; m < 16; ++m) idx[m] = in_range ? w[m] + ge[m] : (uint32_t)(p.L >> 1);
                    if constexpr (BITS == 4) {
                        uint32_t o0 = 0, o1 = 0;
#pragma unroll
                        for (int m = 7; m >= 0; --m) {
                            o0 = o0 * 16u + idx[m];
                            o1 = o1 * 16u + idx[m + 8];
                        }
                        *reinterpret_cast<uint2*>(rowo + (size_t)8 * g) = make_uint2(o0, o1);
                    } else if constexpr (BITS == 2) {
                        uint32_t o0 = 0;
#pragma unroll
                        for (int m = 15; m >= 0; --m) o0 = o0 * 4u + idx[m];
                        *reinterpret_cast<uint32_t*>(rowo + (size_t)4 * g) = o0;
                    } else {  // 6 and 8 bits: one code per byte
                        uint32_t o[4];
#pragma unroll
                        for (int m = 0; m < 16; m += 4)
                            o[m >> 2] = idx[m] | (idx[m + 1] << 8) | (idx[m + 2] << 16) | (idx[m + 3] << 24);
                        *reinterpret_cast<uint4*>(rowo + (size_t)16 * g) = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        }
        __syncthreads();  // the work row is free for the next row
    }
    // a copy in flight must land before the CTA's shared memory goes away
    if (tid == 0 && pending) mbar_wait_bounded(row_bar, (uint32_t)(it & 1));
    if (tid == 0 && !p.starve) mbar_wait_bounded(tab_bar, 0u);
}

template <typename InT, int BITS, int MODE>
cudaError_t launch_big_t(const RpbhParams& p, int kh, int grid, cudaStream_t stream) {
    auto k = rht_big_kernel<InT, BITS, MODE>;
    const int smem = big_layout(p).total;
    static int smem_done[kSmemRecordDevices] = {0};  // this instantiation's limit, per device
    const cudaError_t e = ensure_smem_limit(k, smem, smem_done);
    if (e != cudaSuccess) return e;
    const cudaError_t le = launch_pdl(k, dim3(grid), dim3(kBigThreads), smem, stream, p, kh);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

template <typename InT, int MODE>
cudaError_t launch_big_bits(const RpbhParams& p, int kh, int bits, int grid, cudaStream_t stream) {
    if constexpr (MODE >= 2) {
        return launch_big_t<InT, 4, MODE>(p, kh, grid, stream);
    } else {
        switch (bits) {
            case 2: return launch_big_t<InT, 2, MODE>(p, kh, grid, stream);
            case 4: return launch_big_t<InT, 4, MODE>(p, kh, grid, stream);
            case 6: return launch_big_t<InT, 6, MODE>(p, kh, grid, stream);
            case 8: return launch_big_t<InT, 8, MODE>(p, kh, grid, stream);
        }
        return cudaErrorInvalidValue;
    }
}

}  // namespace

int rht_big_smem_bytes(const RpbhParams& p) { return big_layout(p).total; }

cudaError_t launch_rht_big(const RpbhParams& p, bool in_bf16, int h, int bits, int mode, int grid,
                           cudaStream_t stream) {
    int kh = 0;
    while ((1 << kh) < h) ++kh;
    if (in_bf16) {
        if (mode == 0) return launch_big_bits<__nv_bfloat16, 0>(p, kh, bits, grid, stream);
        if (mode == 1) return launch_big_bits<__nv_bfloat16, 1>(p, kh, bits, grid, stream);
        if (mode == 3) return launch_big_bits<__nv_bfloat16, 3>(p, kh, bits, grid, stream);
        if (mode == 4) return launch_big_bits<__nv_bfloat16, 4>(p, kh, bits, grid, stream);
        return launch_big_bits<__nv_bfloat16, 2>(p, kh, 4, grid, stream);
    }
    if (mode == 0) return launch_big_bits<float, 0>(p, kh, bits, grid, stream);
    if (mode == 1) return launch_big_bits<float, 1>(p, kh, bits, grid, stream);
    if (mode == 3) return launch_big_bits<float, 3>(p, kh, bits, grid, stream);
    if (mode == 4) return launch_big_bits<float, 4>(p, kh, bits, grid, stream);
    return launch_big_bits<float, 2>(p, kh, 4, grid, stream);
}

}  // namespace oq
