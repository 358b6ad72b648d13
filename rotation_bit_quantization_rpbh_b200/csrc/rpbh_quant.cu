// Fused RPBH rotate -> norm/direction split -> Lloyd-Max quantise -> pack.
//
// Method: "OrbitQuant" paper summary (hyper.ai, papers 2607.02461), section
// 方法 (Method):
//   x' = Pi_d x,  Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi;
//   s = ||x'||_2;  x~' = x' / (s + eps);  index = Q_b(x~') under C_d.
// The weight side runs the same kernel on the rows of W (row n of
// W' = W Pi_d^T is Pi_d w_n) and stores r_n as bf16.
//
// Design (sm_100a, HBM-bound):
//   - persistent CTAs, one per SM, each split into NG (1-4) warp groups that
//     take interleaved tiles of R rows and run out of phase (own staging buffers,
//     mbarriers and named barriers), so one group's gathers overlap the
//     others' butterflies and table lookups; a group stages its rows with
//     1-D bulk copies (cp.async.bulk), double buffered so its next tile
//     streams in while this one is computed;
//   - the gather and lookup tables arrive by bulk copy together with each
//     group's first rows;
//   - thread (r, b) owns row r's h-block b: it gathers the block's h inputs
//     x[pi(k)] from the staged row (the sign D is the gather table entry's
//     top bit, XORed into the bf16 sign) and runs the whole Walsh-Hadamard
//     butterfly in registers (packed f32x2 adds).  The row norm is the norm
//     of the gathered inputs (Pi_d is orthogonal, so ||x'|| = ||x||): its
//     cross-warp reduction is posted before the butterflies and read after;
//   - quantisation needs no search: bin(v) = rint(v G) (one fmaf with a
//     magic constant) indexes a small table holding, per bin, the count of
//     thresholds below it and the one threshold inside it, so
//     index = base + (v >= T) -- exactly #{ j : t_j <= v } in fp32;
//   - rows whose norm is not finite or exceeds FLT_MAX / (2 sqrt(h)) (where
//     the fp32 butterfly could overflow) take the middle cell;
//   - indices are packed LSB-first and written 16 bytes at a time as they
//     are produced;
//   - in the value modes the table entry holds, instead of the count, the
//     centroid values of the bin's two possible cells (bf16 or e4m3 of
//     c sqrt(d)), so the same compare selects C[index] itself, written as
//     bf16 pairs or e4m3 quads, 16 bytes at a time.
#include <cuda_bf16.h>

#include "device_util.cuh"
#include "oq_internal.h"
#include "rpbh_quant.cuh"

namespace oq {

namespace {

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

struct SmemLayout {
    int gtab, lut, stage, red, bar, total;
};

// gather table (u16 entries) | lookup table | NG groups x 2 staging buffers
// of R rows | NG groups' norm partials | mbarriers (2 per group + tables)
__host__ __device__ inline SmemLayout smem_layout(const RpbhParams& p) {
    SmemLayout L;
    L.gtab = 0;
    L.lut = align_up(p.d * 2, 16);
    L.stage = align_up(L.lut + p.lut_n * 8, 128);
    L.red = L.stage + p.NG * 2 * p.R * p.srow;
    L.bar = align_up(L.red + p.NG * (p.G / 32) * p.R * 4, 8);
    L.total = L.bar + 8 * (2 * p.NG + 1);
    return L;
}

__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ void group_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <typename InT, int H, int BITS, int MODE>
__global__ void __launch_bounds__(kMaxThreads, 1) rpbh_quant_kernel(const RpbhParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const SmemLayout L = smem_layout(p);
    const uint16_t* s_gtab = reinterpret_cast<const uint16_t*>(smem + L.gtab);
    __shared__ int s_abort[kMaxGroups];

    // NG warp groups per CTA work through interleaved tiles independently
    // (own staging buffers, mbarriers and named barrier), so one group's
    // gathers overlap the others' butterflies and table lookups.
    const int tid = threadIdx.x;
    const int G = p.G, R = p.R, nb = p.nb, NG = p.NG;
    const int grp = tid / G;
    const int tg = tid - grp * G;
    const int r = tg & (R - 1);
    const int b = tg / R;
    const bool active = b < nb;
    const int lane = tg & 31, warp = tg >> 5, nwarps = G >> 5;
    constexpr int ES = sizeof(InT);
    uint8_t* s_stage = smem + L.stage + grp * 2 * R * p.srow;
    float* s_red = reinterpret_cast<float*>(smem + L.red) + grp * nwarps * R;
    uint64_t* all_bars = reinterpret_cast<uint64_t*>(smem + L.bar);
    uint64_t* s_bar = all_bars + 2 * grp;
    uint64_t* tab_bar = all_bars + 2 * NG;

    // returns whether a copy was issued; a starved launch (test hook) issues
    // none, so the stage waits below run out and report a timeout
    auto issue = [&](uint64_t* bars, uint8_t* stage, int tile, int st) -> int {
        if (p.starve) return 0;
        const int row0 = tile * R;
        const int rows = min(R, p.M - row0);
        mbar_arrive_expect_tx(&bars[st], (uint32_t)(rows * p.row_bytes));
        const uint8_t* src = static_cast<const uint8_t*>(p.x) + (size_t)row0 * p.row_bytes;
        uint8_t* dst = stage + st * R * p.srow;
        for (int i = 0; i < rows; ++i) bulk_g2s(dst + i * p.srow, src + (size_t)i * p.row_bytes, p.row_bytes, &bars[st]);
        return 1;
    };

    // this group's tiles: blockIdx.x + (NG k + grp) * gridDim.x
    const int step = NG * gridDim.x;
    int tile = blockIdx.x + grp * gridDim.x;
    if (tid == 0) {
        for (int i = 0; i < 2 * NG + 1; ++i) mbar_init(&all_bars[i], 1);
        fence_mbar_init();
        for (int g = 0; g < kMaxGroups; ++g) s_abort[g] = 0;
        // gather and lookup tables, then each group's first rows: all in flight together
        const uint32_t lut_bytes = (uint32_t)(p.lut_n * 8);
        mbar_arrive_expect_tx(tab_bar, (uint32_t)(p.d * 2) + lut_bytes);
        bulk_g2s(smem + L.gtab, p.gtab, (uint32_t)(p.d * 2), tab_bar);
        if (lut_bytes) bulk_g2s(smem + L.lut, p.lut, lut_bytes, tab_bar);
        for (int g = 0; g < NG; ++g) {
            const int t0 = blockIdx.x + g * gridDim.x;
            if (t0 < p.ntiles) issue(all_bars + 2 * g, smem + L.stage + g * 2 * R * p.srow, t0, 0);
        }
    }
    __syncthreads();  // barriers initialised

    const float2 G2 = make_float2(p.G_lut, p.G_lut);
    const float2 M2 = make_float2(kLutMagic, kLutMagic);
    // shared address of lut[(bits of the magic-biased value) + lut_off], folded into one multiply-add
    const uint32_t lut_addr0 = smem_u32(smem) + (uint32_t)L.lut + (uint32_t)p.lut_off * 8u;
    constexpr int L2H = H / 2;
    int pending_other = 0;  // group leader: a copy into the other stage is in flight

    for (int it = 0; tile < p.ntiles; tile += step, ++it) {
        const int st = it & 1;
        const int next = tile + step;
        pending_other = 0;
        if (tg == 0 && next < p.ntiles) {
            pending_other = issue(s_bar, s_stage, next, st ^ 1);  // streams in while this tile is computed
        }
        if (it == 0 && !mbar_wait_bounded(tab_bar, 0u)) s_abort[grp] = 1;
        if (!mbar_wait_bounded(&s_bar[st], (uint32_t)((it >> 1) & 1))) s_abort[grp] = 1;
        group_sync(1 + grp, G);
        if (s_abort[grp]) {
            // give the prefetch into the other stage (bounded) time to land
            // before this CTA's shared memory goes away
            if (tg == 0 && pending_other) mbar_wait_bounded(&s_bar[st ^ 1], (uint32_t)(((it + 1) >> 1) & 1));
            break;
        }

        const int row = tile * R + r;
        const bool valid = active && row < p.M;

        // ---- A1 + A2: gather sigma_k x[pi(k)] (sign = top bit of the entry) ----
        // and the sum of squares of the gathered values: ||x'|| = ||x|| since
        // Pi_d is orthogonal, so the row norm is reduced across the row's
        // threads while the butterflies run
        float2 v2[L2H];
        float2 acc = make_float2(0.f, 0.f);
        if (valid) {
            const uint32_t rowp = smem_u32(s_stage) + (uint32_t)(st * R * p.srow + r * p.srow);
#pragma unroll
            for (int c = 0; c < H / 8; ++c) {
                const uint4 ch = reinterpret_cast<const uint4*>(s_gtab)[c * nb + b];
                const uint32_t w[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t e0 = w[e], e1 = w[e] >> 16;  // entry k in the low half, k+1 in the high half
                    float f0, f1;
                    if constexpr (ES == 2) {
                        uint32_t r0, r1;
                        asm volatile("ld.shared.u16 %0, [%1];" : "=r"(r0) : "r"(rowp + ((e0 & 0x7fffu) << 1)));
                        asm volatile("ld.shared.u16 %0, [%1];" : "=r"(r1) : "r"(rowp + ((e1 & 0x7fffu) << 1)));
                        // bf16 -> fp32 with the sign flipped where the entry's top bit is set
                        f0 = __uint_as_float((r0 ^ (e0 & 0x8000u)) << 16);
                        f1 = __uint_as_float((r1 ^ (e1 & 0x8000u)) << 16);
                    } else {
                        uint32_t r0, r1;
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r0) : "r"(rowp + ((e0 & 0x7fffu) << 2)));
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r1) : "r"(rowp + ((e1 & 0x7fffu) << 2)));
                        f0 = __uint_as_float(r0 ^ ((e0 & 0x8000u) << 16));
                        f1 = __uint_as_float(r1 ^ ((e1 & 0x8000u) << 16));
                    }
                    v2[c * 4 + e] = make_float2(f0, f1);
                    acc = f2fma(v2[c * 4 + e], v2[c * 4 + e], acc);
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < L2H; ++j) v2[j] = make_float2(0.f, 0.f);
        }

        // ---- A4 (first half): this block's sum of squares, summed over the
        // row's blocks within the warp, one partial per warp and row ----------
        float ss = acc.x + acc.y;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
            if (o >= R) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane < R) s_red[warp * R + lane] = ss;

        // ---- A3: unnormalised Walsh-Hadamard butterflies, Sylvester order ------
#pragma unroll
        for (int j = 0; j < L2H; ++j) {
            const float a = v2[j].x, c = v2[j].y;
            v2[j] = make_float2(a + c, a - c);
        }
#pragma unroll
        for (int hl = 1; hl < L2H; hl <<= 1) {
#pragma unroll
            for (int j = 0; j < L2H; ++j) {
                if ((j & hl) == 0) {
                    const float2 a = v2[j], c = v2[j + hl];
                    v2[j] = f2add(a, c);
                    v2[j + hl] = f2sub(a, c);
                }
            }
        }

        // ---- A4 (second half): the row norm s = ||x'|| ------------------------
        group_sync(1 + grp, G);
        float ssum = 0.f;
        for (int w = 0; w < nwarps; ++w) ssum += s_red[w * R + r];
        const float s = __fsqrt_rn(ssum);

        if (valid) {
            if (b == 0) {
                if constexpr (MODE == 0 || MODE >= 3) p.s_out[row] = s;
                if constexpr (MODE == 1) p.r_out[row] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
                if constexpr (MODE == 2) p.norm_out[row] = s;
            }
            if constexpr (MODE == 2) {
                float4* yo = reinterpret_cast<float4*>(p.y_out + (size_t)row * p.d + b * H);
                const float2 sc = make_float2(p.rsqrt_h, p.rsqrt_h);
#pragma unroll
                for (int j = 0; j < L2H; j += 2) {
                    const float2 a = f2mul(v2[j], sc), c = f2mul(v2[j + 1], sc);
                    yo[j >> 1] = make_float4(a.x, a.y, c.x, c.y);
                }
            } else if constexpr (MODE >= 3) {
                // ---- A5 with the centroid values written instead of the codes:
                // the table entry holds the values of both cells its bin can
                // give (the cell below the bin's threshold and the one above),
                // so one compare selects c_index directly ----------------------
                constexpr int VB = MODE == 3 ? 2 : 1;  // bytes per value: bf16, or e4m3
                uint4* dst = reinterpret_cast<uint4*>(p.idx_out + (size_t)row * p.out_row_bytes + (size_t)b * H * VB);
                if (s <= p.s_max) {
                    const float inv = p.rsqrt_h / (s + p.eps);
                    const float2 inv2 = make_float2(inv, inv);
                    // table word of element pair j and the selector bits of its two values
                    auto pick = [&](int j, uint32_t& val0, uint32_t& val1, uint32_t& ge0, uint32_t& ge1) {
                        const float2 q = f2mul(v2[j], inv2);
                        const float2 z = f2fma(q, G2, M2);
                        float T0, T1;
                        const uint32_t a0 = __float_as_uint(z.x) * 8u + lut_addr0;
                        const uint32_t a1 = __float_as_uint(z.y) * 8u + lut_addr0;
                        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(T0), "=r"(val0) : "r"(a0));
                        asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(T1), "=r"(val1) : "r"(a1));
                        ge0 = q.x >= T0 ? 1u : 0u;
                        ge1 = q.y >= T1 ? 1u : 0u;
                    };
#pragma unroll
                    for (int w0 = 0; w0 < H * VB / 4; w0 += 4) {
                        uint32_t words[4];
#pragma unroll
                        for (int wj = 0; wj < 4; ++wj) {
                            if constexpr (VB == 2) {
                                // bf16 pair: (lo or hi half of entry 0, lo or hi half of entry 1)
                                uint32_t val0, val1, ge0, ge1;
                                pick(w0 + wj, val0, val1, ge0, ge1);
                                words[wj] = prmt_b32(val0, val1, 0x5410u + ge0 * 0x22u + ge1 * 0x2200u);
                            } else {
                                // four e4m3 bytes: byte 0 or 1 of each entry's value word
                                uint32_t val0, val1, val2, val3, ge0, ge1, ge2, ge3;
                                pick(2 * (w0 + wj), val0, val1, ge0, ge1);
                                pick(2 * (w0 + wj) + 1, val2, val3, ge2, ge3);
                                const uint32_t lo = prmt_b32(val0, val1, 0x40u + ge0 + ge1 * 0x10u);
                                const uint32_t hi = prmt_b32(val2, val3, 0x40u + ge2 + ge3 * 0x10u);
                                words[wj] = prmt_b32(lo, hi, 0x5410u);
                            }
                        }
                        dst[w0 >> 2] = make_uint4(words[0], words[1], words[2], words[3]);
                    }
                } else {
                    // the middle cell's value everywhere (see the codes branch)
                    const uint32_t wm = VB == 2 ? p.mid_val * 0x10001u : p.mid_val * 0x01010101u;
#pragma unroll
                    for (int w0 = 0; w0 < H * VB / 4; w0 += 4) dst[w0 >> 2] = make_uint4(wm, wm, wm, wm);
                }
            } else {
                // ---- A5: v = x'/(s+eps) in fp32, index = #{ t_j <= v }, pack -----
                constexpr int NB = BITS == 6 ? H : H * BITS / 8;  // packed bytes per h-block
                constexpr int NW = NB / 4;
                constexpr int CW = NB % 16 == 0 ? 4 : (NB % 8 == 0 ? 2 : 1);  // words per store
                constexpr int PER = BITS == 6 ? 4 : (BITS == 3 ? 8 : 32 / BITS);  // codes per word (3-bit: per 24-bit group)
                constexpr uint32_t SH = BITS == 6 ? 256u : (1u << BITS);
                uint8_t* dst = p.idx_out + (size_t)row * p.out_row_bytes + (size_t)b * NB;
                auto put = [&](int w0, const uint32_t (&words)[CW]) {
                    if constexpr (CW == 4)
                        reinterpret_cast<uint4*>(dst)[w0 >> 2] = make_uint4(words[0], words[1], words[2], words[3]);
                    else if constexpr (CW == 2)
                        reinterpret_cast<uint2*>(dst)[w0 >> 1] = make_uint2(words[0], words[1]);
                    else
                        reinterpret_cast<uint32_t*>(dst)[w0] = words[0];
                };
                // s <= s_max keeps every butterfly value below sqrt(h) s (finite),
                // so |v| <= 1 up to rounding and the table index stays in range;
                // larger, infinite and NaN norms take the middle cell
                if (BITS == 3 && s <= p.s_max) {
                    // 3-bit: codes 8g..8g+7 form a 24-bit group (LSB first); four
                    // groups fill three words
                    const float inv = p.rsqrt_h / (s + p.eps);
                    const float2 inv2 = make_float2(inv, inv);
                    uint32_t words[NW];
#pragma unroll
                    for (int g4 = 0; g4 < H / 32; ++g4) {
                        uint32_t grp[4];
#pragma unroll
                        for (int gi = 0; gi < 4; ++gi) {
                            uint32_t acc_w = 0;
#pragma unroll
                            for (int k = 6; k >= 0; k -= 2) {
                                const float2 q = f2mul(v2[(32 * g4 + 8 * gi + k) >> 1], inv2);
                                const float2 z = f2fma(q, G2, M2);
                                float T0, T1;
                                int b0, b1;
                                const uint32_t a0 = __float_as_uint(z.x) * 8u + lut_addr0;
                                const uint32_t a1 = __float_as_uint(z.y) * 8u + lut_addr0;
                                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(T0), "=r"(b0) : "r"(a0));
                                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(T1), "=r"(b1) : "r"(a1));
                                const uint32_t i0 = (uint32_t)(b0 + (q.x >= T0 ? 1 : 0));
                                const uint32_t i1 = (uint32_t)(b1 + (q.y >= T1 ? 1 : 0));
                                acc_w = (acc_w * 8u + i1) * 8u + i0;
                            }
                            grp[gi] = acc_w;
                        }
                        words[3 * g4] = grp[0] | (grp[1] << 24);
                        words[3 * g4 + 1] = (grp[1] >> 8) | (grp[2] << 16);
                        words[3 * g4 + 2] = (grp[2] >> 16) | (grp[3] << 8);
                    }
#pragma unroll
                    for (int w0 = 0; w0 < NW; w0 += CW) {
                        uint32_t ws[CW];
#pragma unroll
                        for (int wj = 0; wj < CW; ++wj) ws[wj] = words[w0 + wj];
                        put(w0, ws);
                    }
                } else if (BITS != 3 && s <= p.s_max) {
                    // x'/(s+eps) = (H u / sqrt(h)) / (s + eps): one multiplier for the unnormalised butterflies
                    const float inv = p.rsqrt_h / (s + p.eps);
                    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
                    for (int w0 = 0; w0 < NW; w0 += CW) {
                        uint32_t words[CW];
#pragma unroll
                        for (int wj = 0; wj < CW; ++wj) {
                            const int wi = w0 + wj;
                            // codes of this word, highest position first: acc = acc * 2^bits + code
                            uint32_t acc_w = 0;
#pragma unroll
                            for (int k = PER - 2; k >= 0; k -= 2) {
                                const float2 q = f2mul(v2[(wi * PER + k) >> 1], inv2);
                                const float2 z = f2fma(q, G2, M2);
                                float T0, T1;
                                int b0, b1;
                                const uint32_t a0 = __float_as_uint(z.x) * 8u + lut_addr0;
                                const uint32_t a1 = __float_as_uint(z.y) * 8u + lut_addr0;
                                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(T0), "=r"(b0) : "r"(a0));
                                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(T1), "=r"(b1) : "r"(a1));
                                const uint32_t i0 = (uint32_t)(b0 + (q.x >= T0 ? 1 : 0));
                                const uint32_t i1 = (uint32_t)(b1 + (q.y >= T1 ? 1 : 0));
                                acc_w = (acc_w * SH + i1) * SH + i0;
                            }
                            words[wj] = acc_w;
                        }
                        put(w0, words);
                    }
                } else if (BITS == 3) {
                    // middle code 4 everywhere: the 3-bit stream repeats every 3 words
                    constexpr uint32_t g = 04444'4444u;  // eight 3-bit fours (octal)
                    const uint32_t pat[3] = {g | (g << 24), (g >> 8) | (g << 16), (g >> 16) | (g << 8)};
#pragma unroll
                    for (int w0 = 0; w0 < NW; w0 += CW) {
                        uint32_t ws[CW];
#pragma unroll
                        for (int wj = 0; wj < CW; ++wj) ws[wj] = pat[(w0 + wj) % 3];
                        put(w0, ws);
                    }
                } else {
                    uint32_t wmid = 0;
#pragma unroll
                    for (int k = 0; k < PER; ++k) wmid = wmid * SH + (uint32_t)(p.L >> 1);
                    uint32_t words[CW];
#pragma unroll
                    for (int wj = 0; wj < CW; ++wj) words[wj] = wmid;
#pragma unroll
                    for (int w0 = 0; w0 < NW; w0 += CW) put(w0, words);
                }
            }
        }
        group_sync(1 + grp, G);  // this stage and the partials are free for reuse
    }
}

template <typename InT, int H, int BITS, int MODE>
cudaError_t launch_rpbh_t(const RpbhParams& p, int grid, cudaStream_t stream) {
    auto k = rpbh_quant_kernel<InT, H, BITS, MODE>;
    const int smem = smem_layout(p).total;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    k<<<grid, p.T, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename InT, int H, int MODE>
cudaError_t launch_bits(const RpbhParams& p, int bits, int grid, cudaStream_t stream) {
    // the rotation alone and the value outputs do not depend on the code width
    if constexpr (MODE >= 2) {
        return launch_rpbh_t<InT, H, 4, MODE>(p, grid, stream);
    } else {
        switch (bits) {
            case 2: return launch_rpbh_t<InT, H, 2, MODE>(p, grid, stream);
            case 3:
                if constexpr (H >= 32) return launch_rpbh_t<InT, H, 3, MODE>(p, grid, stream);
                return cudaErrorInvalidValue;
            case 4: return launch_rpbh_t<InT, H, 4, MODE>(p, grid, stream);
            case 6: return launch_rpbh_t<InT, H, 6, MODE>(p, grid, stream);
            case 8: return launch_rpbh_t<InT, H, 8, MODE>(p, grid, stream);
        }
        return cudaErrorInvalidValue;
    }
}

template <typename InT, int MODE>
cudaError_t launch_h(const RpbhParams& p, int h, int bits, int grid, cudaStream_t stream) {
    switch (h) {
        case 16: return launch_bits<InT, 16, MODE>(p, bits, grid, stream);
        case 32: return launch_bits<InT, 32, MODE>(p, bits, grid, stream);
        case 64: return launch_bits<InT, 64, MODE>(p, bits, grid, stream);
        case 128: return launch_bits<InT, 128, MODE>(p, bits, grid, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

int rpbh_smem_bytes(const RpbhParams& p) { return smem_layout(p).total; }

cudaError_t launch_rpbh_quant(const RpbhParams& p, bool in_bf16, int h, int bits, int mode, int grid,
                              cudaStream_t stream) {
    if (in_bf16) {
        if (mode == 0) return launch_h<__nv_bfloat16, 0>(p, h, bits, grid, stream);
        if (mode == 1) return launch_h<__nv_bfloat16, 1>(p, h, bits, grid, stream);
        if (mode == 3) return launch_h<__nv_bfloat16, 3>(p, h, bits, grid, stream);
        if (mode == 4) return launch_h<__nv_bfloat16, 4>(p, h, bits, grid, stream);
        return launch_h<__nv_bfloat16, 2>(p, h, 4, grid, stream);
    }
    if (mode == 0) return launch_h<float, 0>(p, h, bits, grid, stream);
    if (mode == 1) return launch_h<float, 1>(p, h, bits, grid, stream);
    if (mode == 3) return launch_h<float, 3>(p, h, bits, grid, stream);
    if (mode == 4) return launch_h<float, 4>(p, h, bits, grid, stream);
    return launch_h<float, 2>(p, h, 4, grid, stream);
}

}  // namespace oq
