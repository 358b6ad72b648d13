// Fused RPBH rotate -> norm/direction split -> Lloyd-Max quantise -> pack:
// the team kernel, and the quantiser epilogue (store_unit) that it shares
// with the warp-group kernel (rpbh_groups.cu).  The library runs the team
// kernel for blocks of at most 128 when d > 8192 or when the plan has no
// permutation (its contiguous read path); the warp-group kernel takes
// permuted plans up to d = 8192, and rht_big.cu blocks of 256 and more.
//
// Method: "OrbitQuant" paper summary (hyper.ai, papers 2607.02461), section
// 方法 (Method):
//   x' = Pi_d x,  Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi;
//   s = ||x'||_2;  x~' = x' / (s + eps);  index = Q_b(x~') under C_d.
// The weight side runs the same kernel on the rows of W (row n of
// W' = W Pi_d^T is Pi_d w_n) and stores r_n as bf16.
//
// Design (sm_100a, HBM-bound):
//   - persistent CTAs, one per SM.  A lane owns one (row, h-block) unit: a
//     warp covers RW rows x 32/RW blocks, and a team of warps covers all the
//     blocks of a set of RW rows.  Teams run independently: each has its own
//     staging slots (a row set arrives by one 1-D bulk copy per row into a
//     slot, completing on that slot's mbarrier) and the team's first warp
//     refills a slot with the team's next row set as soon as every warp of
//     the team has gathered from it, so the copy overlaps the butterflies
//     and the table lookups.  There is no CTA-wide barrier in the loop.
//   - rows of a slot are padded so that the RW rows a warp gathers from fall
//     on different banks; several rows per warp make the random gather of a
//     warp touch fewer words per bank than 32 random columns of one row;
//   - the gather table holds, per post-permutation coordinate k, the byte
//     offset of x[pi(k)] in the row and the sign of D (bit 15), so the sign
//     flip and the bf16 -> fp32 widening are one add and one shift; the RW
//     lanes of one block read the same table words (a broadcast);
//   - the lane runs the whole Walsh-Hadamard butterfly in registers (packed
//     f32x2 adds).  The row norm is the norm of the gathered inputs (Pi_d is
//     orthogonal, so ||x'|| = ||x||): it is summed across the block's lanes
//     by shuffles and across the team's warps through shared memory and a
//     per-team mbarrier, in a fixed order (deterministic), and the exchange
//     overlaps the butterflies;
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
// Every mbarrier wait is bounded; a wait that runs out raises the device
// error flag and a CTA-wide abort flag, every warp leaves its loop, and the
// copies this CTA issued are drained (bounded) before it exits.
#include <cuda_bf16.h>

#include "device_util.cuh"
#include "oq_internal.h"
#include "rpbh_quant.cuh"

namespace oq {

namespace {

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

struct SmemLayout {
    int gtab, lut, stage, part, bar, flag, total;
};

// gather table (u32 entries) | lookup table | tpc teams x slots x RW staged
// rows | norm partials (tpc teams x 2 row sets x team warps x RW rows) |
// mbarriers (tables, full and empty per slot, norm per team and parity) |
// abort flag
__host__ __device__ inline SmemLayout smem_layout(const RpbhParams& p) {
    SmemLayout L;
    L.gtab = 0;
    L.lut = align_up(p.d * 4, 16);
    L.stage = align_up(L.lut + p.lut_n * 8, 128);
    L.part = L.stage + p.tpc * p.slots * p.RW * p.srow;
    L.bar = align_up(L.part + p.tpc * 2 * p.team * p.RW * 4, 8);
    L.flag = L.bar + 8 * (1 + 2 * p.tpc * p.slots + 2 * p.tpc);
    L.total = L.flag + 16;
    return L;
}

__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Bounded wait that also gives up once another warp of the CTA aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (clock64() - t0 > kWaitLimitCycles) {
            atomicExch(&g_error_flag, kErrTimeout);
            *abort_flag = 1;
            return false;
        }
    }
    return true;
}

// The same, by every lane of the warp, with a warp-uniform result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    const bool ok = wait_or_abort(bar, parity, abort_flag);
    return __all_sync(0xffffffffu, ok);
}

// Lookup-table entry at a 32-bit shared-memory address: {T, base or values}.
// Its address depends on the gathered values, which are loaded after the
// table's mbarrier wait, so it cannot move above that wait; it is left free
// to be scheduled (and merged) otherwise.
__device__ __forceinline__ void lut_ld(uint32_t addr, float& T, uint32_t& w) {
    asm("ld.shared.v2.b32 {%0, %1}, [%2];" : "=f"(T), "=r"(w) : "r"(addr));
}

// Shared-memory loads at 32-bit shared addresses (explicit ld.shared).  The
// tables and staged rows arrive by bulk copy, so every load that reads them
// is volatile with a memory clobber: it stays after the mbarrier wait that
// covers the copy (a load whose address depends on nothing loaded after the
// wait could otherwise be moved above it, or out of the loop).
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// 32 bytes of output at a 32-byte-aligned global address: one 256-bit
// store when the launch's output rows are 32-byte aligned throughout
// (p.st32: the base and the row pitch), else two 16-byte stores.  A lane
// writes its own h-block, so the stores of a warp go to 32 different rows
// or blocks; whole 32-byte sectors halve the store instructions and the L2
// sector updates against 16-byte halves.
__device__ __forceinline__ void st_32B(uint8_t* dst, const uint32_t (&w)[8], int st32) {
    if (st32) {
        asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(__cvta_generic_to_global(dst)),
                     "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                     : "memory");
    } else {
        uint4* d = reinterpret_cast<uint4*>(dst);
        d[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
}

// A5 for one lane's HL values of row `row`: v2 holds the unnormalised
// butterfly outputs of columns unit*HL .. unit*HL + HL-1 and s the row norm.
// Writes the norm (the lane of unit 0), then the rotation (test mode), the
// centroid values or the packed codes of those columns.
template <int HL, int BITS, int MODE>
__device__ __forceinline__ void store_unit(const RpbhParams& p, float2 (&v2)[HL / 2], float s, int row, int unit,
                                           uint32_t lut_addr0) {
    constexpr int L2H = HL / 2;
    const float2 G2 = make_float2(p.G_lut, p.G_lut);
    const float2 M2 = make_float2(kLutMagic, kLutMagic);
    if (unit == 0) {
        if constexpr (MODE == 0 || MODE >= 3) p.s_out[row] = s;
        if constexpr (MODE == 1) p.r_out[row] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
        if constexpr (MODE == 2) p.norm_out[row] = s;
    }
    if constexpr (MODE == 2) {
        float4* yo = reinterpret_cast<float4*>(p.y_out + (size_t)row * p.d + (size_t)unit * HL);
        const float2 sc = make_float2(p.rsqrt_h, p.rsqrt_h);
#pragma unroll
        for (int i = 0; i < L2H; i += 2) {
            const float2 a = f2mul(v2[i], sc), c = f2mul(v2[i + 1], sc);
            yo[i >> 1] = make_float4(a.x, a.y, c.x, c.y);
        }
    } else if constexpr (MODE >= 3) {
        // ---- A5 with the centroid values written instead of the codes:
        // the table entry holds the values of both cells its bin can
        // give (the cell below the bin's threshold and the one above),
        // so one compare selects c_index directly ----------------------
        constexpr int VB = MODE == 3 ? 2 : 1;  // bytes per value: bf16, or e4m3
        uint4* dst = reinterpret_cast<uint4*>(p.idx_out + (size_t)row * p.out_row_bytes + (size_t)unit * HL * VB);
        if (s <= p.s_max) {
            const float inv = p.rsqrt_h / (s + p.eps);
            const float2 inv2 = make_float2(inv, inv);
            // table word of element pair i and the selector bits of its two values
            auto pick = [&](int i, uint32_t& val0, uint32_t& val1, uint32_t& ge0, uint32_t& ge1) {
                const float2 q = f2mul(v2[i], inv2);
                const float2 z = f2fma(q, G2, M2);
                float T0, T1;
                lut_ld(__float_as_uint(z.x) * 8u + lut_addr0, T0, val0);
                lut_ld(__float_as_uint(z.y) * 8u + lut_addr0, T1, val1);
                ge0 = q.x >= T0 ? 1u : 0u;
                ge1 = q.y >= T1 ? 1u : 0u;
            };
            constexpr int SW = (HL * VB) % 32 == 0 ? 8 : 4;  // words per store: 32 bytes where the unit holds them
#pragma unroll
            for (int w0 = 0; w0 < HL * VB / 4; w0 += SW) {
                uint32_t words[SW];
#pragma unroll
                for (int wj = 0; wj < SW; ++wj) {
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
                if constexpr (SW == 8)
                    st_32B(reinterpret_cast<uint8_t*>(dst + (w0 >> 2)), words, p.st32);
                else
                    dst[w0 >> 2] = make_uint4(words[0], words[1], words[2], words[3]);
            }
        } else {
            // the middle cell's value everywhere (see the codes branch)
            const uint32_t wm = VB == 2 ? p.mid_val * 0x10001u : p.mid_val * 0x01010101u;
#pragma unroll
            for (int w0 = 0; w0 < HL * VB / 4; w0 += 4) dst[w0 >> 2] = make_uint4(wm, wm, wm, wm);
        }
    } else {
        // ---- A5: v = x'/(s+eps) in fp32, index = #{ t_j <= v }, pack -----
        constexpr int NB = BITS == 6 ? HL : HL * BITS / 8;  // packed bytes of the lane's codes
        constexpr int NW = NB / 4;
        constexpr int CW = NB % 32 == 0 ? 8 : (NB % 16 == 0 ? 4 : (NB % 8 == 0 ? 2 : 1));  // words per store
        constexpr int PER = BITS == 6 ? 4 : (BITS == 3 ? 8 : 32 / BITS);  // codes per word (3-bit: per 24-bit group)
        constexpr uint32_t SH = BITS == 6 ? 256u : (1u << BITS);
        uint8_t* dst = p.idx_out + (size_t)row * p.out_row_bytes + (size_t)unit * NB;
        auto put = [&](int w0, const uint32_t (&words)[CW]) {
            if constexpr (CW == 8)
                st_32B(dst + (size_t)w0 * 4, words, p.st32);
            else if constexpr (CW == 4)
                reinterpret_cast<uint4*>(dst)[w0 >> 2] = make_uint4(words[0], words[1], words[2], words[3]);
            else if constexpr (CW == 2)
                reinterpret_cast<uint2*>(dst)[w0 >> 1] = make_uint2(words[0], words[1]);
            else
                reinterpret_cast<uint32_t*>(dst)[w0] = words[0];
        };
        // code of element pair i: (index of .x, index of .y)
        auto code2 = [&](int i, float2 inv2, uint32_t& i0, uint32_t& i1) {
            const float2 q = f2mul(v2[i], inv2);
            const float2 z = f2fma(q, G2, M2);
            float T0, T1;
            uint32_t b0, b1;
            lut_ld(__float_as_uint(z.x) * 8u + lut_addr0, T0, b0);
            lut_ld(__float_as_uint(z.y) * 8u + lut_addr0, T1, b1);
            i0 = b0 + (q.x >= T0 ? 1u : 0u);
            i1 = b1 + (q.y >= T1 ? 1u : 0u);
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
            for (int g4 = 0; g4 < HL / 32; ++g4) {
                uint32_t grp[4];
#pragma unroll
                for (int gi = 0; gi < 4; ++gi) {
                    uint32_t acc_w = 0;
#pragma unroll
                    for (int kk = 6; kk >= 0; kk -= 2) {
                        uint32_t i0, i1;
                        code2((32 * g4 + 8 * gi + kk) >> 1, inv2, i0, i1);
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
                    for (int kk = PER - 2; kk >= 0; kk -= 2) {
                        uint32_t i0, i1;
                        code2((wi * PER + kk) >> 1, inv2, i0, i1);
                        acc_w = (acc_w * SH + i1) * SH + i0;
                    }
                    words[wj] = acc_w;
                }
                put(w0, words);
            }
        } else if (BITS == 3) {
            // middle code 4 everywhere: the 3-bit stream repeats every 3 words
            constexpr uint32_t gm = 04444'4444u;  // eight 3-bit fours (octal)
            const uint32_t pat[3] = {gm | (gm << 24), (gm >> 8) | (gm << 16), (gm >> 16) | (gm << 8)};
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
            for (int kk = 0; kk < PER; ++kk) wmid = wmid * SH + (uint32_t)(p.L >> 1);
            uint32_t words[CW];
#pragma unroll
            for (int wj = 0; wj < CW; ++wj) words[wj] = wmid;
#pragma unroll
            for (int w0 = 0; w0 < NW; w0 += CW) put(w0, words);
        }
    }
}

// CONTIG: the plan's permutation is the identity (Block-RHT, the rotation
// ablation without P_pi), so a block's inputs are contiguous and are read
// 16 bytes at a time instead of gathered one by one.
template <typename InT, int H, int BITS, int MODE, int SPL, bool CONTIG>
__global__ void __launch_bounds__(SPL == 2 ? kMaxThreadsSplit : kMaxThreads, 1)
    rpbh_quant_kernel(const __grid_constant__ RpbhParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const SmemLayout L = smem_layout(p);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
    uint64_t* tab_bar = bars;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flag);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = warp / p.team, wt = warp - t * p.team;  // team, warp within the team
    // SPL lanes per h-block: lane = ((j * RW + r) * SPL + hf) -- block-major,
    // so the 8 lanes of one phase of a 16-byte load are 8 rows of a block,
    // whose row pads put them on different banks; with SPL = 2 each lane
    // holds half of the block's values (see the gather)
    constexpr int LSPL = SPL == 2 ? 1 : 0;
    const int hf = lane & (SPL - 1);
    const int Bw = 1 << p.lbw;
    const int r = (lane >> LSPL) & (p.RW - 1), j = lane >> (LSPL + p.lrw);  // row within the set, block within the warp
    const int b = wt * Bw + j;                            // h-block of this lane
    const bool bact = b < p.nb;
    const bool loader = wt == 0 && lane == 0;             // issues the team's row copies
    uint64_t* my_full = bars + 1 + t * p.slots;
    uint64_t* my_empty = bars + 1 + p.tpc * p.slots + t * p.slots;
    uint64_t* my_norm = bars + 1 + 2 * p.tpc * p.slots + 2 * t;
    uint8_t* my_stage = smem + L.stage + t * p.slots * p.RW * p.srow;
    float* my_part = reinterpret_cast<float*>(smem + L.part) + t * 2 * p.team * p.RW;
    constexpr int ES = sizeof(InT);
    static_assert(SPL == 1 || ES == 2, "two lanes per block exchange bf16 inputs");
    constexpr int HL = H / SPL;  // values per lane
    constexpr int L2H = HL / 2;

    // this team's row sets: g = k * (gridDim.x * tpc) + t * gridDim.x + blockIdx.x
    const int stride = gridDim.x * p.tpc;
    const int g0 = t * gridDim.x + blockIdx.x;

    // Launched with programmatic serialisation: the set-up above may overlap
    // the end of the kernel before this one in the stream; every global
    // access (tables, rows, outputs) comes after this wait.
    if (tid == 0) grid_launch_dependents();
    grid_dependency_wait();

    if (tid == 0) {
        const int nbar = 1 + 2 * p.tpc * p.slots + 2 * p.tpc;
        for (int i = 0; i < nbar; ++i) {
            const bool team_count = i >= 1 + p.tpc * p.slots;  // empty and norm barriers: one arrival per warp
            mbar_init(&bars[i], team_count ? (uint32_t)p.team : 1u);
        }
        *abort_flag = 0;
        fence_mbar_init();
        if (!p.starve) {
            const uint32_t gbytes = (uint32_t)(p.d * 4), lbytes = (uint32_t)(p.lut_n * 8);
            mbar_arrive_expect_tx(tab_bar, gbytes + lbytes);
            bulk_g2s(smem + L.gtab, p.gtab, gbytes, tab_bar);
            if (lbytes) bulk_g2s(smem + L.lut, p.lut, lbytes, tab_bar);
        }
    }
    __syncthreads();  // barriers initialised

    // loader: copy row set g into slot `slot` (a starved launch copies nothing)
    int issued_k[2] = {-1, -1};  // iteration whose rows were last copied into each slot
    auto issue = [&](int slot, int g, int k) {
        if (p.starve) return;
        const int row0 = g * p.RW;
        const int rows = min(p.RW, p.M - row0);
        uint64_t* bar = &my_full[slot];
        mbar_arrive_expect_tx(bar, (uint32_t)(rows * p.row_bytes));
        const uint8_t* src = static_cast<const uint8_t*>(p.x) + (size_t)row0 * p.row_bytes;
        uint8_t* dst = my_stage + slot * p.RW * p.srow;
        for (int i = 0; i < rows; ++i) bulk_g2s(dst + i * p.srow, src + (size_t)i * p.row_bytes, p.row_bytes, bar);
        issued_k[slot] = k;
    };
    if (loader)
        for (int i = 0; i < p.slots; ++i)
            if (g0 + i * stride < p.nrs) issue(i, g0 + i * stride, i);

    // shared address of lut[(bits of the magic-biased value) + lut_off]
    const uint32_t lut_addr0 = smem_u32(smem) + (uint32_t)L.lut + (uint32_t)p.lut_off * 8u;
    const uint32_t gtab_addr = smem_u32(smem) + (uint32_t)L.gtab;  // table chunks, 16 bytes each
    const uint32_t stage_addr = smem_u32(my_stage);

    // a slot refill that waits for the team's gathers (loader only)
    int pend_slot = -1, pend_g = 0, pend_k = 0;
    uint32_t pend_ph = 0;
    int consumed_k = -1;  // last iteration whose rows this warp waited for
    bool ok = true;
    int k = 0;
    for (int g = g0; g < p.nrs; g += stride, ++k) {
        const int slot = p.slots == 1 ? 0 : (k & 1);
        const uint32_t ph = (uint32_t)((p.slots == 1 ? k : (k >> 1)) & 1);
        // a deferred refill must be issued before this wait (with one slot it is this one)
        if (loader && pend_slot >= 0) {
            if (wait_or_abort(&my_empty[pend_slot], pend_ph, abort_flag)) issue(pend_slot, pend_g, pend_k);
            else ok = false;
            pend_slot = -1;
        }
        if (wt == 0) ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (k == 0 && !warp_wait(tab_bar, 0u, abort_flag)) {
            ok = false;
            break;
        }
        if (!warp_wait(&my_full[slot], ph, abort_flag)) {
            ok = false;
            break;
        }
        consumed_k = k;

        const int row = g * p.RW + r;
        const bool valid = bact && row < p.M;

        // ---- A1 + A2: gather sigma_k x[pi(k)] and the sum of squares -------
        // (||x'|| = ||x|| since Pi_d is orthogonal)
        float2 v2[L2H];
        float2 acc = make_float2(0.f, 0.f);
        if constexpr (SPL == 2) {
            // the lane's half of the block: entries hf*HL .. hf*HL + HL-1, kept
            // as signed bf16 pairs; the pair of lanes swaps them (every lane
            // takes part in the shuffles) and runs the top butterfly stage
            // across the pair: the low lane takes u_lo + u_hi, the high lane
            // u_lo - u_hi (H_128 = [[H64, H64], [H64, -H64]])
            uint32_t pk[L2H];
            if (valid) {
                const uint32_t rowp = stage_addr + (uint32_t)(slot * p.RW * p.srow + r * p.srow);
                const uint32_t tabp = gtab_addr + (uint32_t)b * 16u + (uint32_t)(hf * (HL / 4) * p.nb) * 16u;
#pragma unroll
                for (int c4 = 0; c4 < HL / 4; ++c4) {
                    const uint4 ch = lds_v4(tabp + (uint32_t)(c4 * p.nb) * 16u);
                    const uint32_t e[4] = {ch.x, ch.y, ch.z, ch.w};
                    uint32_t sv[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) sv[q] = lds_u16(rowp + (e[q] >> 16)) + e[q];  // bit 15: sign of D
                    pk[2 * c4] = prmt_b32(sv[0], sv[1], 0x5410u);
                    pk[2 * c4 + 1] = prmt_b32(sv[2], sv[3], 0x5410u);
                }
            } else {
#pragma unroll
                for (int i = 0; i < L2H; ++i) pk[i] = 0u;
            }
            const float2 sgn2 = hf ? make_float2(-1.f, -1.f) : make_float2(1.f, 1.f);
#pragma unroll
            for (int k2 = 0; k2 < L2H; ++k2) {
                const uint32_t o = __shfl_xor_sync(0xffffffffu, pk[k2], 1);
                const float2 own = make_float2(__uint_as_float(pk[k2] << 16), __uint_as_float(pk[k2] & 0xffff0000u));
                const float2 oth = make_float2(__uint_as_float(o << 16), __uint_as_float(o & 0xffff0000u));
                acc = f2fma(own, own, acc);
                v2[k2] = f2fma(own, sgn2, oth);
            }
        } else if (!valid) {
#pragma unroll
            for (int i = 0; i < L2H; ++i) v2[i] = make_float2(0.f, 0.f);
        } else if constexpr (CONTIG) {
            // identity permutation: the block's h inputs are contiguous in the
            // row; 16-byte loads, the signs of D from the table's bit 15
            const uint32_t rowp = stage_addr + (uint32_t)(slot * p.RW * p.srow + r * p.srow) + (uint32_t)(b * H * ES);
            const uint32_t tabp = gtab_addr + (uint32_t)b * 16u;
            constexpr int PER16 = 16 / ES;  // elements per 16-byte load
#pragma unroll
            for (int c = 0; c < H / PER16; ++c) {
                const uint4 dv = lds_v4(rowp + (uint32_t)c * 16u);
                const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
                float f[PER16];
#pragma unroll
                for (int c4 = 0; c4 < PER16 / 4; ++c4) {
                    const int chunk = (c * PER16) / 4 + c4;  // table chunk of entries 4 chunk .. 4 chunk + 3
                    const uint4 ch = lds_v4(tabp + (uint32_t)(chunk * p.nb) * 16u);
                    const uint32_t e[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t sg = (e[q] & 0x8000u) << 16;  // sign of D_k in bit 31
                        if constexpr (ES == 2) {
                            const uint32_t w = dw[(4 * c4 + q) >> 1];
                            const uint32_t bits = ((4 * c4 + q) & 1) ? (w & 0xffff0000u) : (w << 16);
                            f[4 * c4 + q] = __uint_as_float(bits ^ sg);
                        } else {
                            f[4 * c4 + q] = __uint_as_float(dw[q] ^ sg);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < PER16; q += 2) {
                    const int i2 = (c * PER16 + q) >> 1;
                    v2[i2] = make_float2(f[q], f[q + 1]);
                    acc = f2fma(v2[i2], v2[i2], acc);
                }
            }
        } else {
            const uint32_t rowp = stage_addr + (uint32_t)(slot * p.RW * p.srow + r * p.srow);
            const uint32_t tabp = gtab_addr + (uint32_t)b * 16u;
#pragma unroll
            for (int c4 = 0; c4 < H / 4; ++c4) {
                // entries 4 c4 .. 4 c4 + 3 of block b (chunk c4 * nb + b)
                const uint4 ch = lds_v4(tabp + (uint32_t)(c4 * p.nb) * 16u);
                const uint32_t e[4] = {ch.x, ch.y, ch.z, ch.w};
                float f[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    // entry: byte offset of x[pi(k)] (bf16 element) in bits 16-31, sign of D in bit 15
                    if constexpr (ES == 2) {
                        const uint32_t rv = lds_u16(rowp + (e[q] >> 16));
                        f[q] = __uint_as_float((rv + e[q]) << 16);  // bit 15 of e flips the sign; the rest shifts out
                    } else {
                        const uint32_t rv = lds_u32(rowp + ((e[q] >> 16) << 1));
                        f[q] = __uint_as_float(rv ^ (e[q] << 16));
                    }
                }
                v2[2 * c4] = make_float2(f[0], f[1]);
                v2[2 * c4 + 1] = make_float2(f[2], f[3]);
                acc = f2fma(v2[2 * c4], v2[2 * c4], acc);
                acc = f2fma(v2[2 * c4 + 1], v2[2 * c4 + 1], acc);
            }
        }
        // this warp is done with the slot
        __syncwarp();
        if (lane == 0) mbar_arrive(&my_empty[slot]);
        // loader: refill the slot with the team's row set k + slots once every
        // warp has gathered from it (now if they have, else later)
        const int gn = g + p.slots * stride;
        if (loader && gn < p.nrs) {
            if (mbar_test_wait(&my_empty[slot], ph)) {
                issue(slot, gn, k + p.slots);
            } else {
                pend_slot = slot;
                pend_ph = ph;
                pend_g = gn;
                pend_k = k + p.slots;
            }
        }

        // ---- A4 (first half): the row's sum of squares over this warp's blocks ----
        float ss = acc.x + acc.y;
        if (SPL == 2) ss += __shfl_xor_sync(0xffffffffu, ss, 1);  // the block's two halves
        for (int o = p.RW << LSPL; o < 32; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);  // the row's blocks
        float* part = my_part + (k & 1) * p.team * p.RW;
        if (p.team > 1) {
            if (j == 0 && hf == 0) part[wt * p.RW + r] = ss;
            __syncwarp();
            if (lane == 0) mbar_arrive(&my_norm[k & 1]);
        }

        // ---- A3: unnormalised Walsh-Hadamard butterflies, Sylvester order ------
#pragma unroll
        for (int i = 0; i < L2H; ++i) {
            const float a = v2[i].x, c = v2[i].y;
            v2[i] = make_float2(a + c, a - c);
        }
#pragma unroll
        for (int hl = 1; hl < L2H; hl <<= 1) {
#pragma unroll
            for (int i = 0; i < L2H; ++i) {
                if ((i & hl) == 0) {
                    const float2 a = v2[i], c = v2[i + hl];
                    v2[i] = f2add(a, c);
                    v2[i + hl] = f2sub(a, c);
                }
            }
        }

        // a deferred refill may be possible by now
        if (loader && pend_slot >= 0 && mbar_test_wait(&my_empty[pend_slot], pend_ph)) {
            issue(pend_slot, pend_g, pend_k);
            pend_slot = -1;
        }

        // ---- A4 (second half): the row norm s = ||x'||, summed in team order ----
        float ssum = ss;
        if (p.team > 1) {
            if (!warp_wait(&my_norm[k & 1], (uint32_t)((k >> 1) & 1), abort_flag)) {
                ok = false;
                break;
            }
            ssum = 0.f;
            const uint32_t pa = smem_u32(part) + (uint32_t)r * 4u;
            for (int w2 = 0; w2 < p.team; ++w2) ssum += lds_f32(pa + (uint32_t)(w2 * p.RW) * 4u);
        }
        const float s = __fsqrt_rn(ssum);

        if (valid) store_unit<HL, BITS, MODE>(p, v2, s, row, b * SPL + hf, lut_addr0);
    }

    // Leaving (normally or after an abort): copies this CTA issued must land
    // before its shared memory goes away.
    if (loader) {
        for (int sl = 0; sl < p.slots; ++sl)
            if (issued_k[sl] > consumed_k) {
                const int kk = issued_k[sl];
                mbar_wait_bounded(&my_full[sl], (uint32_t)((p.slots == 1 ? kk : (kk >> 1)) & 1));
            }
    }
    if (tid == 0 && !p.starve) mbar_wait_bounded(tab_bar, 0u);
}

template <typename InT, int H, int BITS, int MODE, int SPL, bool CONTIG>
cudaError_t launch_rpbh_spl(const RpbhParams& p, int grid, cudaStream_t stream) {
    auto k = rpbh_quant_kernel<InT, H, BITS, MODE, SPL, CONTIG>;
    const int smem = smem_layout(p).total;
    static int smem_done[kSmemRecordDevices] = {0};  // this instantiation's limit, per device
    const cudaError_t e = ensure_smem_limit(k, smem, smem_done);
    if (e != cudaSuccess) return e;
    const cudaError_t le = launch_pdl(k, dim3(grid), dim3(p.tpc * p.team * 32), smem, stream, p);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

// contiguous blocks (identity permutation): one lane per block; two lanes
// per block: bf16 inputs, blocks of 64 or 128
template <typename InT, int H, int BITS, int MODE>
cudaError_t launch_rpbh_t(const RpbhParams& p, int grid, cudaStream_t stream) {
    if (p.contig) return launch_rpbh_spl<InT, H, BITS, MODE, 1, true>(p, grid, stream);
    if constexpr (sizeof(InT) == 2 && H >= 64)
        if (p.SPL == 2) return launch_rpbh_spl<InT, H, BITS, MODE, 2, false>(p, grid, stream);
    return launch_rpbh_spl<InT, H, BITS, MODE, 1, false>(p, grid, stream);
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

// Layout choice.  More rows per warp spread the warp's random gather over
// more banks: consecutive rows of a slot start 128 / RW bytes apart modulo
// 128 (16 bytes at least, the bulk copies' alignment), so the RW rows' copies
// of one column sit in RW different groups of 32 / RW banks and only the
// warp's 32 / RW blocks can collide.  Larger RW costs larger slots and
// larger teams.  Among the layouts that fit, the one with the most warps is
// taken (they hide the gathers' latency), then the one with two slots per
// team (the next row set streams in during the whole computation of this
// one), then the one with the most rows per warp.  A forced layout (test
// and tuning hook) is taken when it fits.
static int g_force_rw = 0, g_force_slots = 0, g_force_spl = 0;

void rpbh_force_layout(int rows_per_warp, int slots, int lanes_per_block) {
    g_force_rw = rows_per_warp;
    g_force_slots = slots;
    g_force_spl = lanes_per_block;
}

bool rpbh_choose_layout(RpbhParams& p, int h, int esize) {
    const int nb = p.d / h;
    p.row_bytes = p.d * esize;
    RpbhParams best = p;
    int best_key = -1;
    // two lanes per block (more warps per SM, half the registers) only for
    // bf16 inputs and blocks of 64 or 128, and only when forced for now
    const int spl_max = (esize == 2 && h >= 64 && g_force_spl == 2 && !p.contig) ? 2 : 1;
    for (int spl = spl_max; spl >= 1; --spl) {
        const int max_warps = spl == 2 ? kMaxWarpsSplit : kMaxWarps;
        for (int slots = 2; slots >= 1; --slots) {
            for (int RW = 8; RW >= 1; RW >>= 1) {
                if (g_force_rw && RW != g_force_rw) continue;
                if (g_force_slots && slots != g_force_slots) continue;
                const int Bw = 32 / (RW * spl);
                if (Bw < 1) continue;
                const int team = (nb + Bw - 1) / Bw;
                if (team > max_warps) continue;
                RpbhParams c = p;
                c.SPL = spl;
                c.RW = RW;
                int lbw = 0, lrw = 0;
                while ((1 << lbw) < Bw) ++lbw;
                while ((1 << lrw) < RW) ++lrw;
                c.lbw = lbw;
                c.lrw = lrw;
                c.team = team;
                c.slots = slots;
                c.srow = c.row_bytes + (RW == 1 ? 16 : 128 / RW);
                for (c.tpc = max_warps / team; c.tpc >= 1; --c.tpc)
                    if (rpbh_smem_bytes(c) <= kSmemLimit) break;
                if (c.tpc < 1) continue;
                const int key = spl * 100000 + (c.tpc * team) * 100 + slots * 10 + RW;
                if (key > best_key) {
                    best_key = key;
                    best = c;
                }
            }
        }
    }
    if (best_key < 0) return false;
    p = best;
    return true;
}

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
