// Fused RPBH rotate -> norm/direction split -> Lloyd-Max quantise -> pack:
// the warp-group kernel, for permuted plans of moderate width.
//
// Method: "OrbitQuant" paper summary (hyper.ai, papers 2607.02461), section
// 方法 (Method): x' = Pi_d x with Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi,
// s = ||x'||_2, index = Q_b(x' / (s + eps)) under C_d.  It computes exactly
// what rpbh_quant.cu's team kernel computes (the same gather semantics, the
// same butterflies, the same quantiser epilogue: store_unit); only the work
// split and the synchronisation differ, and with them the order in which the
// row norm's partial sums are added.
//
// Design (sm_100a, HBM-bound):
//   - persistent CTAs, one per SM, each split into NG (1-4) warp groups of G
//     threads.  A group takes tiles of R rows (interleaved over the grid) and
//     runs out of phase with the CTA's other groups: its own two staging
//     buffers (one 1-D bulk copy per row, completing on the buffer's
//     mbarrier), its own named barrier, so one group's gathers overlap the
//     others' butterflies and lookups.  The next tile's rows stream into the
//     other buffer while this one is computed;
//   - thread (r, b) of a group owns row r's h-block b.  The gather table has
//     16-bit entries, pi(k) with the sign of D_k in bit 15, in 16-byte
//     chunks of 8 entries (chunk (c, b) at c*nb + b): one 16-byte table load
//     per 8 gathered inputs;
//   - the row norm is the norm of the gathered inputs (Pi_d is orthogonal):
//     a shuffle sum over the row's threads of a warp, then one partial per
//     warp and row through shared memory, read after the butterflies;
//   - the quantiser epilogue (bin lookup, codes or centroid values, 16-byte
//     stores) is store_unit, shared with the team kernel.
// The first table copy and every stage wait are bounded: a wait that runs
// out raises the device error flag, the group leaves its loop and drains
// the copy it has in flight (bounded) before the CTA exits.
#include <cuda_bf16.h>

#include "device_util.cuh"
#include "oq_internal.h"
#include "rpbh_quant.cuh"

namespace oq {

namespace {

struct GroupLayout {
    int gtab, lut, stage, red, bar, total;
};

// 16-bit gather table | lookup table | NG groups x 2 staging buffers of R
// rows | NG groups' norm partials (one per warp and row) | mbarriers (two per
// group, then the tables')
__host__ __device__ inline GroupLayout group_layout(const RpbhParams& p) {
    auto up = [](int x, int a) { return (x + a - 1) / a * a; };
    GroupLayout L;
    L.gtab = 0;
    L.lut = up(p.d * 2, 16);
    L.stage = up(L.lut + p.lut_n * 8, 128);
    L.red = L.stage + p.NG * 2 * p.R * p.srow;
    L.bar = up(L.red + p.NG * (p.G / 32) * p.R * 4, 8);
    L.total = L.bar + 8 * (2 * p.NG + 1);
    return L;
}

__device__ __forceinline__ void named_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

template <typename InT, int H, int BITS, int MODE>
__global__ void __launch_bounds__(kMaxThreads, 1) rpbh_groups_kernel(const __grid_constant__ RpbhParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const GroupLayout L = group_layout(p);
    __shared__ int s_abort[kMaxGroups];

    const int tid = threadIdx.x;
    const int G = p.G, R = p.R, NG = p.NG;
    const int grp = tid / G, tg = tid - grp * G;
    const int r = tg & (R - 1), b = tg / R;  // row of the tile, h-block
    const bool active = b < p.nb;
    const int lane = tg & 31, warp = tg >> 5, nwarps = G >> 5;
    constexpr int ES = sizeof(InT);
    uint8_t* stage = smem + L.stage + grp * 2 * R * p.srow;
    float* red = reinterpret_cast<float*>(smem + L.red) + grp * nwarps * R;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
    uint64_t* my_bar = bars + 2 * grp;
    uint64_t* tab_bar = bars + 2 * NG;

    // Launched with programmatic serialisation: every global access comes
    // after this wait (the set-up above may overlap the previous kernel).
    if (tid == 0) grid_launch_dependents();
    grid_dependency_wait();

    // copy tile `tile`'s rows into buffer `buf` of group `g`; returns whether
    // a copy was issued (a starved launch, a test hook, issues none, so the
    // waits run out)
    auto issue = [&](int g, int tile, int buf) -> bool {
        if (p.starve) return false;
        const int row0 = tile * R;
        const int rows = min(R, p.M - row0);
        uint64_t* bar = bars + 2 * g + buf;
        mbar_arrive_expect_tx(bar, (uint32_t)(rows * p.row_bytes));
        const uint8_t* src = static_cast<const uint8_t*>(p.x) + (size_t)row0 * p.row_bytes;
        uint8_t* dst = smem + L.stage + (g * 2 + buf) * R * p.srow;
        for (int i = 0; i < rows; ++i) bulk_g2s(dst + i * p.srow, src + (size_t)i * p.row_bytes, p.row_bytes, bar);
        return true;
    };

    // this group's tiles: blockIdx.x + (NG k + grp) gridDim.x, k = 0, 1, ...
    const int step = NG * gridDim.x;
    if (tid == 0) {
        for (int i = 0; i < 2 * NG + 1; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        for (int g = 0; g < kMaxGroups; ++g) s_abort[g] = 0;
        if (!p.starve) {
            const uint32_t lut_bytes = (uint32_t)(p.lut_n * 8);
            mbar_arrive_expect_tx(tab_bar, (uint32_t)(p.d * 2) + lut_bytes);
            bulk_g2s(smem + L.gtab, p.gtab16, (uint32_t)(p.d * 2), tab_bar);
            if (lut_bytes) bulk_g2s(smem + L.lut, p.lut, lut_bytes, tab_bar);
        }
        for (int g = 0; g < NG; ++g) {
            const int t0 = blockIdx.x + g * gridDim.x;
            if (t0 < p.ntiles) issue(g, t0, 0);
        }
    }
    __syncthreads();  // barriers initialised, first copies in flight

    const uint32_t lut_addr0 = smem_u32(smem) + (uint32_t)L.lut + (uint32_t)p.lut_off * 8u;
    const uint4* gtab = reinterpret_cast<const uint4*>(smem + L.gtab);
    constexpr int L2H = H / 2;
    bool tab_ok = true;

    int it = 0;  // (every CTA's group 0 has a tile: grid <= ntiles)
    for (int tile = blockIdx.x + grp * gridDim.x; tile < p.ntiles; tile += step, ++it) {
        const int buf = it & 1;
        const int next = tile + step;
        bool pending = false;  // group leader: a copy into the other buffer is in flight
        if (tg == 0 && next < p.ntiles) pending = issue(grp, next, buf ^ 1);
        if (tg == 0) {
            if (it == 0) tab_ok = mbar_wait_bounded(tab_bar, 0u);
            if (!tab_ok || !mbar_wait_bounded(&my_bar[buf], (uint32_t)((it >> 1) & 1))) s_abort[grp] = 1;
        }
        named_sync(1 + grp, G);
        if (s_abort[grp]) {
            // the copy into the other buffer must land before the CTA exits
            if (tg == 0 && pending) mbar_wait_bounded(&my_bar[buf ^ 1], (uint32_t)(((it + 1) >> 1) & 1));
            break;
        }

        const int row = tile * R + r;
        const bool valid = active && row < p.M;

        // ---- A1 + A2: gather sigma_k x[pi(k)] and the sum of squares -------
        float2 v2[L2H];
        float2 acc = make_float2(0.f, 0.f);
        if (valid) {
            const uint32_t rowp = smem_u32(stage) + (uint32_t)((buf * R + r) * p.srow);
#pragma unroll
            for (int c = 0; c < H / 8; ++c) {
                const uint4 ch = gtab[c * p.nb + b];  // entries 8c .. 8c+7 of block b
                const uint32_t w[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t e0 = w[e] & 0xffffu, e1 = w[e] >> 16;
                    float f0, f1;
                    if constexpr (ES == 2) {
                        uint32_t r0, r1;
                        asm volatile("ld.shared.u16 %0, [%1];" : "=r"(r0) : "r"(rowp + ((e0 & 0x7fffu) << 1)));
                        asm volatile("ld.shared.u16 %0, [%1];" : "=r"(r1) : "r"(rowp + ((e1 & 0x7fffu) << 1)));
                        // bf16 -> fp32, the sign flipped where the entry's bit 15 is set
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

        // ---- A4 (first half): the row's sum of squares over this warp's blocks ----
        float ss = acc.x + acc.y;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
            if (o >= R) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane < R) red[warp * R + lane] = ss;

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

        // ---- A4 (second half): the row norm, partials added in warp order ----
        named_sync(1 + grp, G);
        float ssum = 0.f;
        for (int w = 0; w < nwarps; ++w) ssum += red[w * R + r];
        const float s = __fsqrt_rn(ssum);

        if (valid) store_unit<H, BITS, MODE>(p, v2, s, row, b, lut_addr0);
        named_sync(1 + grp, G);  // this buffer and the partials are free for reuse
    }
}

template <typename InT, int H, int BITS, int MODE>
cudaError_t launch_groups_t(const RpbhParams& p, int grid, cudaStream_t stream) {
    auto k = rpbh_groups_kernel<InT, H, BITS, MODE>;
    const int smem = group_layout(p).total;
    static int smem_done[kSmemRecordDevices] = {0};  // this instantiation's limit, per device
    const cudaError_t e = ensure_smem_limit(k, smem, smem_done);
    if (e != cudaSuccess) return e;
    const cudaError_t le = launch_pdl(k, dim3(grid), dim3(p.NG * p.G), smem, stream, p);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

template <typename InT, int H, int MODE>
cudaError_t launch_groups_bits(const RpbhParams& p, int bits, int grid, cudaStream_t stream) {
    // the rotation alone and the value outputs do not depend on the code width
    if constexpr (MODE >= 2) {
        return launch_groups_t<InT, H, 4, MODE>(p, grid, stream);
    } else {
        switch (bits) {
            case 2: return launch_groups_t<InT, H, 2, MODE>(p, grid, stream);
            case 3:
                if constexpr (H >= 32) return launch_groups_t<InT, H, 3, MODE>(p, grid, stream);
                return cudaErrorInvalidValue;
            case 4: return launch_groups_t<InT, H, 4, MODE>(p, grid, stream);
            case 6: return launch_groups_t<InT, H, 6, MODE>(p, grid, stream);
            case 8: return launch_groups_t<InT, H, 8, MODE>(p, grid, stream);
        }
        return cudaErrorInvalidValue;
    }
}

template <typename InT, int MODE>
cudaError_t launch_groups_h(const RpbhParams& p, int h, int bits, int grid, cudaStream_t stream) {
    switch (h) {
        case 16: return launch_groups_bits<InT, 16, MODE>(p, bits, grid, stream);
        case 32: return launch_groups_bits<InT, 32, MODE>(p, bits, grid, stream);
        case 64: return launch_groups_bits<InT, 64, MODE>(p, bits, grid, stream);
        case 128: return launch_groups_bits<InT, 128, MODE>(p, bits, grid, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// Rows per tile: a power of two, at most 128 threads per group (R nb <= 128),
// four staging buffers (two groups x two stages) within ~180 KB.  Groups:
// as many (up to four) as the launch bound and shared memory hold.  The rows
// of a buffer are padded by 16 bytes so that consecutive rows start four
// banks apart.
bool rpbh_choose_groups(RpbhParams& p, int esize) {
    p.row_bytes = p.d * esize;
    p.srow = p.row_bytes + 16;
    int R = 1;
    while (R < 32 && 2 * R * p.nb <= 128 && 4 * (2 * R) * p.srow <= 180 * 1024) R *= 2;
    p.R = R;
    p.G = (p.nb * R + 31) / 32 * 32;
    if (p.G > 128) return false;
    for (p.NG = kMaxGroups; p.NG > 1; --p.NG)
        if (p.NG * p.G <= kMaxThreads && group_layout(p).total <= kSmemLimit - 64) break;
    if (group_layout(p).total > kSmemLimit - 64) return false;  // 64 B: the static abort flags
    p.ntiles = (p.M + R - 1) / R;
    return true;
}

cudaError_t launch_rpbh_groups(const RpbhParams& p, bool in_bf16, int h, int bits, int mode, int grid,
                               cudaStream_t stream) {
    if (in_bf16) {
        if (mode == 0) return launch_groups_h<__nv_bfloat16, 0>(p, h, bits, grid, stream);
        if (mode == 1) return launch_groups_h<__nv_bfloat16, 1>(p, h, bits, grid, stream);
        if (mode == 3) return launch_groups_h<__nv_bfloat16, 3>(p, h, bits, grid, stream);
        if (mode == 4) return launch_groups_h<__nv_bfloat16, 4>(p, h, bits, grid, stream);
        return launch_groups_h<__nv_bfloat16, 2>(p, h, 4, grid, stream);
    }
    if (mode == 0) return launch_groups_h<float, 0>(p, h, bits, grid, stream);
    if (mode == 1) return launch_groups_h<float, 1>(p, h, bits, grid, stream);
    if (mode == 3) return launch_groups_h<float, 3>(p, h, bits, grid, stream);
    if (mode == 4) return launch_groups_h<float, 4>(p, h, bits, grid, stream);
    return launch_groups_h<float, 2>(p, h, 4, grid, stream);
}

}  // namespace oq
