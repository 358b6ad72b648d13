// C ABI of liboq (declared in include/oq.h): argument checks, handle
// management, lazy per-device uploads and kernel dispatch.
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <new>

#include "device_util.cuh"
#include "oq_internal.h"
#include "qgemm.cuh"
#include "rpbh_quant.cuh"

namespace oq {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int device_sms() {
    static int count[kMaxDevices] = {0};
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    if (!count[dev]) cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
    return count[dev] > 0 ? count[dev] : 148;
}

// Test hooks (failure detection without a GPU fault): pending allocation
// failures and the kernels whose next launch issues no input copies.
static std::atomic<int> g_fail_allocs{0};
static std::atomic<int> g_starve_mask{0};

static bool device_alloc(void** ptr, size_t bytes) {
    int n = g_fail_allocs.load();
    while (n > 0 && !g_fail_allocs.compare_exchange_weak(n, n - 1)) {
    }
    if (n > 0) return false;
    return cudaMalloc(ptr, bytes) == cudaSuccess;
}

// true (once) if the next launch of `kernel` is to be starved
bool take_starve(int kernel) { return (g_starve_mask.fetch_and(~kernel) & kernel) != 0; }

bool quant_bits_ok(int bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 6 || bits == 8; }

int packed_row_bytes(int d, int bits) { return bits == 6 ? d : d * bits / 8; }  // 8: one byte per code too

// Launch the fused rotate/quantise kernel in one of its modes: 0 activation
// codes, 1 weight codes, 2 rotation only, 3 / 4 activation values (bf16 /
// e4m3 of c sqrt(d)) written to idx_out.
// Tuning hook: 0 chooses the kernel family per shape, 1 forces the
// warp-group kernel, 2 the team kernel (blocks of at most 128).
std::atomic<int> g_force_kernel{0};

oq_status run_rpbh(const oq_plan_t* plan, oq_codebook_t* cb, const void* x, oq_dtype dtype, int M, int mode,
                   uint8_t* idx_out, float* s_out, uint16_t* r_out, float* y_out, float* norm_out, cudaStream_t st) {
    if (!plan || M < 0) return OQ_ERR_INVALID_ARG;
    if (dtype != OQ_BF16 && dtype != OQ_F32) return OQ_ERR_INVALID_ARG;
    if (mode != 2 && (!cb || cb->d != plan->d)) return OQ_ERR_INVALID_ARG;
    if (mode != 2 && !quant_bits_ok(cb->bits)) return OQ_ERR_UNSUPPORTED;
    if (M == 0) return OQ_OK;  // an empty batch: buffers may be null
    if (!x) return OQ_ERR_INVALID_ARG;
    if (mode != 2) {
        if (!idx_out) return OQ_ERR_INVALID_ARG;
        if (cb->d != plan->d) return OQ_ERR_INVALID_ARG;
        if (!quant_bits_ok(cb->bits)) return OQ_ERR_UNSUPPORTED;
        if (mode < 2 && packed_row_bytes(plan->d, cb->bits) % 4 != 0) return OQ_ERR_UNSUPPORTED;
        if (mode < 2 && cb->bits == 3 && (plan->h < 32 || plan->d % 128 != 0))
            return OQ_ERR_UNSUPPORTED;  // 16-byte rows
        if (!aligned16(idx_out)) return OQ_ERR_ALIGNMENT;
    }
    if ((mode == 0 || mode >= 3) && (!s_out || !aligned16(s_out))) return s_out ? OQ_ERR_ALIGNMENT : OQ_ERR_INVALID_ARG;
    if (mode == 1 && (!r_out || !aligned16(r_out))) return r_out ? OQ_ERR_ALIGNMENT : OQ_ERR_INVALID_ARG;
    if (mode == 2 && (!y_out || !norm_out)) return OQ_ERR_INVALID_ARG;
    if (mode == 2 && (!aligned16(y_out) || !aligned16(norm_out))) return OQ_ERR_ALIGNMENT;
    if (!aligned16(x)) return OQ_ERR_ALIGNMENT;
    if (current_device() != plan->device) return OQ_ERR_INVALID_ARG;

    const DeviceCodebook* dcb = nullptr;
    if (mode != 2) {
        oq_status s = codebook_device(cb, &dcb);
        if (s != OQ_OK) return s;
    }
    const int d = plan->d, h = plan->h, nb = d / h;
    const int esize = dtype == OQ_BF16 ? 2 : 4;
    if (esize == 4 && d > 16384) return OQ_ERR_UNSUPPORTED;  // fp32 byte offsets of the gather table
    const bool big = h > 128;  // blocks beyond the in-register kernel (rht_big.cu)
    if (big && mode != 2 && cb->bits == 3) return OQ_ERR_UNSUPPORTED;
    RpbhParams p;
    std::memset(&p, 0, sizeof(p));
    p.x = x;
    p.M = M;
    p.d = d;
    p.nb = nb;
    p.lut_n = mode != 2 ? (int)cb->lut.size() : 0;
    p.contig = plan->variant == OQ_ROT_BLOCK_RHT ? 1 : 0;
    // Kernel family for blocks of at most 128: the warp-group kernel for
    // permuted plans up to d = 8192 (measured faster there), the team kernel
    // above that and for Block-RHT plans (its contiguous read path); the
    // tuning hook may force either.
    bool groups = false;
    if (big) {
        p.row_bytes = d * esize;
        if (rht_big_smem_bytes(p) > kSmemLimit) return OQ_ERR_UNSUPPORTED;
    } else {
        const int force = g_force_kernel.load();
        groups = force == 1 || (force == 0 && !p.contig && d <= 8192);
        if (groups && !rpbh_choose_groups(p, esize)) groups = false;
        if (!groups) {
            if (!rpbh_choose_layout(p, h, esize)) return OQ_ERR_UNSUPPORTED;
            p.nrs = (M + p.RW - 1) / p.RW;
        }
    }
    p.gtab = plan->dev.gtab;
    p.gtab16 = plan->dev.gtab16;
    if (mode != 2) {
        p.lut = mode == 3 ? dcb->lut_vb : (mode == 4 ? dcb->lut_v8 : dcb->lut);
        p.lut_off = -(int)kLutMagicBits - cb->kmin;
        p.G_lut = cb->G;
        p.L = cb->L;
        p.out_row_bytes = mode == 3 ? 2 * d : (mode == 4 ? d : packed_row_bytes(d, cb->bits));
        p.mid_val = mode == 3 ? cb->c_bf16[cb->L / 2] : (mode == 4 ? cb->c_e4m3[cb->L / 2] : 0u);
    }
    p.idx_out = idx_out;
    p.st32 = (reinterpret_cast<uintptr_t>(idx_out) % 32 == 0 && p.out_row_bytes % 32 == 0) ? 1 : 0;
    p.s_out = s_out;
    p.r_out = r_out;
    p.y_out = y_out;
    p.norm_out = norm_out;
    p.rsqrt_h = (float)(1.0 / std::sqrt((double)h));
    p.eps = (float)kEps;
    p.s_max = (float)(3.4028234663852886e38 / (2.0 * std::sqrt((double)h)));
    p.starve = take_starve(OQ_STARVE_RPBH) ? 1 : 0;  // consumed by a launch that happens
    cudaError_t e;
    if (big) {
        // one row per CTA at a time, as many CTAs per SM as shared memory holds (at most 8)
        int per_sm = kSmemLimit / rht_big_smem_bytes(p);
        per_sm = per_sm < 1 ? 1 : (per_sm > 8 ? 8 : per_sm);
        const int cap = per_sm * device_sms();
        e = launch_rht_big(p, dtype == OQ_BF16, h, mode == 2 ? 4 : cb->bits, mode, M < cap ? M : cap, st);
    } else if (groups) {
        const int grid = p.ntiles < device_sms() ? p.ntiles : device_sms();
        e = launch_rpbh_groups(p, dtype == OQ_BF16, h, mode == 2 ? 4 : cb->bits, mode, grid, st);
    } else {
        const int per_cta = (p.nrs + p.tpc - 1) / p.tpc;
        const int grid = per_cta < device_sms() ? per_cta : device_sms();
        e = launch_rpbh_quant(p, dtype == OQ_BF16, h, mode == 2 ? 4 : cb->bits, mode, grid, st);
    }
    return e == cudaSuccess ? OQ_OK : OQ_ERR_CUDA;
}

}  // namespace

oq_status codebook_device(oq_codebook_t* cb, const DeviceCodebook** out) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return OQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(cb->mu);
    DeviceCodebook& dc = cb->dev[dev];
    if (!dc.lut) {
        // three tables of the same bins: code counts, then the bf16 and the
        // e4m3 centroid values of the two cells each bin can give (the one
        // below its threshold in the low half, the one above in the high)
        const size_t n = cb->lut.size();
        std::vector<LutEntry> all(3 * n);
        for (size_t i = 0; i < n; ++i) {
            const LutEntry& e = cb->lut[i];
            const int lo = e.base, hi = e.base + 1 < cb->L ? e.base + 1 : e.base;
            all[i] = e;
            all[n + i] = {e.T, (int32_t)((uint32_t)cb->c_bf16[lo] | ((uint32_t)cb->c_bf16[hi] << 16))};
            all[2 * n + i] = {e.T, (int32_t)((uint32_t)cb->c_e4m3[lo] | ((uint32_t)cb->c_e4m3[hi] << 8))};
        }
        void* ptr = nullptr;
        const size_t bytes = all.size() * sizeof(LutEntry);
        if (!device_alloc(&ptr, bytes)) return OQ_ERR_OOM;
        if (cudaMemcpy(ptr, all.data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess) {
            cudaFree(ptr);
            return OQ_ERR_CUDA;
        }
        dc.lut = static_cast<LutEntry*>(ptr);
        dc.lut_vb = dc.lut + n;
        dc.lut_v8 = dc.lut + 2 * n;
    }
    *out = &dc;
    return OQ_OK;
}

}  // namespace oq

using namespace oq;

extern "C" {

const char* oq_status_str(oq_status s) {
    switch (s) {
        case OQ_OK: return "OQ_OK";
        case OQ_ERR_INVALID_ARG: return "OQ_ERR_INVALID_ARG";
        case OQ_ERR_UNSUPPORTED: return "OQ_ERR_UNSUPPORTED";
        case OQ_ERR_ALIGNMENT: return "OQ_ERR_ALIGNMENT";
        case OQ_ERR_CUDA: return "OQ_ERR_CUDA";
        case OQ_ERR_TIMEOUT: return "OQ_ERR_TIMEOUT";
        case OQ_ERR_OOM: return "OQ_ERR_OOM";
        case OQ_ERR_NO_CONVERGENCE: return "OQ_ERR_NO_CONVERGENCE";
        case OQ_ERR_TOO_LARGE: return "OQ_ERR_TOO_LARGE";
    }
    return "OQ_ERR_UNKNOWN";
}

oq_status oq_codebook(int d, int bits, oq_codebook_t** out) {
    if (!out) return OQ_ERR_INVALID_ARG;
    *out = nullptr;
    if (d < 3 || bits < 1 || bits > 8) return OQ_ERR_UNSUPPORTED;
    oq_codebook_t* cb = new (std::nothrow) oq_codebook_s();
    if (!cb) return OQ_ERR_OOM;
    oq_status s = build_codebook(d, bits, cb);
    if (s != OQ_OK) {
        delete cb;
        return s;
    }
    *out = cb;
    return OQ_OK;
}

oq_status oq_codebook_upload(const oq_codebook_t* cb) {
    if (!cb) return OQ_ERR_INVALID_ARG;
    const DeviceCodebook* dcb = nullptr;
    return codebook_device(const_cast<oq_codebook_t*>(cb), &dcb);
}

oq_status oq_codebook_values(const oq_codebook_t* cb, double* centroids, double* thresholds) {
    if (!cb) return OQ_ERR_INVALID_ARG;
    if (centroids) std::memcpy(centroids, cb->c.data(), sizeof(double) * cb->L);
    if (thresholds) std::memcpy(thresholds, cb->t.data(), sizeof(double) * (cb->L - 1));
    return OQ_OK;
}

oq_status oq_codebook_bf16(const oq_codebook_t* cb, uint16_t* centroids_bf16) {
    if (!cb || !centroids_bf16) return OQ_ERR_INVALID_ARG;
    std::memcpy(centroids_bf16, cb->c_bf16.data(), sizeof(uint16_t) * cb->L);
    return OQ_OK;
}

oq_status oq_codebook_shape(const oq_codebook_t* cb, int* d, int* bits) {
    if (!cb) return OQ_ERR_INVALID_ARG;
    if (d) *d = cb->d;
    if (bits) *bits = cb->bits;
    return OQ_OK;
}

void oq_codebook_free(oq_codebook_t* cb) {
    if (!cb) return;
    for (int i = 0; i < kMaxDevices; ++i)
        if (cb->dev[i].lut) cudaFree(cb->dev[i].lut);
    delete cb;
}

// Device plans: h a power of two in [16, 16384] dividing d (h <= 128: the
// in-register kernel; larger blocks, e.g. the ablation's Full RHT h = d: the
// staged kernel of rht_big.cu).
static oq_status check_plan_args(int d, int h) {
    if (d <= 0 || h <= 0) return OQ_ERR_INVALID_ARG;
    if ((h & (h - 1)) != 0 || h < 16 || h > 16384 || d % h != 0 || d > 32767 || d % 8 != 0) return OQ_ERR_UNSUPPORTED;
    return OQ_OK;
}

oq_status oq_rpbh_plan_host(int d, int h, uint64_t seed, int32_t* perm, int8_t* sign) {
    return oq_rotation_plan_host(d, h, seed, OQ_ROT_RPBH, perm, sign);
}

oq_status oq_rotation_plan_host(int d, int h, uint64_t seed, int variant, int32_t* perm, int8_t* sign) {
    // no device tables: any d in [1, 32767] and any block size h >= 1 dividing d
    if (d <= 0 || h <= 0) return OQ_ERR_INVALID_ARG;
    if (d > 32767 || d % h != 0) return OQ_ERR_UNSUPPORTED;
    if (variant != OQ_ROT_RPBH && variant != OQ_ROT_BLOCK_RHT) return OQ_ERR_INVALID_ARG;
    std::vector<int32_t> pv(d);
    std::vector<int8_t> sv(d);
    make_plan(d, h, seed, pv.data(), sv.data(), variant);
    if (perm) std::memcpy(perm, pv.data(), sizeof(int32_t) * d);
    if (sign) std::memcpy(sign, sv.data(), d);
    return OQ_OK;
}

oq_status oq_rpbh_plan(int d, int h, uint64_t seed, oq_plan_t** out) {
    return oq_rotation_plan(d, h, seed, OQ_ROT_RPBH, out);
}

oq_status oq_rotation_plan(int d, int h, uint64_t seed, int variant, oq_plan_t** out) {
    if (!out) return OQ_ERR_INVALID_ARG;
    *out = nullptr;
    oq_status s = check_plan_args(d, h);
    if (s != OQ_OK) return s;
    if (variant != OQ_ROT_RPBH && variant != OQ_ROT_BLOCK_RHT) return OQ_ERR_INVALID_ARG;
    const int dev = current_device();
    if (dev < 0) return OQ_ERR_CUDA;
    oq_plan_t* p = new (std::nothrow) oq_plan_s();
    if (!p) return OQ_ERR_OOM;
    p->d = d;
    p->h = h;
    p->seed = seed;
    p->device = dev;
    p->variant = variant;
    p->perm.resize(d);
    p->sign.resize(d);
    make_plan(d, h, seed, p->perm.data(), p->sign.data(), variant);
    build_gather_table(p, p->gtab_host);
    build_gather_table16(p, p->gtab16_host);
    // one allocation: the 32-bit table, then the 16-bit one (16-byte aligned: 4 d bytes in)
    void* ptr = nullptr;
    const size_t b32 = sizeof(uint32_t) * d, b16 = sizeof(uint16_t) * d;
    if (!device_alloc(&ptr, b32 + b16)) {
        delete p;
        return OQ_ERR_OOM;
    }
    uint8_t* base = static_cast<uint8_t*>(ptr);
    if (cudaMemcpy(base, p->gtab_host.data(), b32, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(base + b32, p->gtab16_host.data(), b16, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(ptr);
        delete p;
        return OQ_ERR_CUDA;
    }
    p->dev.gtab = reinterpret_cast<uint32_t*>(base);
    p->dev.gtab16 = reinterpret_cast<uint16_t*>(base + b32);
    *out = p;
    return OQ_OK;
}

oq_status oq_rpbh_plan_export(const oq_plan_t* plan, int32_t* perm, int8_t* sign) {
    if (!plan) return OQ_ERR_INVALID_ARG;
    if (perm) std::memcpy(perm, plan->perm.data(), sizeof(int32_t) * plan->d);
    if (sign) std::memcpy(sign, plan->sign.data(), plan->d);
    return OQ_OK;
}

oq_status oq_plan_shape(const oq_plan_t* plan, int* d, int* h) {
    if (!plan) return OQ_ERR_INVALID_ARG;
    if (d) *d = plan->d;
    if (h) *h = plan->h;
    return OQ_OK;
}

void oq_plan_free(oq_plan_t* plan) {
    if (!plan) return;
    if (plan->dev.gtab) cudaFree(plan->dev.gtab);
    delete plan;
}

oq_status oq_quantize_weights(const oq_plan_t* plan, const oq_codebook_t* cb_w, const void* W, oq_dtype dtype, int N,
                              uint8_t* idx_out, uint16_t* r_out, void* stream) {
    if (N <= 0) return OQ_ERR_INVALID_ARG;
    return run_rpbh(plan, const_cast<oq_codebook_t*>(cb_w), W, dtype, N, 1, idx_out, nullptr, r_out, nullptr, nullptr,
                    static_cast<cudaStream_t>(stream));
}

oq_status oq_quantize_acts(const oq_plan_t* plan, const oq_codebook_t* cb_a, const void* x, oq_dtype dtype, int M,
                           uint8_t* idx_out, float* s_out, void* stream) {
    return run_rpbh(plan, const_cast<oq_codebook_t*>(cb_a), x, dtype, M, 0, idx_out, s_out, nullptr, nullptr, nullptr,
                    static_cast<cudaStream_t>(stream));
}

oq_status oq_quantize_acts_values(const oq_plan_t* plan, const oq_codebook_t* cb_a, const void* x, oq_dtype dtype,
                                  int M, uint16_t* val_out, float* s_out, void* stream) {
    return run_rpbh(plan, const_cast<oq_codebook_t*>(cb_a), x, dtype, M, 3, reinterpret_cast<uint8_t*>(val_out), s_out,
                    nullptr, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

oq_status oq_quantize_acts_values_fp8(const oq_plan_t* plan, const oq_codebook_t* cb_a, const void* x, oq_dtype dtype,
                                      int M, uint8_t* val_out, float* s_out, void* stream) {
    if (cb_a && cb_a->d % 128 != 0) return OQ_ERR_UNSUPPORTED;  // the fp8 product's K step
    return run_rpbh(plan, const_cast<oq_codebook_t*>(cb_a), x, dtype, M, 4, val_out, s_out, nullptr, nullptr, nullptr,
                    static_cast<cudaStream_t>(stream));
}

oq_status oq_rpbh_apply(const oq_plan_t* plan, const void* x, oq_dtype dtype, int M, float* x_rot, float* norm_out,
                        void* stream) {
    return run_rpbh(plan, nullptr, x, dtype, M, 2, nullptr, nullptr, nullptr, x_rot, norm_out,
                    static_cast<cudaStream_t>(stream));
}

// Whether the products support these code widths: the codes product
// decodes both operands (2, 4 or 6 bits, or a pair of 3- and 4-bit codes),
// the values product decodes W only (2, 3, 4 or 6 bits).  8-bit codes have no
// in-kernel decoder (8-bit activations take the values schedule).  K steps
// take d % 64 == 0 (bf16) or d % 128 == 0 (e4m3); 3-bit rows need
// d % 128 == 0 (rows of whole 16-byte groups).
static bool codes_product_ok(int ba, int bw, int d, bool fp8) {
    if (d % (fp8 ? 128 : 64) != 0) return false;
    if ((ba == 3 || bw == 3) && d % 128 != 0) return false;
    auto ok246 = [](int b) { return b == 2 || b == 4 || b == 6; };
    if (ok246(ba) && ok246(bw)) return true;
    return (ba == 3 || ba == 4) && (bw == 3 || bw == 4);
}

static bool values_product_ok(int bw, int d, bool fp8) {
    if (d % (fp8 ? 128 : 64) != 0) return false;
    if (bw == 3) return d % 128 == 0;
    return bw == 2 || bw == 4 || bw == 6;
}

static oq_status run_qgemm(const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, int M, int N, const uint8_t* a_idx,
                           const float* s, const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias,
                           uint16_t* y, void* stream, bool fp8) {
    if (!cb_a || !cb_w || M < 0 || N <= 0) return OQ_ERR_INVALID_ARG;
    if (cb_a->d != cb_w->d) return OQ_ERR_INVALID_ARG;
    if (!codes_product_ok(cb_a->bits, cb_w->bits, cb_a->d, fp8)) return OQ_ERR_UNSUPPORTED;
    if (M == 0) return OQ_OK;  // an empty batch: activation and output buffers may be null
    if (!a_idx || !s || !w_idx || !w_r || !y) return OQ_ERR_INVALID_ARG;
    if (!aligned16(a_idx) || !aligned16(s) || !aligned16(w_idx) || !aligned16(w_r) || !aligned16(y) ||
        (bias && !aligned16(bias)))
        return OQ_ERR_ALIGNMENT;
    QgemmArgs a;
    a.M = M;
    a.N = N;
    a.K = cb_a->d;
    a.bits_a = cb_a->bits;
    a.bits_w = cb_w->bits;
    a.a_idx = a_idx;
    a.w_idx = w_idx;
    a.s = s;
    a.w_r = w_r;
    a.bias = bias;
    a.y = y;
    a.ca_bf16 = cb_a->c_bf16.data();
    a.cw_bf16 = cb_w->c_bf16.data();
    a.fp8 = fp8;
    a.ca_e4m3 = cb_a->c_e4m3.data();
    a.cw_e4m3 = cb_w->c_e4m3.data();
    a.starve = take_starve(OQ_STARVE_GEMM);
    cudaError_t e = launch_qgemm(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? OQ_OK : OQ_ERR_CUDA;
}

// The product with A given as centroid values (bf16, or e4m3 of c sqrt(d)).
static oq_status run_qgemm_values(const oq_codebook_t* cb_w, int M, int N, const void* a_val, const float* s,
                                  const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y,
                                  void* stream, bool fp8) {
    if (!cb_w || M < 0 || N <= 0) return OQ_ERR_INVALID_ARG;
    if (!values_product_ok(cb_w->bits, cb_w->d, fp8)) return OQ_ERR_UNSUPPORTED;
    if (M == 0) return OQ_OK;
    if (!a_val || !s || !w_idx || !w_r || !y) return OQ_ERR_INVALID_ARG;
    if (!aligned16(a_val) || !aligned16(s) || !aligned16(w_idx) || !aligned16(w_r) || !aligned16(y) ||
        (bias && !aligned16(bias)))
        return OQ_ERR_ALIGNMENT;
    QgemmArgs a;
    a.M = M;
    a.N = N;
    a.K = cb_w->d;
    a.bits_a = 0;
    a.bits_w = cb_w->bits;
    a.a_idx = nullptr;
    a.a_val = a_val;
    a.w_idx = w_idx;
    a.s = s;
    a.w_r = w_r;
    a.bias = bias;
    a.y = y;
    a.ca_bf16 = nullptr;
    a.cw_bf16 = cb_w->c_bf16.data();
    a.fp8 = fp8;
    a.ca_e4m3 = nullptr;
    a.cw_e4m3 = cb_w->c_e4m3.data();
    a.starve = take_starve(OQ_STARVE_GEMM);
    cudaError_t e = launch_qgemm(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? OQ_OK : OQ_ERR_CUDA;
}

oq_status oq_qgemm_values(const oq_codebook_t* cb_w, int M, int N, const uint16_t* a_val, const float* s,
                          const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y, void* stream) {
    return run_qgemm_values(cb_w, M, N, a_val, s, w_idx, w_r, bias, y, stream, false);
}

oq_status oq_qgemm_values_fp8(const oq_codebook_t* cb_w, int M, int N, const uint8_t* a_val, const float* s,
                              const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y,
                              void* stream) {
    return run_qgemm_values(cb_w, M, N, a_val, s, w_idx, w_r, bias, y, stream, true);
}

oq_status oq_qgemm(const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, int M, int N, const uint8_t* a_idx,
                   const float* s, const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y,
                   void* stream) {
    return run_qgemm(cb_a, cb_w, M, N, a_idx, s, w_idx, w_r, bias, y, stream, false);
}

oq_status oq_qgemm_fp8(const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, int M, int N, const uint8_t* a_idx,
                       const float* s, const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y,
                       void* stream) {
    return run_qgemm(cb_a, cb_w, M, N, a_idx, s, w_idx, w_r, bias, y, stream, true);
}

oq_status oq_codebook_fp8(const oq_codebook_t* cb, uint8_t* out) {
    if (!cb || !out) return OQ_ERR_INVALID_ARG;
    std::memcpy(out, cb->c_e4m3.data(), cb->c_e4m3.size());
    return OQ_OK;
}

size_t oq_qlinear_workspace(int M, int d, int bits_a) {
    if (M <= 0 || d <= 0 || !quant_bits_ok(bits_a)) return 0;
    const size_t idx = (size_t)M * (size_t)packed_row_bytes(d, bits_a);
    const size_t idx_al = (idx + 255) / 256 * 256;
    return idx_al + ((size_t)M * sizeof(float) + 255) / 256 * 256;
}

size_t oq_qlinear_workspace_values(int M, int d) {
    if (M <= 0 || d <= 0) return 0;
    return ((size_t)M * (size_t)d * 2 + 255) / 256 * 256 + ((size_t)M * sizeof(float) + 255) / 256 * 256;
}

static size_t values_workspace(int M, int d, bool fp8) {
    return ((size_t)M * (size_t)d * (fp8 ? 1 : 2) + 255) / 256 * 256 + ((size_t)M * sizeof(float) + 255) / 256 * 256;
}

// The layer's schedule for a workspace of ws_bytes, decided before any
// launch: values when the values product supports the widths and the
// workspace holds the values; else codes when the workspace holds the codes
// (OQ_ERR_UNSUPPORTED if the codes product does not support the widths);
// else OQ_ERR_OOM, or OQ_ERR_UNSUPPORTED if neither product supports them.
// *fits_larger tells whether a supported schedule would run with a larger
// workspace.
static oq_status choose_schedule(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, int M,
                                 size_t ws_bytes, bool fp8, bool* values, bool* fits_larger) {
    const int d = plan->d;
    const bool v_ok = values_product_ok(cb_w->bits, d, fp8);
    const bool c_ok = codes_product_ok(cb_a->bits, cb_w->bits, d, fp8);
    *fits_larger = v_ok || c_ok;
    if (v_ok && ws_bytes >= values_workspace(M, d, fp8)) {
        *values = true;
        return OQ_OK;
    }
    if (ws_bytes >= oq_qlinear_workspace(M, d, cb_a->bits)) {
        *values = false;
        return c_ok ? OQ_OK : OQ_ERR_UNSUPPORTED;
    }
    return *fits_larger ? OQ_ERR_OOM : OQ_ERR_UNSUPPORTED;
}

static oq_status run_qlinear(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w,
                             const void* x, oq_dtype dtype, int M, const uint8_t* w_idx, const uint16_t* w_r, int N,
                             const uint16_t* bias, uint16_t* y, void* workspace, size_t ws_bytes, void* stream,
                             bool fp8) {
    if (!plan || !cb_a || !cb_w) return OQ_ERR_INVALID_ARG;
    if (M < 0 || N <= 0) return OQ_ERR_INVALID_ARG;
    if (cb_a->d != plan->d || cb_w->d != plan->d) return OQ_ERR_INVALID_ARG;
    if (!quant_bits_ok(cb_a->bits) || !quant_bits_ok(cb_w->bits)) return OQ_ERR_UNSUPPORTED;
    if (M == 0) return OQ_OK;
    if (!workspace) return OQ_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return OQ_ERR_ALIGNMENT;
    // The values schedule (the quantiser writes c_index itself; the product
    // loads A's values by TMA and decodes only W) trades A's in-kernel decode
    // for four (bf16) or two (e4m3) times the bytes of A to stream per tile;
    // with a deep A ring and N-fastest tiles it is the faster one on B200 at
    // every shape measured, so it is taken whenever the workspace holds it.
    bool values = false, fits_larger = false;
    oq_status st = choose_schedule(plan, cb_a, cb_w, M, ws_bytes, fp8, &values, &fits_larger);
    if (st != OQ_OK) return st;
    if (values) {
        const size_t val_al = ((size_t)M * plan->d * (fp8 ? 1 : 2) + 255) / 256 * 256;
        float* s = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + val_al);
        st = fp8 ? oq_quantize_acts_values_fp8(plan, cb_a, x, dtype, M, static_cast<uint8_t*>(workspace), s, stream)
                 : oq_quantize_acts_values(plan, cb_a, x, dtype, M, static_cast<uint16_t*>(workspace), s, stream);
        if (st != OQ_OK) return st;
        return run_qgemm_values(cb_w, M, N, workspace, s, w_idx, w_r, bias, y, stream, fp8);
    }
    uint8_t* a_idx = static_cast<uint8_t*>(workspace);
    const size_t idx_al = ((size_t)M * packed_row_bytes(plan->d, cb_a->bits) + 255) / 256 * 256;
    float* s = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + idx_al);
    st = oq_quantize_acts(plan, cb_a, x, dtype, M, a_idx, s, stream);
    if (st != OQ_OK) return st;
    return run_qgemm(cb_a, cb_w, M, N, a_idx, s, w_idx, w_r, bias, y, stream, fp8);
}

oq_status oq_qlinear(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, const void* x,
                     oq_dtype dtype, int M, const uint8_t* w_idx, const uint16_t* w_r, int N, const uint16_t* bias,
                     uint16_t* y, void* workspace, size_t ws_bytes, void* stream) {
    return run_qlinear(plan, cb_a, cb_w, x, dtype, M, w_idx, w_r, N, bias, y, workspace, ws_bytes, stream, false);
}

oq_status oq_qlinear_fp8(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, const void* x,
                         oq_dtype dtype, int M, const uint8_t* w_idx, const uint16_t* w_r, int N,
                         const uint16_t* bias, uint16_t* y, void* workspace, size_t ws_bytes, void* stream) {
    return run_qlinear(plan, cb_a, cb_w, x, dtype, M, w_idx, w_r, N, bias, y, workspace, ws_bytes, stream, true);
}

// ---------------------------------------------------------------------------
// oq_qlinear without device allocation (no counterpart in the paper).
// Scratch for the packed activation codes and norms lives in this fixed,
// file-scope device array; its device address is looked up once per device.
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_noalloc_scratch[OQ_NOALLOC_SCRATCH_BYTES];

static oq_status noalloc_scratch_ptr(void** out) {
    static std::mutex mu;
    static void* ptrs[kMaxDevices] = {nullptr};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return OQ_ERR_CUDA;
        ptrs[dev] = p;
    }
    *out = ptrs[dev];
    return OQ_OK;
}

static bool codebook_resident(oq_codebook_t* cb) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(cb->mu);
    return cb->dev[dev].lut != nullptr;
}

oq_status oq_qlinear_noalloc(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w,
                             const void* x, oq_dtype dtype, int M, const uint8_t* w_idx, const uint16_t* w_r, int N,
                             const uint16_t* bias, uint16_t* y, void* stream) {
    if (!plan || !cb_a || !cb_w) return OQ_ERR_INVALID_ARG;
    if (M < 0 || N <= 0) return OQ_ERR_INVALID_ARG;
    if (cb_a->d != plan->d || cb_w->d != plan->d) return OQ_ERR_INVALID_ARG;
    if (!quant_bits_ok(cb_a->bits) || !quant_bits_ok(cb_w->bits)) return OQ_ERR_UNSUPPORTED;
    if (M == 0) return OQ_OK;
    // the schedule the scratch allows, decided before any work: values when
    // they fit, else codes; a supported request that fits neither is too large
    bool values = false, fits_larger = false;
    const oq_status sched = choose_schedule(plan, cb_a, cb_w, M, OQ_NOALLOC_SCRATCH_BYTES, false, &values, &fits_larger);
    if (sched != OQ_OK) return fits_larger ? OQ_ERR_TOO_LARGE : sched;
    if (current_device() != plan->device) return OQ_ERR_INVALID_ARG;
    // the activation codebook's tables must already be here (its upload would allocate)
    if (!codebook_resident(const_cast<oq_codebook_t*>(cb_a))) return OQ_ERR_INVALID_ARG;
    void* scratch = nullptr;
    oq_status st = noalloc_scratch_ptr(&scratch);
    if (st != OQ_OK) return st;
    return oq_qlinear(plan, cb_a, cb_w, x, dtype, M, w_idx, w_r, N, bias, y, scratch, OQ_NOALLOC_SCRATCH_BYTES,
                      stream);
}

void oq_debug_fail_allocations(int n) { g_fail_allocs.store(n > 0 ? n : 0); }

void oq_debug_starve(int mask) { g_starve_mask.store(mask & (OQ_STARVE_RPBH | OQ_STARVE_GEMM)); }

void oq_debug_qgemm_tile_rows(int rows) { qgemm_force_tile_rows(rows); }

void oq_debug_rpbh_kernel(int which) { g_force_kernel.store(which == 1 || which == 2 ? which : 0); }

void oq_debug_rpbh_layout(int rows_per_warp, int slots, int lanes_per_block) {
    const bool rw_ok = rows_per_warp == 0 || rows_per_warp == 1 || rows_per_warp == 2 || rows_per_warp == 4 ||
                       rows_per_warp == 8;
    rpbh_force_layout(rw_ok ? rows_per_warp : 0, (slots == 1 || slots == 2) ? slots : 0,
                      lanes_per_block == 2 ? 2 : 0);
}

oq_status oq_device_status(int clear, int* out, void* stream) {
    if (!out) return OQ_ERR_INVALID_ARG;
    int v = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyFromSymbolAsync(&v, g_error_flag, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return OQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return OQ_ERR_CUDA;
    if (clear) {
        const int zero = 0;
        if (cudaMemcpyToSymbolAsync(g_error_flag, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
            return OQ_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return OQ_ERR_CUDA;
    }
    *out = v ? OQ_ERR_TIMEOUT : OQ_OK;
    return OQ_OK;
}

}  // extern "C"
