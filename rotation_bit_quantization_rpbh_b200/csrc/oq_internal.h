// Internal declarations shared by the host side and the CUDA side of liboq.
#pragma once

#include <cstddef>
#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/oq.h"

namespace oq {

constexpr int kMaxDevices = 64;
constexpr double kEps = 1e-12;        // the split's epsilon, weights and activations
constexpr float kLutMagic = 12582912.0f;       // 1.5 * 2^23: fmaf(v, G, magic) holds rint(v*G) in its low bits
constexpr uint32_t kLutMagicBits = 0x4B400000u;

// One entry of the quantiser lookup table: for values v whose bin is this
// entry, index = base + (v >= T) (T = +inf when no threshold is in the bin).
struct LutEntry {
    float T;
    int32_t base;
};

struct DeviceCodebook {
    LutEntry* lut = nullptr;     // device copy of the lookup table
    LutEntry* lut_vb = nullptr;  // the same bins with bf16 centroid values (see codebook_device)
    LutEntry* lut_v8 = nullptr;  // the same bins with e4m3 values of c sqrt(d)
};

struct DevicePlan {
    uint32_t* gtab = nullptr;    // device gather table (see build_gather_table)
    uint16_t* gtab16 = nullptr;  // the 16-bit one (see build_gather_table16), same allocation
};

}  // namespace oq

struct oq_codebook_s {
    int d = 0, bits = 0, L = 0;
    std::vector<double> c;         // L centroids, ascending (fp64)
    std::vector<double> t;         // L-1 thresholds
    std::vector<float> t32;        // fp32 thresholds (the kernels' decision values)
    std::vector<uint16_t> c_bf16;  // bf16 centroids as the product uses them
    std::vector<uint8_t> c_e4m3;   // e4m3 bytes of c_j sqrt(d) (the fp8 product variant)
    // quantiser lookup table over v in [-vmax, vmax]:
    //   bin(v) = rint(v * G) (computed as fmaf(v, G, 1.5*2^23) in fp32)
    //   entry index = bin(v) - kmin
    float G = 0.f;
    int kmin = 0;
    std::vector<oq::LutEntry> lut;
    // per-device uploads (lazily on first use on a device)
    std::mutex mu;
    oq::DeviceCodebook dev[oq::kMaxDevices];
};

struct oq_plan_s {
    int d = 0, h = 0;
    uint64_t seed = 0;
    int device = -1;
    int variant = 0;  // OQ_ROT_RPBH or OQ_ROT_BLOCK_RHT (identity permutation)
    std::vector<int32_t> perm;
    std::vector<int8_t> sign;
    std::vector<uint32_t> gtab_host;    // chunked gather table (see build_gather_table)
    std::vector<uint16_t> gtab16_host;  // 16-bit entries (see build_gather_table16)
    oq::DevicePlan dev;
};

namespace oq {

// host-side pieces (host.cpp)
oq_status build_codebook(int d, int bits, oq_codebook_t* cb);
void make_plan(int d, int h, uint64_t seed, int32_t* perm, int8_t* sign, int variant);
uint8_t e4m3_round(double v);
void build_gather_table(const oq_plan_t* p, std::vector<uint32_t>& out);
void build_gather_table16(const oq_plan_t* p, std::vector<uint16_t>& out);
uint16_t bf16_round(double x);

// device-side pieces (api.cu)
oq_status codebook_device(oq_codebook_t* cb, const DeviceCodebook** out);

}  // namespace oq
