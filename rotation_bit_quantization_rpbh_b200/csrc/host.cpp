// Host-side pieces of liboq: the Lloyd-Max codebook C_d, the RPBH plan, the
// quantiser lookup table and bf16 rounding.  No GPU needed.
//
// Method: "OrbitQuant" paper summary (hyper.ai, papers 2607.02461), section
// 方法 (Method): C_d is the Lloyd-Max quantiser of the fixed marginal f_d of a
// rotated unit coordinate; Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi with
// a uniformly random permutation and Rademacher signs.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>

#include "oq_internal.h"

namespace oq {
namespace {

// ---------------------------------------------------------------------------
// log(Gamma(z + 1/2) / Gamma(z)).  For large z the difference of two lgamma
// values near z log z loses digits, so use the asymptotic expansion
//   a log z + sum_k (-1)^(k+1) [B_{k+1}(a) - B_{k+1}(0)] / (k (k+1) z^k),
// a = 1/2 (DLMF 5.11.13 with Bernoulli polynomials at 1/2):
//   1/2 log z - 1/(8z) + 1/(192 z^3) - 1/(640 z^5) + 17/(14336 z^7) ...
// ---------------------------------------------------------------------------
double log_gamma_ratio_half(double z) {
    if (z < 20.0) return std::lgamma(z + 0.5) - std::lgamma(z);
    const double iz = 1.0 / z, iz2 = iz * iz;
    return 0.5 * std::log(z) + iz * (-1.0 / 8.0 + iz2 * (1.0 / 192.0 + iz2 * (-1.0 / 640.0 + iz2 * (17.0 / 14336.0))));
}

// Continued fraction of the regularised incomplete beta function, evaluated
// by the modified Lentz method (Lentz 1976; Thompson & Barnett 1986).
double beta_cf(double a, double b, double x) {
    const double tiny = 1e-300;
    double c = 1.0;
    double dd = 1.0 - (a + b) * x / (a + 1.0);
    if (std::fabs(dd) < tiny) dd = tiny;
    dd = 1.0 / dd;
    double f = dd;
    for (int m = 1; m <= 20000; ++m) {
        const double m2 = 2.0 * m;
        // even step
        double num = m * (b - m) * x / ((a - 1.0 + m2) * (a + m2));
        dd = 1.0 + num * dd;
        if (std::fabs(dd) < tiny) dd = tiny;
        c = 1.0 + num / c;
        if (std::fabs(c) < tiny) c = tiny;
        dd = 1.0 / dd;
        f *= dd * c;
        // odd step
        num = -(a + m) * (a + b + m) * x / ((a + m2) * (a + 1.0 + m2));
        dd = 1.0 + num * dd;
        if (std::fabs(dd) < tiny) dd = tiny;
        c = 1.0 + num / c;
        if (std::fabs(c) < tiny) c = tiny;
        dd = 1.0 / dd;
        const double step = dd * c;
        f *= step;
        if (std::fabs(step - 1.0) < 1e-16) break;
    }
    return f;
}

// The marginal f_d(t) = c_d (1 - t^2)^((d-3)/2) on [-1, 1]:
//   c_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) = 1 / B(1/2, (d-1)/2),
//   P(|T| < x) = I_{x^2}(1/2, (d-1)/2).
struct Marginal {
    int d;
    double beta;   // (d-1)/2
    double log_c;  // log c_d

    explicit Marginal(int d_) : d(d_), beta(0.5 * (d_ - 1)) {
        log_c = log_gamma_ratio_half(beta) - 0.5 * std::log(M_PI);
    }

    double density(double x) const {
        if (std::fabs(x) >= 1.0) return 0.0;
        return std::exp(log_c + 0.5 * (d - 3) * std::log1p(-x * x));
    }

    // P(T > x) for 0 <= x <= 1
    double tail(double x) const {
        if (x <= 0.0) return 0.5;
        if (x >= 1.0) return 0.0;
        const double x2 = x * x, a = 0.5, b = beta;
        const double front = std::exp(log_c + a * std::log(x2) + b * std::log1p(-x2));
        if (x2 < (a + 1.0) / (a + b + 2.0)) {
            const double I = front * beta_cf(a, b, x2) / a;  // I_{x^2}(1/2, beta)
            return 0.5 * (1.0 - I);
        }
        const double Ic = front * beta_cf(b, a, 1.0 - x2) / b;  // 1 - I_{x^2}(1/2, beta)
        return 0.5 * Ic;
    }

    double mass(double lo, double hi) const { return tail(lo) - tail(hi); }  // 0 <= lo <= hi <= 1

    // closed form: int_lo^hi t f_d = c_d [(1-lo^2)^((d-1)/2) - (1-hi^2)^((d-1)/2)] / (d-1)
    double first(double lo, double hi) const {
        auto g = [&](double t) {
            if (t >= 1.0) return 0.0;
            return std::exp(log_c + 0.5 * (d - 1) * std::log1p(-t * t));
        };
        return (g(lo) - g(hi)) / (d - 1);
    }
};

// Solve the positive half of the symmetric Lloyd-Max quantiser with n
// positive levels q_1 < ... < q_n: cell i is [p_{i-1}, p_i] with p_0 = 0,
// p_n = 1, p_i = (q_i + q_{i+1}) / 2, and each q_i must equal the centroid of
// its cell.  A few Lloyd sweeps give a start; Newton's method on the
// residual R_i = q_i - centroid_i (a tridiagonal Jacobian) finishes it.
bool solve_positive_half(const Marginal& f, int n, std::vector<double>& q) {
    const double sigma = 1.0 / std::sqrt((double)f.d);
    q.resize(n);
    for (int i = 0; i < n; ++i) q[i] = sigma * 3.0 * (i + 0.5) / n;
    std::vector<double> p(n + 1), m(n), F0(n), R(n), lo(n), di(n), up(n), rhs(n);
    auto eval = [&](const std::vector<double>& qq) {
        p[0] = 0.0;
        p[n] = 1.0;
        for (int i = 1; i < n; ++i) p[i] = 0.5 * (qq[i - 1] + qq[i]);
        double worst = 0.0;
        for (int i = 0; i < n; ++i) {
            F0[i] = f.mass(p[i], p[i + 1]);
            m[i] = f.first(p[i], p[i + 1]) / F0[i];
            R[i] = qq[i] - m[i];
            worst = std::max(worst, std::fabs(R[i]));
        }
        return worst;
    };
    for (int it = 0; it < 60; ++it) {  // Lloyd sweeps
        eval(q);
        for (int i = 0; i < n; ++i) q[i] = m[i];
    }
    double res = eval(q);
    for (int it = 0; it < 200 && res > 1e-17 * sigma; ++it) {
        // Jacobian of R
        for (int i = 0; i < n; ++i) {
            const double dlo = (i > 0) ? f.density(p[i]) * (m[i] - p[i]) / F0[i] : 0.0;          // d m_i / d p_{i-1}
            const double dhi = (i < n - 1) ? f.density(p[i + 1]) * (p[i + 1] - m[i]) / F0[i] : 0.0;  // d m_i / d p_i
            di[i] = 1.0 - 0.5 * dlo - 0.5 * dhi;
            lo[i] = -0.5 * dlo;
            up[i] = -0.5 * dhi;
            rhs[i] = -R[i];
        }
        // Thomas algorithm
        for (int i = 1; i < n; ++i) {
            const double w = lo[i] / di[i - 1];
            di[i] -= w * up[i - 1];
            rhs[i] -= w * rhs[i - 1];
        }
        std::vector<double> step(n);
        step[n - 1] = rhs[n - 1] / di[n - 1];
        for (int i = n - 2; i >= 0; --i) step[i] = (rhs[i] - up[i] * step[i + 1]) / di[i];
        // damped update: keep the levels ordered inside (0, 1) and the residual falling
        double lam = 1.0;
        std::vector<double> trial(n);
        double tres = 0.0;
        for (int tries = 0; tries < 40; ++tries, lam *= 0.5) {
            bool ok = true;
            for (int i = 0; i < n; ++i) {
                trial[i] = q[i] + lam * step[i];
                if (!(trial[i] > (i ? trial[i - 1] : 0.0)) || !(trial[i] < 1.0)) ok = false;
            }
            if (!ok) continue;
            tres = eval(trial);
            if (tres <= res || tres < 1e-17 * sigma) break;
        }
        double move = 0.0;
        for (int i = 0; i < n; ++i) move = std::max(move, std::fabs(trial[i] - q[i]));
        q = trial;
        res = eval(q);
        if (move < 1e-18 * sigma) break;
    }
    // the cell moments carry about 1e-13 of noise (differences of incomplete
    // beta tails), which at 256 levels and large d is above 1e-11 sigma
    return res < 1e-11 * sigma || res < 4e-13;
}

}  // namespace

// ---------------------------------------------------------------------------
// bf16 round-to-nearest-even straight from the fp64 bit pattern (one
// rounding of the 52-bit significand to 7 stored bits).  Normal range.
// ---------------------------------------------------------------------------
uint16_t bf16_round(double x) {
    uint64_t u;
    std::memcpy(&u, &x, 8);
    const uint64_t sign = u >> 63;
    const int64_t e = (int64_t)((u >> 52) & 0x7ff);
    if (e == 0) return (uint16_t)(sign << 15);  // zero (fp64 subnormals are far below bf16's range)
    uint64_t mant = u & ((1ull << 52) - 1);
    // keep 7 bits: round at bit 45 with ties to even
    const uint64_t lsb = (mant >> 45) & 1u;
    mant += (1ull << 44) - 1 + lsb;
    int64_t eb = e - 1023 + 127;
    if (mant >> 52) {  // carried into the exponent
        mant = 0;
        eb += 1;
    }
    if (eb >= 255) return (uint16_t)((sign << 15) | 0x7f80u);
    if (eb <= 0) return (uint16_t)(sign << 15);  // below bf16's normal range: flush (not reached here)
    return (uint16_t)((sign << 15) | ((uint64_t)eb << 7) | (mant >> 45));
}

// ---------------------------------------------------------------------------
// C_d for (d, bits), and the tables the kernels use.
// ---------------------------------------------------------------------------
oq_status build_codebook(int d, int bits, oq_codebook_t* cb) {
    if (d < 3 || bits < 1 || bits > 8) return OQ_ERR_UNSUPPORTED;
    const int L = 1 << bits, n = L / 2;
    Marginal f(d);
    std::vector<double> q;
    if (!solve_positive_half(f, n, q)) return OQ_ERR_NO_CONVERGENCE;
    cb->d = d;
    cb->bits = bits;
    cb->L = L;
    cb->c.assign(L, 0.0);
    for (int i = 0; i < n; ++i) {
        cb->c[n + i] = q[i];
        cb->c[n - 1 - i] = -q[i];
    }
    cb->t.assign(L - 1, 0.0);
    for (int j = 0; j + 1 < L; ++j) cb->t[j] = 0.5 * (cb->c[j] + cb->c[j + 1]);
    cb->t32.resize(L - 1);
    for (int j = 0; j + 1 < L; ++j) cb->t32[j] = (float)cb->t[j];
    cb->c_bf16.resize(L);
    for (int j = 0; j < L; ++j) cb->c_bf16[j] = bf16_round(cb->c[j]);
    cb->c_e4m3.resize(L);
    for (int j = 0; j < L; ++j) cb->c_e4m3[j] = e4m3_round(cb->c[j] * std::sqrt((double)d));

    // Lookup table over v in [-vmax, vmax] with at most one fp32 threshold
    // per bin.  The bins are exactly the kernel's: bin(v) = bits of
    // fmaf(v, G, 1.5*2^23) minus the magic's bits, so host and device agree.
    auto bin_of = [](float v, float G) {
        const float z = std::fmaf(v, G, kLutMagic);
        uint32_t b;
        std::memcpy(&b, &z, 4);
        return (int)(int32_t)(b - kLutMagicBits);
    };
    double min_gap = 1.0;
    for (int j = 0; j + 2 < L; ++j) min_gap = std::min(min_gap, (double)cb->t32[j + 1] - (double)cb->t32[j]);
    float G = (float)(1.0 / min_gap);
    if (L == 2) G = 4.0f;
    const float vmax = 1.0f + 1.0f / 16.0f;  // |v| <= 1 up to fp32 rounding for the rows the kernel quantises
    bool separated = false;
    for (int tries = 0; tries < 64 && !separated; ++tries) {
        separated = true;
        for (int j = 0; j + 2 < L; ++j)
            if (bin_of(cb->t32[j], G) >= bin_of(cb->t32[j + 1], G)) separated = false;
        if (!separated) G *= 1.25f;
    }
    // the kernels' one-compare lookup is exact only with at most one
    // threshold per bin: refuse the codebook rather than build a wrong table
    if (!separated) return OQ_ERR_NO_CONVERGENCE;
    cb->G = G;
    const int kmin = bin_of(-vmax, G), kmax = bin_of(vmax, G);
    cb->kmin = kmin;
    cb->lut.assign(kmax - kmin + 1, LutEntry{std::numeric_limits<float>::infinity(), 0});
    for (int k = kmin; k <= kmax; ++k) {
        LutEntry& e = cb->lut[k - kmin];
        int base = 0;
        for (int j = 0; j + 1 < L; ++j) {
            const int bj = bin_of(cb->t32[j], G);
            if (bj < k) ++base;
            if (bj == k) e.T = cb->t32[j];
        }
        e.base = base;
    }
    // an even entry count: the kernels stage the table with a 16-byte-multiple
    // bulk copy (the extra entry is never indexed)
    if (cb->lut.size() % 2) cb->lut.push_back(cb->lut.back());
    return OQ_OK;
}

// ---------------------------------------------------------------------------
// e4m3 (8 bits: sign, 4 exponent bits with bias 7, 3 mantissa bits; no
// infinities; largest finite 448; subnormals k * 2^-9): round to nearest,
// ties to even, once from the exact value; saturates at +-448.
// ---------------------------------------------------------------------------
uint8_t e4m3_round(double v) {
    const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
    const double a = std::fabs(v);
    if (std::isnan(a)) return sign | 0x7f;
    int e = 0;
    std::frexp(a, &e);                        // a in [2^(e-1), 2^e)
    const int E = std::max(e - 1, -6);        // binade (subnormals share the 2^-6 spacing)
    const double q = std::ldexp(1.0, E - 3);  // spacing of 3 mantissa bits
    double r = std::nearbyint(a / q) * q;     // a / q is exact; the default mode rounds ties to even
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return sign;
    if (r < std::ldexp(1.0, -6)) return sign | (uint8_t)(r / std::ldexp(1.0, -9));
    std::frexp(r, &e);
    const int E2 = e - 1;
    const int mant = (int)((r / std::ldexp(1.0, E2) - 1.0) * 8.0);
    return sign | (uint8_t)(((E2 + 7) << 3) | mant);
}

// ---------------------------------------------------------------------------
// RPBH plan: SplitMix64 (Steele, Lea & Flood 2014) drives a Fisher-Yates
// (Durstenfeld) shuffle of the identity, then the Rademacher signs.
// ---------------------------------------------------------------------------
void make_plan(int d, int h, uint64_t seed, int32_t* perm, int8_t* sign, int variant) {
    (void)h;
    uint64_t state = seed;
    auto next = [&state]() {
        state += 0x9E3779B97F4A7C15ull;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        return z ^ (z >> 31);
    };
    for (int i = 0; i < d; ++i) perm[i] = i;
    if (variant == OQ_ROT_RPBH)
        for (int i = d - 1; i > 0; --i) {
            const int j = (int)(next() % (uint64_t)(i + 1));
            std::swap(perm[i], perm[j]);
        }
    // Block-RHT (the ablation without P_pi): identity permutation, signs
    // from the first d draws of the same generator
    for (int k = 0; k < d; ++k) sign[k] = (next() >> 63) ? (int8_t)-1 : (int8_t)1;
}

// Gather table: the entry of post-permutation coordinate k = b*h + i is
// (2 pi(k)) << 16 | 0x8000 * (sigma_k < 0): the byte offset of the bf16
// element x[pi(k)] in its row (the fp32 kernel doubles it) and the sign of
// D_k.  Stored in 16-byte chunks of 4 entries, chunk (c, b) (entries
// b*h + 4c .. b*h + 4c + 3) at chunk index c*nb + b, so that lanes working on
// neighbouring blocks read neighbouring chunks.  Offsets fit 16 bits since
// d <= 32767.
void build_gather_table(const oq_plan_t* p, std::vector<uint32_t>& out) {
    const int d = p->d, h = p->h, nb = d / h, nc = h / 4;
    out.assign(d, 0);
    for (int b = 0; b < nb; ++b)
        for (int c = 0; c < nc; ++c)
            for (int e = 0; e < 4; ++e) {
                const int k = b * h + c * 4 + e;
                out[(size_t)(c * nb + b) * 4 + e] =
                    ((uint32_t)(2 * p->perm[k]) << 16) | (p->sign[k] < 0 ? 0x8000u : 0u);
            }
}

// The warp-group kernel's gather table: the entry of coordinate k = b*h + i
// is pi(k) | 0x8000 * (sigma_k < 0) (the element index, 15 bits since
// d <= 32767, and the sign of D_k), in 16-byte chunks of 8 entries, chunk
// (c, b) (entries b*h + 8c .. b*h + 8c + 7) at chunk index c*nb + b.
void build_gather_table16(const oq_plan_t* p, std::vector<uint16_t>& out) {
    const int d = p->d, h = p->h, nb = d / h, nc = h / 8;
    out.assign(d, 0);
    for (int b = 0; b < nb; ++b)
        for (int c = 0; c < nc; ++c)
            for (int e = 0; e < 8; ++e) {
                const int k = b * h + c * 8 + e;
                out[(size_t)(c * nb + b) * 8 + e] = (uint16_t)(p->perm[k] | (p->sign[k] < 0 ? 0x8000 : 0));
            }
}

}  // namespace oq
