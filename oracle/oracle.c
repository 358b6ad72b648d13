/*
 * oracle.c -- plain fp64 CPU oracle for the OrbitQuant rotate-then-quantize
 * linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA library; neither includes or
 * links the other.  It is written for a reader who checks it against the
 * pages by eye: no blocking, no fusion, no reordering beyond what the method
 * states, fp64 throughout.
 *
 * Source of every step: "OrbitQuant" paper summary (hyper.ai, papers
 * 2607.02461), section 方法 (Method):
 *   - offline weight stage:  W' = W Pi_d^T, r'_i = ||w'_i||, w~'_i = w'_i / r'_i,
 *     W^' = diag(r') Q_bw(W~'), r' stored as BF16;
 *   - online activation stage: x' = Pi_d x, s = ||x'||, x~' = x' / (s + eps),
 *     x^' = s Q_ba(x~');  the product W^' x^' approximates W x;
 *   - RPBH: Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi;
 *   - codebook C_d: Lloyd-Max run offline on the fixed marginal f_d of a
 *     rotated unit coordinate.
 *
 * Readings taken where the page is silent (each is listed in the design
 * notes of the repository):
 *   - f_d(t) = c_d (1 - t^2)^((d-3)/2) on [-1, 1], the exact marginal of one
 *     coordinate of a uniformly random unit vector in R^d.
 *   - H_h is the Sylvester-ordered Walsh-Hadamard matrix scaled by 1/sqrt(h),
 *     H[a][b] = (-1)^popcount(a & b) / sqrt(h).
 *   - (P_pi x)_k = x_{pi(k)}; D_i signs are indexed by the post-permutation
 *     coordinate k.
 *   - pi and the signs come from SplitMix64(seed): a Fisher-Yates
 *     (Durstenfeld) shuffle of the identity for i = d-1 .. 1 with
 *     j = next() mod (i+1), then d signs sigma_k = (next() >> 63) ? -1 : +1.
 *   - quantiser index = #{ j : t_j <= v } over the sorted thresholds
 *     (ties go to the upper cell); eps = 1e-12 on both sides.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Gauss-Legendre nodes on [-1, 1] by Newton's iteration on P_n (the classic  */
/* method of Golub & Welsch's predecessors; see e.g. Abramowitz & Stegun     */
/* 25.4.29).                                                                  */
/* ------------------------------------------------------------------------ */
#define GL_N 20
static double gl_x[GL_N], gl_w[GL_N];
static int gl_ready = 0;

static void gl_init(void) {
    if (gl_ready) return;
    const int n = GL_N;
    for (int i = 0; i < n; ++i) {
        double x = cos(M_PI * (i + 0.75) / (n + 0.5));
        double dp = 0.0;
        for (int it = 0; it < 100; ++it) {
            double p0 = 1.0, p1 = x;
            for (int k = 2; k <= n; ++k) {
                double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
                p0 = p1;
                p1 = p2;
            }
            /* p1 = P_n(x), p0 = P_{n-1}(x) */
            dp = n * (x * p1 - p0) / (x * x - 1.0);
            double dx = p1 / dp;
            x -= dx;
            if (fabs(dx) < 1e-16) break;
        }
        {
            double p0 = 1.0, p1 = x;
            for (int k = 2; k <= n; ++k) {
                double p2 = ((2.0 * k - 1.0) * x * p1 - (k - 1.0) * p0) / k;
                p0 = p1;
                p1 = p2;
            }
            dp = n * (x * p1 - p0) / (x * x - 1.0);
        }
        gl_x[i] = x;
        gl_w[i] = 2.0 / ((1.0 - x * x) * dp * dp);
    }
    gl_ready = 1;
}

/* ------------------------------------------------------------------------ */
/* The density whose Lloyd-Max quantiser is sought, in the scaled variable   */
/* u = t * sqrt(d) (so that the spread is O(1) for every d).                 */
/*   kind 0: f_d of a rotated unit coordinate, f_d(t) = c_d (1-t^2)^((d-3)/2) */
/*           on [-1, 1].  Cells are integrated in theta with t = sin(theta): */
/*           f_d(t) dt = c_d cos(theta)^(d-2) dtheta is smooth up to the     */
/*           support's edge for every d (in t it is not, for small d).       */
/*   kind 1: the standard normal (used only to pin the solver against the    */
/*           published Gaussian Lloyd-Max tables), integrated in u.          */
/* ------------------------------------------------------------------------ */
typedef struct {
    int kind;
    int d;
    double logc; /* kind 0: log c_d (t units); kind 1: log 1/sqrt(2 pi) */
    double sd;   /* sqrt(d) for kind 0, 1 for kind 1 */
    double xmax; /* half-width of the integration variable carrying fp64 mass */
    double panel;/* panel width in the integration variable */
} density_t;

static void integrate2(const density_t* g, double a, double b, double* m0, double* m1);

static density_t density_make(int kind, int d) {
    density_t g;
    g.kind = kind;
    g.d = d;
    if (kind == 0) {
        g.sd = sqrt((double)d);
        /* c_d = Gamma(d/2) / (sqrt(pi) Gamma((d-1)/2)) */
        g.logc = lgamma(0.5 * d) - 0.5 * log(M_PI) - lgamma(0.5 * (d - 1));
        /* |u| = 40 carries no fp64 mass (density below exp(-790)) */
        g.xmax = (g.sd > 40.0) ? asin(40.0 / g.sd) : 0.5 * M_PI;
        g.panel = 0.125 / g.sd; /* the same resolution as 0.125 in u at the centre */
        /* The lgamma difference loses ~1e-12 relative at d ~ 1e4 (two values  */
        /* near 1e4 cancel); refine c_d so that the total mass is 1.           */
        double m0, m1;
        integrate2(&g, -INFINITY, INFINITY, &m0, &m1);
        g.logc -= log(m0);
    } else {
        g.sd = 1.0;
        g.logc = -0.5 * log(2.0 * M_PI);
        g.xmax = 40.0;
        g.panel = 0.125;
    }
    return g;
}

/* Mass and first moment (in u units) of the density over u in [a, b], by   */
/* composite 20-point Gauss-Legendre in the integration variable.            */
static void integrate2(const density_t* g, double a, double b, double* m0, double* m1) {
    gl_init();
    *m0 = 0.0;
    *m1 = 0.0;
    double xa, xb;
    if (g->kind == 0) {
        xa = (a <= -g->sd) ? -0.5 * M_PI : asin(a / g->sd);
        xb = (b >= g->sd) ? 0.5 * M_PI : asin(b / g->sd);
    } else {
        xa = a;
        xb = b;
    }
    if (xa < -g->xmax) xa = -g->xmax;
    if (xb > g->xmax) xb = g->xmax;
    if (!(xb > xa)) return;
    int np = (int)ceil((xb - xa) / g->panel);
    if (np < 1) np = 1;
    double w = (xb - xa) / np, s0 = 0.0, s1 = 0.0;
    for (int p = 0; p < np; ++p) {
        double mid = xa + (p + 0.5) * w, p0 = 0.0, p1 = 0.0;
        for (int i = 0; i < GL_N; ++i) {
            double x = mid + 0.5 * w * gl_x[i];
            double f, u;
            if (g->kind == 0) {
                double c = cos(x);
                f = exp(g->logc + (g->d - 2) * log(c)); /* c_d cos^(d-2) */
                u = g->sd * sin(x);
            } else {
                f = exp(g->logc - 0.5 * x * x);
                u = x;
            }
            p0 += gl_w[i] * f;
            p1 += gl_w[i] * u * f;
        }
        s0 += 0.5 * w * p0;
        s1 += 0.5 * w * p1;
    }
    *m0 = s0;
    *m1 = s1;
}

/* ------------------------------------------------------------------------ */
/* Lloyd-Max (Lloyd's "method I" / Max's conditions): thresholds are the     */
/* midpoints of adjacent centroids, each centroid is the conditional mean of */
/* its cell; iterate until the centroids stop moving.                        */
/* Works in u units; returns the number of iterations, or -1 if the cap was  */
/* hit.                                                                       */
/* ------------------------------------------------------------------------ */
static int lloyd_max_u(const density_t* g, int L, double* cu, double* tu, double tol, int max_iter) {
    gl_init();
    /* start: levels spread evenly over +-3 (any start converges: the density */
    /* is log-concave, so the fixed point is unique)                          */
    for (int j = 0; j < L; ++j) cu[j] = 3.0 * (2.0 * (j + 0.5) / L - 1.0);
    int it;
    for (it = 1; it <= max_iter; ++it) {
        for (int j = 0; j + 1 < L; ++j) tu[j] = 0.5 * (cu[j] + cu[j + 1]);
        double delta = 0.0;
        for (int j = 0; j < L; ++j) {
            double a = (j == 0) ? -INFINITY : tu[j - 1];
            double b = (j == L - 1) ? INFINITY : tu[j];
            double m0, m1;
            integrate2(g, a, b, &m0, &m1);
            double c = (m0 > 0.0) ? m1 / m0 : 0.5 * (a + b);
            double dd = fabs(c - cu[j]);
            if (dd > delta) delta = dd;
            cu[j] = c;
        }
        if (delta < tol) break;
    }
    for (int j = 0; j + 1 < L; ++j) tu[j] = 0.5 * (cu[j] + cu[j + 1]);
    return (it > max_iter) ? -1 : it;
}

/* C_d for a dimension d and a bit width (levels L = 2^bits), in t units.    */
/* centroids: L values, thresholds: L-1 values.  Returns iterations or <0.   */
/* f_d is even, so C_d is symmetric about 0; with symmetrize != 0 the        */
/* rounding-level asymmetry of the iteration is removed (c_j = -c_{L-1-j}    */
/* exactly), which makes the middle threshold exactly 0 for even L.          */
int oracle_codebook_ex(int d, int bits, int symmetrize, double* centroids, double* thresholds) {
    if (d < 3 || bits < 1 || bits > 8) return -2;
    int L = 1 << bits;
    density_t g = density_make(0, d);
    double* cu = (double*)malloc(sizeof(double) * L);
    double* tu = (double*)malloc(sizeof(double) * L);
    int it = lloyd_max_u(&g, L, cu, tu, 1e-14, 200000);
    if (symmetrize) {
        for (int j = 0; j < L / 2; ++j) {
            double m = 0.5 * (cu[L - 1 - j] - cu[j]);
            cu[j] = -m;
            cu[L - 1 - j] = m;
        }
        for (int j = 0; j + 1 < L; ++j) tu[j] = 0.5 * (cu[j] + cu[j + 1]);
    }
    double sd = sqrt((double)d);
    for (int j = 0; j < L; ++j) centroids[j] = cu[j] / sd;
    for (int j = 0; j + 1 < L; ++j) thresholds[j] = tu[j] / sd;
    free(cu);
    free(tu);
    return it;
}

int oracle_codebook(int d, int bits, double* centroids, double* thresholds) {
    return oracle_codebook_ex(d, bits, 1, centroids, thresholds);
}

/* The same solver on N(0, 1), to pin it against published Gaussian tables. */
int oracle_codebook_gauss(int levels, double* centroids, double* thresholds) {
    if (levels < 2 || levels > 256) return -2;
    density_t g = density_make(1, 0);
    return lloyd_max_u(&g, levels, centroids, thresholds, 1e-14, 200000);
}

/* Cell mass and first moment of f_d over [a, b] (t units), by the same      */
/* quadrature; exposed so tests can compare it with closed forms.            */
void oracle_fd_moments(int d, double a, double b, double* mass, double* first) {
    density_t g = density_make(0, d);
    integrate2(&g, a * g.sd, b * g.sd, mass, first);
    *first /= g.sd;
}

/* ------------------------------------------------------------------------ */
/* RPBH plan: SplitMix64 (Steele, Lea & Flood 2014; Vigna's reference        */
/* generator), Fisher-Yates / Durstenfeld shuffle, Rademacher signs.         */
/* ------------------------------------------------------------------------ */
static uint64_t splitmix64_next(uint64_t* state) {
    uint64_t z = (*state += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

void oracle_splitmix64(uint64_t seed, int n, uint64_t* out) {
    uint64_t s = seed;
    for (int i = 0; i < n; ++i) out[i] = splitmix64_next(&s);
}

int oracle_plan_variant(int d, int h, uint64_t seed, int variant, int32_t* perm, int8_t* sign);

int oracle_plan(int d, int h, uint64_t seed, int32_t* perm, int8_t* sign) {
    return oracle_plan_variant(d, h, seed, 0, perm, sign);
}

/* variant 0: RPBH (above).  variant 1: Block-RHT, the page's ablation
 * without the permutation (section 实验, rotation ablation): pi is the
 * identity and the d signs are the generator's first d draws. */
int oracle_plan_variant(int d, int h, uint64_t seed, int variant, int32_t* perm, int8_t* sign) {
    if (d <= 0 || h <= 0 || d % h != 0 || (variant != 0 && variant != 1)) return -1;
    uint64_t s = seed;
    for (int i = 0; i < d; ++i) perm[i] = i;
    if (variant == 0)
        for (int i = d - 1; i >= 1; --i) {
            uint64_t j = splitmix64_next(&s) % (uint64_t)(i + 1);
            int32_t t = perm[i];
            perm[i] = perm[j];
            perm[j] = t;
        }
    for (int k = 0; k < d; ++k) sign[k] = (splitmix64_next(&s) >> 63) ? -1 : 1;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* RPBH of one row, evaluated straight from the definition:                  */
/*   y_k = (1/sqrt(h)) sum_{j in block(k)} H[k mod h][j mod h] sigma_j x_{pi(j)} */
/* an O(h) sum per output (no butterfly).                                    */
/* ------------------------------------------------------------------------ */
static void rpbh_row(int d, int h, const int32_t* perm, const int8_t* sign, const double* x, double* y) {
    double inv = 1.0 / sqrt((double)h);
    for (int b0 = 0; b0 < d; b0 += h) {
        for (int a = 0; a < h; ++a) {
            double acc = 0.0;
            for (int c = 0; c < h; ++c) {
                int j = b0 + c;
                double u = sign[j] * x[perm[j]];
                acc += (__builtin_popcount((unsigned)(a & c)) & 1) ? -u : u;
            }
            y[b0 + a] = acc * inv;
        }
    }
}

void oracle_rpbh(int M, int d, int h, const int32_t* perm, const int8_t* sign, const double* x, double* y) {
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) rpbh_row(d, h, perm, sign, x + (size_t)m * d, y + (size_t)m * d);
}

/* ------------------------------------------------------------------------ */
/* Norm / direction split and Lloyd-Max quantisation of rows.                */
/*   y = Pi x;  s = ||y||_2;  v = y / (s + eps);  idx_k = #{ j : t_j <= v_k }  */
/* decision = 64: the comparison is made in fp64 on fp64 thresholds;         */
/* decision = 32: v and the thresholds are first rounded to fp32 and the     */
/*               comparison is made in fp32 (the precision the GPU kernel    */
/*               decides in).                                                */
/* Outputs: idx (M x d, one byte per index, unpacked), s (M), and optionally */
/* y (M x d) and v (M x d) for diagnostics (pass NULL to skip).              */
/* ------------------------------------------------------------------------ */
void oracle_quantize_rows(int M, int d, int h, const int32_t* perm, const int8_t* sign, const double* x,
                          int L, const double* thresholds, double eps, int decision, uint8_t* idx, double* s_out,
                          double* y_out, double* v_out) {
    float* t32 = (float*)malloc(sizeof(float) * (L > 1 ? L - 1 : 1));
    for (int j = 0; j + 1 < L; ++j) t32[j] = (float)thresholds[j];
#pragma omp parallel
    {
        double* y = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(static)
        for (int m = 0; m < M; ++m) {
            rpbh_row(d, h, perm, sign, x + (size_t)m * d, y);
            double ss = 0.0;
            for (int k = 0; k < d; ++k) ss += y[k] * y[k];
            double s = sqrt(ss);
            s_out[m] = s;
            for (int k = 0; k < d; ++k) {
                double v = y[k] / (s + eps);
                int cnt = 0;
                if (decision == 32) {
                    float v32 = (float)v;
                    for (int j = 0; j + 1 < L; ++j) cnt += (t32[j] <= v32);
                } else {
                    for (int j = 0; j + 1 < L; ++j) cnt += (thresholds[j] <= v);
                }
                idx[(size_t)m * d + k] = (uint8_t)cnt;
                if (y_out) y_out[(size_t)m * d + k] = y[k];
                if (v_out) v_out[(size_t)m * d + k] = v;
            }
        }
        free(y);
    }
    free(t32);
}

/* ------------------------------------------------------------------------ */
/* bf16 round-to-nearest-even, taken straight from the fp64 value: the       */
/* 8-bit significand is rounded once (no intermediate fp32 rounding).        */
/* Normal bf16 range only (the values stored here are norms and centroids).  */
/* ------------------------------------------------------------------------ */
static double bf16_rne(double x) {
    if (x == 0.0 || !isfinite(x)) return (double)(float)x;
    int e;
    double m = frexp(x, &e);          /* x = m 2^e, 0.5 <= |m| < 1 */
    double r = nearbyint(ldexp(m, 8)); /* 8 significant bits, ties to even */
    return ldexp(r, e - 8);
}

static uint16_t bf16_bits_of(double v) {
    float f = (float)v; /* exact: v has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

void oracle_round_bf16(int n, const double* in, uint16_t* out_bits, double* out_val) {
    for (int i = 0; i < n; ++i) {
        double v = bf16_rne(in[i]);
        if (out_bits) out_bits[i] = bf16_bits_of(v);
        if (out_val) out_val[i] = v;
    }
}

/* ------------------------------------------------------------------------ */
/* Quantised linear layer:                                                   */
/*   y[m][n] = r[n] * s[m] * sum_k cw[iw[n][k]] * ca[ia[m][k]]               */
/* where cw / ca are the centroid values as they are stored for the product */
/* (the caller passes them; bf16-rounded C_d entries), r the stored row norm */
/* and s the activation norm.  Only rows listed in rows[] (all if NULL) and */
/* columns listed in cols[] (all if NULL) are produced; out is               */
/* n_rows x n_cols.                                                           */
/* ------------------------------------------------------------------------ */
void oracle_qlinear(int M, int N, int d, const uint8_t* ia, const double* s, const uint8_t* iw, const double* r,
                    const double* ca, const double* cw, int n_rows, const int32_t* rows, int n_cols,
                    const int32_t* cols, double* out) {
    if (!rows) n_rows = M;
    if (!cols) n_cols = N;
#pragma omp parallel for schedule(dynamic, 4)
    for (int a = 0; a < n_rows; ++a) {
        int m = rows ? rows[a] : a;
        const uint8_t* xa = ia + (size_t)m * d;
        for (int b = 0; b < n_cols; ++b) {
            int n = cols ? cols[b] : b;
            const uint8_t* wn = iw + (size_t)n * d;
            double acc = 0.0;
            for (int k = 0; k < d; ++k) acc += cw[wn[k]] * ca[xa[k]];
            out[(size_t)a * n_cols + b] = r[n] * s[m] * acc;
        }
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Thread count of the following parallel loops (timing the oracle on one
 * core and on all of them); n <= 0 restores the default. */
static int oracle_default_threads = 0;

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (!oracle_default_threads) oracle_default_threads = omp_get_max_threads();
    omp_set_num_threads(n > 0 ? n : oracle_default_threads);
#else
    (void)n;
#endif
}
