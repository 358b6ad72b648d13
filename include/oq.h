/*
 * oq.h -- C ABI of liboq: OrbitQuant-style rotate-then-quantize linear layers
 * on NVIDIA B200 (sm_100a).
 *
 * Method: "OrbitQuant" paper summary (hyper.ai, papers 2607.02461), section
 * 方法 (Method).  A linear layer with input dimension d shares one rotation
 * Pi_d between its weights and its activations:
 *   offline:  W' = W Pi_d^T; each row w'_n = r_n * w~'_n with r_n = ||w'_n||_2
 *             stored as BF16; w~'_n is quantised with the Lloyd-Max codebook
 *             C_d of b_w bits.
 *   online:   x' = Pi_d x; s = ||x'||_2; x~' = x' / (s + eps) quantised with
 *             C_d of b_a bits; y = (W^' x^') with no inverse rotation.
 *   RPBH:     Pi_d = blkdiag(H_h D_1, ..., H_h D_{d/h}) P_pi.
 *   C_d:      Lloyd-Max quantiser of the marginal f_d of one coordinate of a
 *             rotated unit vector, built once per (d, bits), data-free.
 *
 * Conventions for every call:
 *   - Status codes are returned; nothing throws and nothing exits.
 *   - Tensor buffers are owned by the caller.  "device" pointers must be
 *     CUDA device memory of the device that is current on the calling
 *     thread (the device the plan was created on); "host" pointers are
 *     ordinary host memory.  Device pointers must be 16-byte aligned
 *     (OQ_ERR_ALIGNMENT otherwise).
 *   - Plan and codebook handles are owned by the library and released with
 *     their free functions.  A plan holds device tables on the device that
 *     was current when it was created.
 *   - Device work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and is asynchronous.  Only set-up calls synchronise:
 *     oq_rpbh_plan / oq_rotation_plan and oq_codebook_upload allocate and copy
 *     their tables with a synchronous copy, and so does the first quantising
 *     call of a codebook on a device that it was not uploaded to (call
 *     oq_codebook_upload at set-up to keep the hot calls free of allocation
 *     and synchronisation).  oq_device_status synchronises its stream.
 *     Launch failures are reported as OQ_ERR_CUDA.  A kernel that gives up a
 *     bounded wait records OQ_ERR_TIMEOUT in a device flag read by
 *     oq_device_status().
 *   - The quantising calls, the products and the layer calls may be
 *     captured in a CUDA graph (stream capture) once one eager call of the
 *     same kind has run on the device: that call uploads what is missing
 *     and sets the kernels' launch attributes, which capture cannot do.
 *     A quantiser followed by its product keeps their programmatic
 *     dependency inside the graph.
 *   - Layouts are row-major.  Packed indices are K-major rows, LSB-first:
 *     bits = 4: two indices per byte (index k in bits 4*(k%2) of byte k/2);
 *     bits = 2: four per byte (bits 2*(k%4) of byte k/4);
 *     bits = 6: one index per byte (low 6 bits);
 *     bits = 8: one index per byte (activations and weights are quantised;
 *               the products take 8-bit activations as values only);
 *     bits = 3: a bit stream, index k in bits 3k..3k+2 of the row (eight
 *               indices per three bytes); needs h >= 32 and d % 128 == 0,
 *               and runs through the fp8 product variant only.
 *     Index j means centroid c_j of C_d sorted ascending (0 = most negative).
 *   - eps = 1e-12 on both the weight and the activation side.
 */
#ifndef OQ_H
#define OQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    OQ_OK = 0,
    OQ_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, mismatched handles */
    OQ_ERR_UNSUPPORTED = 2, /* d % h != 0, h not a power of two in [16, 128], bits not in {2,3,4,6,8}, d % 64 != 0 */
    OQ_ERR_ALIGNMENT = 3,   /* a device pointer is not 16-byte aligned */
    OQ_ERR_CUDA = 4,        /* a CUDA runtime call or a kernel launch failed */
    OQ_ERR_TIMEOUT = 5,     /* a kernel gave up a bounded wait (see oq_device_status) */
    OQ_ERR_OOM = 6,         /* a library-owned allocation failed, or the workspace is too small */
    OQ_ERR_NO_CONVERGENCE = 7, /* the codebook solver did not converge */
    OQ_ERR_TOO_LARGE = 8       /* the request does not fit the fixed scratch of oq_qlinear_noalloc */
} oq_status;

typedef enum { OQ_BF16 = 0, OQ_F32 = 1 } oq_dtype;

typedef struct oq_codebook_s oq_codebook_t;
typedef struct oq_plan_s oq_plan_t;

/* Human-readable name of a status code (static string). */
const char* oq_status_str(oq_status s);

/* ---------------------------------------------------------------------- */
/* A0. Codebook C_d  [OrbitQuant, Method: "Lloyd-Max run offline on f_d,   */
/*     one codebook per dimension"].                                       */
/* Builds the 2^bits-level Lloyd-Max quantiser of                          */
/*   f_d(t) = c_d (1 - t^2)^((d-3)/2),  t in [-1, 1]                        */
/* on the host in fp64 (Newton iteration on the Lloyd-Max conditions, cell */
/* masses from the regularised incomplete beta function), then derives the */
/* fp32 thresholds, bf16 centroids and the quantiser lookup table the      */
/* kernels use.  Host-only: needs no GPU.                                  */
/*   d    >= 3;  bits in {1..8} (the quantising calls accept               */
/*   {2, 3, 4, 6, 8}).                                                     */
/*   out  receives a library-owned handle (free with oq_codebook_free).    */
oq_status oq_codebook(int d, int bits, oq_codebook_t** out);

/* Uploads the codebook's quantiser tables to the current device          */
/* (allocation and a synchronous copy; once per codebook and device --     */
/* later calls return at once).  The quantising calls do it themselves on  */
/* first use; calling it at set-up keeps them free of both.  The tables    */
/* are freed by oq_codebook_free.  OQ_ERR_OOM / OQ_ERR_CUDA on failure.    */
oq_status oq_codebook_upload(const oq_codebook_t* cb);

/* Copies the fp64 codebook: centroids[2^bits] ascending and               */
/* thresholds[2^bits - 1] (midpoints of adjacent centroids; the middle one */
/* is exactly 0).  Host pointers; either may be NULL.                       */
oq_status oq_codebook_values(const oq_codebook_t* cb, double* centroids, double* thresholds);

/* Copies the bf16 bit patterns of the centroids as the product uses them  */
/* (round-to-nearest-even of the fp64 values).  Host pointer, 2^bits.      */
oq_status oq_codebook_bf16(const oq_codebook_t* cb, uint16_t* centroids_bf16);

/* (d, bits) of a codebook.  Host pointers; either may be NULL. */
oq_status oq_codebook_shape(const oq_codebook_t* cb, int* d, int* bits);

void oq_codebook_free(oq_codebook_t* cb);

/* ---------------------------------------------------------------------- */
/* RPBH plan  [OrbitQuant, Method: Pi_d = blkdiag(H_h D_1..H_h D_{d/h}) P_pi, */
/*            P_pi a uniformly random permutation, D_i Rademacher signs].   */
/* pi and the signs come from SplitMix64(seed): a Fisher-Yates shuffle of  */
/* the identity (i = d-1..1, j = next() mod (i+1)), then d signs           */
/* sigma_k = (next() >> 63) ? -1 : +1.  (P_pi x)_k = x[pi(k)]; sigma_k     */
/* multiplies post-permutation coordinate k; H_h is Sylvester-ordered and  */
/* scaled by 1/sqrt(h).                                                     */
/*   d % h == 0, h a power of two in [16, 128], d <= 32767.                */
/* Uploads the plan's gather table to the current device.                  */
oq_status oq_rpbh_plan(int d, int h, uint64_t seed, oq_plan_t** out);

/* Host copy of the plan: perm[d] (int32, (P_pi x)_k = x[perm[k]]) and     */
/* sign[d] (int8, +-1).  Either may be NULL.                               */
oq_status oq_rpbh_plan_export(const oq_plan_t* plan, int32_t* perm, int8_t* sign);

/* Host-only plan generation (no device tables): same arrays as above.    */
/* Accepts any d in [1, 32767] and any h >= 1 dividing d (the arrays do    */
/* not depend on h); the device calls keep the limits of oq_rpbh_plan.     */
oq_status oq_rpbh_plan_host(int d, int h, uint64_t seed, int32_t* perm, int8_t* sign);

/* Rotation variants for the page's rotation ablation [OrbitQuant, section */
/* 实验 (Experiments), the rotation ablation: Block-RHT, RPBH].            */
/*   OQ_ROT_RPBH       the plan of oq_rpbh_plan.                           */
/*   OQ_ROT_BLOCK_RHT  Block-RHT: P_pi = identity; the signs are the first  */
/*                     d draws of SplitMix64(seed), with the same rule.    */
/* The variant plan feeds the same calls as an RPBH plan.  Unknown          */
/* variants return OQ_ERR_INVALID_ARG.                                     */
#define OQ_ROT_RPBH 0
#define OQ_ROT_BLOCK_RHT 1
oq_status oq_rotation_plan(int d, int h, uint64_t seed, int variant, oq_plan_t** out);
oq_status oq_rotation_plan_host(int d, int h, uint64_t seed, int variant, int32_t* perm, int8_t* sign);

/* (d, h) of a plan.  Host pointers; either may be NULL. */
oq_status oq_plan_shape(const oq_plan_t* plan, int* d, int* h);

void oq_plan_free(oq_plan_t* plan);

/* ---------------------------------------------------------------------- */
/* Offline weight pass  [OrbitQuant, Method: offline weight stage].         */
/* Row n of W' = W Pi_d^T is Pi_d w_n, so the same rotate-split-quantise   */
/* kernel runs on the rows of W:                                            */
/*   w'_n = Pi_d w_n;  r_n = ||w'_n||_2;  idx = Q_bw(w'_n / (r_n + eps)).   */
/*   W       device, [N, d] of `dtype` (bf16 or fp32), row-major.          */
/*   N       rows (> 0).                                                    */
/*   idx_out device, [N, d*bits/8] bytes (bits 6: [N, d]), packed as above. */
/*   r_out   device, [N] bf16 bit patterns: r_n rounded to nearest even.    */
oq_status oq_quantize_weights(const oq_plan_t* plan, const oq_codebook_t* cb_w, const void* W, oq_dtype dtype, int N,
                              uint8_t* idx_out, uint16_t* r_out, void* stream);

/* ---------------------------------------------------------------------- */
/* Online activation pass  [OrbitQuant, Method: online activation stage].  */
/*   x' = Pi_d x;  s = ||x'||_2 (fp32);  idx = Q_ba(x' / (s + eps)).        */
/*   x       device, [M, d] of `dtype`, row-major.  M >= 0 (0: no work; the */
/*           buffers may then be NULL).                                    */
/*   idx_out device, [M, d*bits/8] bytes (bits 6: [M, d]).                  */
/*   s_out   device, [M] fp32.                                              */
/* The decision v >= t_j is taken in fp32 (v = x'_k / (s + eps) rounded to */
/* fp32, t_j the fp32-rounded thresholds).  s is accumulated in fp32 from  */
/* the inputs (Pi_d is orthogonal, so ||x'|| = ||x||).  Rows whose norm is */
/* not finite or above FLT_MAX / (2 sqrt(h)) (where the fp32 transform     */
/* could overflow) are quantised to the middle cell (index 2^(bits-1))     */
/* with s stored as is.                                                    */
oq_status oq_quantize_acts(const oq_plan_t* plan, const oq_codebook_t* cb_a, const void* x, oq_dtype dtype, int M,
                           uint8_t* idx_out, float* s_out, void* stream);

/* The online pass with the centroid values written instead of the codes:  */
/* val_out[m, k] = C_a[idx[m, k]] with idx as oq_quantize_acts decides it  */
/* (same decision, same middle-cell rule), and the same s_out.            */
/*   val_out device, [M, d] bf16 bit patterns (the bf16 centroid values    */
/*           the product uses), row-major.                                 */
/* The _fp8 form writes the e4m3 bytes of c sqrt(d) that oq_qgemm_fp8      */
/* decodes to (oq_codebook_fp8); it needs d % 128 == 0.  Any bits in       */
/* {2, 3, 4, 6, 8}.  Used by the values schedule of oq_qlinear.            */
oq_status oq_quantize_acts_values(const oq_plan_t* plan, const oq_codebook_t* cb_a, const void* x, oq_dtype dtype,
                                  int M, uint16_t* val_out, float* s_out, void* stream);
oq_status oq_quantize_acts_values_fp8(const oq_plan_t* plan, const oq_codebook_t* cb_a, const void* x, oq_dtype dtype,
                                      int M, uint8_t* val_out, float* s_out, void* stream);

/* Test hook: steps A1-A4 only (permute, sign, block WHT, norm).           */
/*   x_rot   device, [M, d] fp32: x' = Pi_d x.   norm_out device, [M] fp32. */
oq_status oq_rpbh_apply(const oq_plan_t* plan, const void* x, oq_dtype dtype, int M, float* x_rot, float* norm_out,
                        void* stream);

/* ---------------------------------------------------------------------- */
/* Codebook-decode GEMM  [OrbitQuant, Method: W^' x^' ~ W x, no inverse     */
/* rotation at run time].                                                   */
/*   y[m, n] = r_n * s_m * sum_k  C_w[iw[n, k]] * C_a[ia[m, k]]  (+ bias_n)  */
/* with C_w, C_a the bf16 centroid values, fp32 accumulation, bf16 output.  */
/*   a_idx   device, [M, d*ba/8] packed activation indices; s device [M] f32. */
/*   w_idx   device, [N, d*bw/8] packed weight indices; w_r device [N] bf16. */
/*   bias    device [N] bf16 or NULL.   y device [M, N] bf16.              */
/*   d % 64 == 0; bits_w, bits_a in {2, 4, 6} (8-bit codes: no in-kernel  */
/*   decoder, OQ_ERR_UNSUPPORTED; 8-bit activations take the values        */
/*   schedule).  M >= 0, N > 0.                                            */
oq_status oq_qgemm(const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, int M, int N, const uint8_t* a_idx,
                   const float* s, const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y,
                   void* stream);

/* fp8 variant of oq_qgemm (a low-precision MMA variant the pages do not   */
/* describe).  The centroids enter the product as e4m3 values of           */
/* c_j sqrt(d) (rounded once, nearest-even; oq_codebook_fp8), multiplied   */
/* on tcgen05 kind::f8f6f4 in fp32; the epilogue applies s_m r_n / d (+bias) */
/* and rounds to bf16 once.  This trades the bf16 centroid values of       */
/* oq_qgemm (about 2^-9 relative error each) for e4m3 ones (about 2^-4) in */
/* exchange for throughput.  Same arguments and layouts as oq_qgemm;       */
/* d % 128 == 0 (OQ_ERR_UNSUPPORTED otherwise).                             */
oq_status oq_qgemm_fp8(const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, int M, int N, const uint8_t* a_idx,
                       const float* s, const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y,
                       void* stream);

/* oq_qgemm with A given as centroid values instead of codes:             */
/*   y[m, n] = r_n * s_m * sum_k  C_w[iw[n, k]] * a_val[m, k]  (+ bias_n)    */
/*   a_val   device, [M, d] bf16 (oq_quantize_acts_values), row-major.     */
/* With a_val = C_a[ia] this gives oq_qgemm's result bit for bit: the       */
/* tensor cores see the same values in the same order; only W is decoded   */
/* in the kernel, and A's values arrive by TMA.  d % 64 == 0, bits_w in     */
/* {2, 4, 6}.  The _fp8 form takes e4m3 bytes of c sqrt(d)                  */
/* (oq_quantize_acts_values_fp8) and matches oq_qgemm_fp8 bit for bit;     */
/* d % 128 == 0, bits_w in {2, 3, 4, 6}.                                    */
oq_status oq_qgemm_values(const oq_codebook_t* cb_w, int M, int N, const uint16_t* a_val, const float* s,
                          const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y, void* stream);
oq_status oq_qgemm_values_fp8(const oq_codebook_t* cb_w, int M, int N, const uint8_t* a_val, const float* s,
                              const uint8_t* w_idx, const uint16_t* w_r, const uint16_t* bias, uint16_t* y,
                              void* stream);

/* The fp8 variant's centroid values: out[2^bits] host bytes, e4m3 of     */
/* c_j sqrt(d) (sign, 4 exponent bits with bias 7, 3 mantissa bits).        */
oq_status oq_codebook_fp8(const oq_codebook_t* cb, uint8_t* out);

/* Bytes of workspace oq_qlinear needs for M rows in its codes schedule   */
/* (packed activation indices plus their norms, 256-byte aligned sections) */
/* and in its values schedule (bf16 activation values plus norms; enough  */
/* for the fp8 form too).                                                  */
size_t oq_qlinear_workspace(int M, int d, int bits_a);
size_t oq_qlinear_workspace_values(int M, int d);

/* Full layer x -> y.  Two schedules with the same result bit for bit:    */
/*   values: oq_quantize_acts_values into `workspace`, then               */
/*     oq_qgemm_values; taken when ws_bytes >=                             */
/*     oq_qlinear_workspace_values(M, d) (fp8: M*d bytes plus the norms,  */
/*     256-byte aligned sections, suffice).  The faster one on B200.      */
/*   codes: oq_quantize_acts into `workspace`, then oq_qgemm; otherwise,  */
/*     with ws_bytes >= oq_qlinear_workspace(M, d, bits_a).                */
/*   x device [M, d] of dtype; w_idx / w_r from oq_quantize_weights with the */
/*   same plan; workspace device, 256-byte aligned (OQ_ERR_OOM if smaller   */
/*   than both sizes).  Other arguments as in oq_qgemm.                     */
oq_status oq_qlinear(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, const void* x,
                     oq_dtype dtype, int M, const uint8_t* w_idx, const uint16_t* w_r, int N, const uint16_t* bias,
                     uint16_t* y, void* workspace, size_t ws_bytes, void* stream);

/* oq_qlinear with the fp8 variant of the product (oq_qgemm_fp8).          */
oq_status oq_qlinear_fp8(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w, const void* x,
                         oq_dtype dtype, int M, const uint8_t* w_idx, const uint16_t* w_r, int N,
                         const uint16_t* bias, uint16_t* y, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* The full layer without any device allocation.  The paper has no        */
/* counterpart to this call: it exists for callers that may not allocate  */
/* device memory once they are running -- serving processes that reserve  */
/* all device memory at start-up and forbid cudaMalloc/cudaFree on the    */
/* request path (an allocation there can block, fragment the reserve or   */
/* fail under memory pressure), and host code that cannot hold a torch    */
/* allocator.                                                              */
/*   Same arguments and results as oq_qlinear, minus the workspace: the   */
/*   packed activation codes and their norms go to a scratch array that   */
/*   the library reserves statically on every device that loads it        */
/*   (OQ_NOALLOC_SCRATCH_BYTES, 128 MiB, held until the process exits),   */
/*   in the values schedule when its workspace fits there, else in the    */
/*   codes schedule.                                                       */
/*   The schedule is decided before any work: requests that fit neither   */
/*   schedule the code widths allow (values: oq_qlinear_workspace_values; */
/*   codes: oq_qlinear_workspace(M, d, bits_a)) within                     */
/*   OQ_NOALLOC_SCRATCH_BYTES return OQ_ERR_TOO_LARGE, widths no product  */
/*   supports OQ_ERR_UNSUPPORTED, and nothing runs.                        */
/*   Nothing is allocated here: the plan and the activation codebook must */
/*   already have their tables on this device (a plan gets them when      */
/*   created; a codebook on oq_codebook_upload or on its first quantising  */
/*   call on the device), else OQ_ERR_INVALID_ARG.  The weight codebook    */
/*   reaches the product through launch parameters and needs no tables.   */
/*   The first call on a device looks up the scratch array's device       */
/*   address (once per device); make that first call before any stream   */
/*   capture.  All calls share the one array and it keeps the last call's */
/*   contents; every call overwrites the part it reads, so nothing needs  */
/*   clearing.  Calls whose kernels overlap on the GPU (other streams,    */
/*   other host threads) race on the array: order them on one stream.    */
#define OQ_NOALLOC_SCRATCH_BYTES ((size_t)128 << 20)
oq_status oq_qlinear_noalloc(const oq_plan_t* plan, const oq_codebook_t* cb_a, const oq_codebook_t* cb_w,
                             const void* x, oq_dtype dtype, int M, const uint8_t* w_idx, const uint16_t* w_r, int N,
                             const uint16_t* bias, uint16_t* y, void* stream);

/* ---------------------------------------------------------------------- */
/* Device status: reads (and, if `clear`, resets) the current device's     */
/* error flag that kernels set when a bounded wait runs out.  Synchronises */
/* `stream`.  *out receives OQ_OK or OQ_ERR_TIMEOUT.                        */
oq_status oq_device_status(int clear, int* out, void* stream);

/* ---------------------------------------------------------------------- */
/* Test hooks: failures made on the host, so that error handling is tested */
/* without faulting a GPU.  Not for production use.                        */
/*                                                                          */
/* oq_debug_fail_allocations(n): the next n device allocations the library */
/*   makes for its own tables (a plan's gather table, a codebook's lookup   */
/*   table on first use on a device) report failure, so the call returns    */
/*   OQ_ERR_OOM and leaves no partial state; n <= 0 cancels.                */
/* oq_debug_starve(mask): the next launch of each kernel named in `mask`    */
/*   issues none of its input copies, so its bounded waits run out (about   */
/*   one second), it records OQ_ERR_TIMEOUT for oq_device_status() and      */
/*   returns without faulting; the context stays usable.  The output of     */
/*   that launch is undefined.  The call itself still returns OQ_OK.        */
/*   Each call replaces the pending set; mask 0 cancels.                    */
/* oq_debug_rpbh_layout(rows_per_warp, slots, lanes_per_block): the team  */
/*   kernel's work layout -- rows of x per warp (1, 2, */
/*   4 or 8), staging slots per warp team (1 or 2) and lanes per h-block   */
/*   (2: each lane holds half of a block; bf16 inputs, h of 64 or 128) --  */
/*   is forced for the following launches where it fits in shared memory   */
/*   (0 or another value: chosen by the library, the default).  Results do  */
/*   not depend on it except for the rounding order of the row norm's sum  */
/*   and of the butterflies.  For tests and tuning.                         */
/* oq_debug_qgemm_tile_rows(rows): the product with A given as values     */
/*   (oq_qgemm_values, the values schedule) uses tiles of `rows` = 256 or  */
/*   512 rows of A for the following launches (0 or another value: 256,   */
/*   the default).  The result does not depend on it.  For tests and       */
/*   tuning.                                                                */
/* oq_debug_rpbh_kernel(which): the rotate-and-quantise kernel family for  */
/*   plans with h <= 128 in the following launches: 1 the warp-group       */
/*   kernel, 2 the team kernel (whose work layout oq_debug_rpbh_layout     */
/*   forces), 0 or another value: chosen by the library (the warp-group    */
/*   kernel for permuted plans with d <= 8192, else the team kernel).      */
/*   Results do not depend on it except for the rounding order of the row   */
/*   norm's sum.  For tests and tuning.                                     */
#define OQ_STARVE_RPBH 1 /* the rotate-and-quantise kernel (acts and weights) */
#define OQ_STARVE_GEMM 2 /* the codebook-decode GEMM (bf16 and fp8)           */
void oq_debug_fail_allocations(int n);
void oq_debug_starve(int mask);
void oq_debug_rpbh_layout(int rows_per_warp, int slots, int lanes_per_block);
void oq_debug_qgemm_tile_rows(int rows);
void oq_debug_rpbh_kernel(int which);

#ifdef __cplusplus
}
#endif

#endif /* OQ_H */
