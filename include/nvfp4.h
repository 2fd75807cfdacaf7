/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 block-scaled W4A4 linear-layer
 * library.
 *
 * NVFP4 (Replay the Curvature ... NVFP4 Quantization, abstract; ARCQuant blog
 * post, section 1): a tensor of 4-bit E2M1 values in which every 16
 * consecutive values along a row share one E4M3 block scale, under one FP32
 * per-tensor scale.  An element decodes to v(code) * d(block) * s(tensor).
 *
 * Conventions for every entry point
 *  - Pointers marked "device" are CUDA device (or managed) memory owned by the
 *    caller; the library allocates nothing and keeps no state between calls
 *    except the caller-owned workspace described below.
 *  - Calls are asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *    stream).  A return of NVFP4_OK means the work was enqueued.
 *  - Argument errors are detected on the host, before any launch, and returned
 *    synchronously; nothing is enqueued then.
 *  - Data-dependent errors (a NaN/Inf input, a device-side wait that timed out)
 *    are written to `*dev_status` (device int, may be NULL) as an
 *    nvfp4_status value; the first error written sticks.  Zero it before use.
 *  - Row-major matrices; `ld*` arguments are row strides in elements.
 *  - Activations and weights are quantized by the same entry points: weights
 *    are simply quantized once, offline.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad enum value        */
  NVFP4_ERR_ALIGNMENT = 2,   /* pointer or row stride not 16-byte aligned     */
  NVFP4_ERR_UNSUPPORTED = 3, /* valid but not implemented shape/layout combo  */
  NVFP4_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed             */
  NVFP4_ERR_NONFINITE = 5,   /* device: an input element was NaN or Inf       */
  NVFP4_ERR_TIMEOUT = 6,     /* device: a bounded wait gave up                */
  NVFP4_ERR_WORKSPACE = 7    /* workspace missing or smaller than required    */
} nvfp4_status;

typedef enum { NVFP4_F32 = 0, NVFP4_BF16 = 1 } nvfp4_dtype;

/* Block-scale storage.
 *  ROWMAJOR: scale of (row r, block b) at byte r * (cols/16) + b.
 *  TILED:    the 128-row x 4-block atom layout that tcgen05 block-scaled MMAs
 *            consume: rows padded to a multiple of 128, blocks to a multiple
 *            of 4; atom (rt, kt) = rows [128rt, 128rt+128) x blocks [4kt, 4kt+4)
 *            starts at byte (rt * ceil(cols/64) + kt) * 512 and holds
 *            (r, b) at (r % 32) * 16 + ((r / 32) % 4) * 4 + (b % 4).
 *            Padding entries are never written: zero the buffer once after
 *            allocating it. */
typedef enum { NVFP4_SF_ROWMAJOR = 0, NVFP4_SF_TILED = 1 } nvfp4_sf_layout;

/* An NVFP4 matrix of rows x cols (cols a multiple of 16). */
typedef struct {
  uint8_t* codes;        /* device, rows x cols/2 bytes, row-major; element 2j of a
                            row in the low nibble of byte j, element 2j+1 in the
                            high nibble; nibble = sign(bit 3) | E2M1 magnitude   */
  uint8_t* scales;       /* device, E4M3 block scales in sf_layout              */
  float* tensor_scale;   /* device, one FP32 per-tensor scale                   */
  int64_t rows;
  int64_t cols;
  nvfp4_sf_layout sf_layout;
} nvfp4_tensor;

/* Bytes of block-scale storage for a rows x cols NVFP4 matrix. */
size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout);

/* Bytes of workspace the quantizers need for an M x K input (RMSNorm variant
 * included).  The workspace is device memory that must be zero-filled once
 * after allocation; every successful call leaves it zero-filled again.  Calls
 * sharing one workspace must be ordered (same stream).  After a call that
 * reported an error through dev_status, zero it again. */
size_t nvfp4_workspace_size(int64_t M, int64_t K);

/* Quantize X (M x K, dtype dt, row stride ldx) to NVFP4 into q.
 * Definition (ARCQuant post section 1; per-tensor scale as s_aug in section 3.1):
 *   s = scale_in ? *scale_in : fl32(amax|X| / 2688)     (2688 = 6 * 448)
 *   per 16-block: d = E4M3_RNE_satfinite(fl32(amax_block / fl32(6 s)))
 *   per element:  code = E2M1_RNE_satfinite(fl32(x * fl32(1 / fl32(d s))))
 *   (d = 0 or s < 2^-110 gives all-zero magnitudes).  *q->tensor_scale = s.
 * x: device, 16-byte aligned, ldx * sizeof(dt) a multiple of 16; K % 16 == 0.
 * q: rows == M, cols == K; codes 16-byte aligned.
 * scale_in: device float or NULL (NULL = computed from X on the device).
 * workspace: device, >= nvfp4_workspace_size(M, K) bytes (used when
 *            scale_in == NULL).  */
nvfp4_status nvfp4_quantize(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                            const float* scale_in, nvfp4_tensor* q, void* workspace,
                            size_t ws_bytes, int* dev_status, void* stream);

/* ResServe-style full residue (ResServe abstract: an FP4 activation base plus
 * an FP4-quantized residue of what quantization lost):
 *   q = Q(X) as nvfp4_quantize;  R = fl32(X - fl32(fl32(v d) s));
 *   r = Q(R) with its own tensor scale s_R = rscale_in ? *rscale_in
 *       : fl32(amax|R| / 2688).
 * q and r are both M x K.  Other arguments as nvfp4_quantize. */
nvfp4_status nvfp4_quantize_residue(const void* x, nvfp4_dtype dt, int64_t M, int64_t K,
                                    int64_t ldx, const float* scale_in, const float* rscale_in,
                                    nvfp4_tensor* q, nvfp4_tensor* r, void* workspace,
                                    size_t ws_bytes, int* dev_status, void* stream);

/* ARCQuant fused quantizer (ARCQuant post sections 3.1-3.2): RMSNorm, channel
 * reorder, main quantization and residue quantization of the outlier channels
 * in one pass, producing X_aug (M x (K+S)):
 *   y[:,c]  = gamma ? fl32(fl32(x[:,c] * rinv_row) * gamma[c]) : x[:,c]
 *             rinv_row = fl32(1 / sqrt(mean_row(x^2) + eps)), the mean square
 *             formed exactly (squares truncated at 2^-34 of the row's largest
 *             power of two, summed as integers, finished in binary64);
 *   y'[:,j] = y[:, perm[j]]  (perm NULL = identity; outlier channels first);
 *   s_aug   = scale_in ? *scale_in : fl32(amax|y'| / 2688);
 *   X_aug[:, 0..K)    = Q(y') under s_aug;
 *   X_aug[:, K..K+S)  = Q(y'[:, :S] - deq(Q(y'))[:, :S]) under the same s_aug.
 * gamma: device, K elements of dtype dt, or NULL (no normalisation).
 * perm: device int32[K], a permutation of 0..K-1, or NULL.
 * S: 0 <= S <= K, S % 16 == 0.  x_aug: rows == M, cols == K + S.
 * workspace: device, >= nvfp4_workspace_size(M, K) bytes. */
nvfp4_status nvfp4_rmsnorm_reorder_quantize(const void* x, nvfp4_dtype dt, int64_t M, int64_t K,
                                            int64_t ldx, const void* gamma, float eps,
                                            const int32_t* perm, int64_t S, const float* scale_in,
                                            nvfp4_tensor* x_aug, void* workspace, size_t ws_bytes,
                                            int* dev_status, void* stream);

/* Offline weight preparation for the augmented linear (ARCQuant post sections
 * 3.1 and 6.3: the weight takes the activations' channel order and repeats its
 * S outlier columns, so that one GEMM over K+S columns also multiplies the
 * activation residue; OSFP4 page, abstract: a per-channel smoothing vector is
 * absorbed as W diag(sigma) on the weight side and 1/sigma in the RMSNorm gain
 * of the activation side):
 *   W'[:, j] = fl32(W[:, perm[j]] * sigma[perm[j]])   (sigma NULL: W[:, perm[j]])
 *   W_aug    = [W' | W'[:, 0..S)]                      (N x (K+S))
 *   s_w      = scale_in ? *scale_in : fl32(amax|W'| / 2688)
 *   w_aug    = Q(W_aug) under s_w, as nvfp4_quantize (its last S columns repeat
 *              the first S columns' codes and block scales).
 * w: device, N x K of dtype dt, row stride ldw >= K (elements), aligned to
 *   the element size; K % 16 == 0.
 * sigma: device float[K] or NULL; perm: device int32[K], a permutation of
 *   0..K-1, or NULL (identity); an entry outside 0..K-1 is reported as
 *   NVFP4_ERR_INVALID_ARG through dev_status and never indexed.
 * S: 0 <= S <= K, S % 16 == 0.  w_aug: rows == N, cols == K + S, either scale
 *   layout.  workspace: >= nvfp4_workspace_size(N, K) bytes when scale_in is
 *   NULL.  The weight is read with gathers through perm: this is the offline
 *   step, not tuned for speed. */
nvfp4_status nvfp4_quantize_weight(const void* w, nvfp4_dtype dt, int64_t N, int64_t K, int64_t ldw,
                                   const float* sigma, const int32_t* perm, int64_t S, const float* scale_in,
                                   nvfp4_tensor* w_aug, void* workspace, size_t ws_bytes, int* dev_status,
                                   void* stream);

/* Block-scaled W4A4 linear: Y = s_a s_w * A W^T with A (M x K) and W (N x K)
 * NVFP4, fp32 accumulation, output dtype out_dt (row stride ldy).
 * ARCQuant's K -> K+S compensation is this call with K+S columns
 * (ARCQuant post section 3.1-3.2: "unified GEMM call").
 * Kernel choice (K % 64 == 0 always):
 *   ROWMAJOR scales on both operands, M <= 16: CUDA-core decode GEMV (K split
 *     across a cluster of up to 8 CTAs when the activations, expanded to 1.25
 *     bytes per element, do not fit one CTA's shared memory; K up to 71,680
 *     at M = 16, 35,840 with a residue, twice that for each halving of M,
 *     else NVFP4_ERR_UNSUPPORTED);
 *   TILED W scales, M <= 16 (A in either layout): tensor-core decode kernel (W
 *     is the 128-row MMA operand, K split across a thread-block cluster of up
 *     to 8 CTAs), K >= 256;
 *   TILED scales on both operands, 16 < M <= 128: tensor-core few-row kernel,
 *     K >= 256;
 *   TILED scales, M > 128: tensor-core 128x256-tile GEMM, K >= 256.
 *   Other combinations return NVFP4_ERR_UNSUPPORTED.
 * The tensor-core decode and few-row kernels may start before the preceding
 * kernel on `stream` has finished (programmatic dependent launch); they read
 * nothing that kernel produces until it has completed, so stream order is
 * preserved.
 * y: device, aligned to sizeof(out_dt), row stride ldy >= N elements. */
nvfp4_status nvfp4_gemm(const nvfp4_tensor* a, const nvfp4_tensor* w, void* y,
                        nvfp4_dtype out_dt, int64_t ldy, int* dev_status, void* stream);

/* ResServe compensated linear (ResServe abstract):
 *   Y = s_a s_w * A W^T + s_r s_w * R W^T,
 * both products accumulated on-chip and written once.  a and r are M x K (same
 * scale layout), w is N x K.  M <= 128 runs the decode / few-row kernels with
 * a second accumulator fed by the same W tiles; M > 128 (TILED scales) runs the
 * 128x256-tile GEMM with two accumulation passes per tile, A W^T then R W^T,
 * the first held in registers until the second is added.  Other conventions
 * as nvfp4_gemm. */
nvfp4_status nvfp4_gemm_residue(const nvfp4_tensor* a, const nvfp4_tensor* r,
                                const nvfp4_tensor* w, void* y, nvfp4_dtype out_dt, int64_t ldy,
                                int* dev_status, void* stream);

/* Decode linear with online activation quantization, in one kernel launch:
 *   q <- nvfp4_quantize(X, scale_in)            (identical codes, scales, s)
 *   y <- nvfp4_gemm(q, w)                        (same accumulation as above)
 * The ks CTAs of each thread-block cluster together read all of X, agree on
 * s = fl32(amax|X| / 2688) through distributed shared memory and encode their
 * K-slice directly into the MMA operand; q is written as a by-product.  This
 * is the decode step of the pages' pipeline (quantize activations, then the
 * W4A4 GEMM) without the global-memory round trip of Q(X) in between.
 * Requirements: M <= 16, K % 64 == 0, K >= 256, w with TILED scales, and
 * M * K / 8 <= 65536 (bf16) / 32768 (fp32); otherwise NVFP4_ERR_UNSUPPORTED.
 * q: M x K output in either scale layout.  No workspace is needed.  When the
 * activation slice of a CTA does not fit its registers the call runs two
 * launches (one-launch quantizer, then the decode kernel) with identical
 * results.  Other arguments as nvfp4_quantize and nvfp4_gemm. */
nvfp4_status nvfp4_quantize_gemm(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                 const float* scale_in, nvfp4_tensor* q, const nvfp4_tensor* w, void* y,
                                 nvfp4_dtype out_dt, int64_t ldy, int* dev_status, void* stream);

/* nvfp4_quantize_gemm from and to host memory, all on `stream`:
 *   x_dev <- x_host   (M x K dense host rows copied into rows of stride ldx)
 *   nvfp4_quantize_gemm(x_dev, ..., y_dev)
 *   y_host <- y_dev   (M x N: rows of stride ldy copied into dense host rows)
 * x_host and y_host are host pointers (page-locked memory makes the copies
 * asynchronous and lets the call be captured in a CUDA graph); x_dev and y_dev
 * are device buffers the caller owns, with the layouts nvfp4_quantize_gemm
 * takes.  y_host holds the result once `stream` has reached this point.  Every
 * argument is checked before the first copy is issued; errors as
 * nvfp4_quantize_gemm, NVFP4_ERR_CUDA when a copy cannot be issued. */
nvfp4_status nvfp4_quantize_gemm_host(const void* x_host, void* x_dev, nvfp4_dtype dt, int64_t M, int64_t K,
                                      int64_t ldx, const float* scale_in, nvfp4_tensor* q,
                                      const nvfp4_tensor* w, void* y_dev, void* y_host, nvfp4_dtype out_dt,
                                      int64_t ldy, int* dev_status, void* stream);

/* Number of kernel launches nvfp4_quantize_gemm (residue = 0) or
 * nvfp4_quantize_residue_gemm (residue != 0) makes for these sizes on the
 * current device: 1 (quantization fused into the GEMM), 2 (quantize, then the
 * GEMM on the NVFP4 operands, chosen when estimated faster), 0 (unsupported).
 * It launches nothing and reads no device memory; it may initialise the CUDA
 * runtime on the current device (kernel attribute queries). */
int nvfp4_quantize_gemm_plan(int64_t M, int64_t N, int64_t K, nvfp4_dtype dt, int residue, nvfp4_dtype out_dt);

/* ResServe compensated decode linear with online quantization of X and of its
 * residue, in one kernel launch:
 *   (q, r) <- nvfp4_quantize_residue(X, scale_in, rscale_in)
 *   y <- nvfp4_gemm_residue(q, r, w)
 * The residue tensor scale needs a second cluster-wide maximum.  r may be
 * NULL (then this is nvfp4_quantize_gemm).  Requirements and other arguments
 * as nvfp4_quantize_gemm; r has the same shape and scale layout as q. */
nvfp4_status nvfp4_quantize_residue_gemm(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                         const float* scale_in, const float* rscale_in, nvfp4_tensor* q,
                                         nvfp4_tensor* r, const nvfp4_tensor* w, void* y, nvfp4_dtype out_dt,
                                         int64_t ldy, int* dev_status, void* stream);

/* Largest M accepted by nvfp4_rmsnorm_reorder_quantize_noalloc. */
#define NVFP4_NOALLOC_MAX_ROWS 65536

/* nvfp4_rmsnorm_reorder_quantize without a caller workspace, for callers that
 * cannot allocate device memory (hosts that own every allocation, paths that
 * must never call the allocator).  The
 * method's pages have no counterpart: this is a deployment variant of the
 * fused quantizer above, with identical results.
 * Its scratch (reduction cells + one fp32 per row) is a device array inside the
 * library, allocated when the library is loaded and held by every GPU that
 * loads it until the process exits; M > NVFP4_NOALLOC_MAX_ROWS returns
 * NVFP4_ERR_WORKSPACE.  Every call on a device shares that array and finds it
 * as the previous call left it: each call first clears the reduction cells on
 * `stream`, so calls ordered on one stream are safe, while calls that may
 * overlap on the GPU (unordered streams) race on it.  The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current.
 * It calls no allocation routine.  Other arguments and errors as
 * nvfp4_rmsnorm_reorder_quantize. */
nvfp4_status nvfp4_rmsnorm_reorder_quantize_noalloc(const void* x, nvfp4_dtype dt, int64_t M, int64_t K,
                                                    int64_t ldx, const void* gamma, float eps,
                                                    const int32_t* perm, int64_t S,
                                                    const float* scale_in, nvfp4_tensor* x_aug,
                                                    int* dev_status, void* stream);

/* MXFP4 quantization (a NEXT row; ARCQuant post sections 2.2 and 4.2: MX
 * formats use 32-element blocks and E8M0 power-of-two scales, no tensor scale).
 * Scale rule (the pages give none; the MX shared-exponent rule):
 *   per 32-block: b = clamp(floor(log2 amax_block) - 2 + 127, 0, 254), b = 0
 *                 for an all-zero block; scale = 2^(b - 127)
 *   per element:  code = E2M1_RNE_satfinite(x / scale)  (elements in (6, 8) x
 *                 scale clip to 6 x scale)
 * With r_codes != NULL also the residue R = fl32(x - v(code) scale), quantized
 * the same way with its own block scales (ResServe abstract: FP4 base plus FP4
 * residue).
 * x: device, 16-byte aligned, ldx * sizeof(dt) a multiple of 16; K % 32 == 0.
 * codes, r_codes: device, M x K/2 bytes, row-major, 16-byte aligned (element 2j
 *   in the low nibble of byte j of its row).
 * scales, r_scales: device, nvfp4_mx_scales_bytes(M, K, sf_layout) bytes, one
 *   E8M0 byte per block: ROWMAJOR (M x K/32) or TILED (the NVFP4 atom layout
 *   with 32-element blocks: an atom holds 128 rows x 4 blocks = K 128; padding
 *   bytes of a partial atom are left untouched).
 * A NaN/Inf input sets NVFP4_ERR_NONFINITE in *dev_status. */
nvfp4_status nvfp4_mx_quantize(const void* x, nvfp4_dtype dt, int64_t M, int64_t K, int64_t ldx,
                               uint8_t* codes, uint8_t* scales, uint8_t* r_codes, uint8_t* r_scales,
                               nvfp4_sf_layout sf_layout, int* dev_status, void* stream);

/* Bytes of an MXFP4 scale buffer for a rows x cols matrix in `layout`
 * (0 for an empty matrix). */
size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout);

/* MXFP4 W4A4 linear (ARCQuant post section 2.2: the MX block-scaled format on
 * the same tensor cores): Y = deq(A) deq(W)^T, A = (a_codes, a_scales) M x K,
 * W = (w_codes, w_scales) N x K, both quantized by nvfp4_mx_quantize with
 * TILED scales; fp32 accumulation of the exact block products, output dtype
 * out_dt with row stride ldy >= N.  One tensor-core kernel (128 x 256 tiles,
 * kind::mxf4, one scale byte per 32 elements).
 * Requirements: K % 128 == 0, K >= 256 (else NVFP4_ERR_UNSUPPORTED); codes and
 * scales 16-byte aligned; y aligned to sizeof(out_dt).  The caller owns every
 * buffer; nothing is allocated. */
nvfp4_status nvfp4_mx_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w_codes,
                           const uint8_t* w_scales, int64_t M, int64_t N, int64_t K, void* y,
                           nvfp4_dtype out_dt, int64_t ldy, int* dev_status, void* stream);

/* MXFP4 compensated linear (ResServe abstract: FP4 base plus FP4 residue; its
 * largest gains are reported for MXFP4): Y = deq(A) deq(W)^T + deq(R) deq(W)^T,
 * with (r_codes, r_scales) the residue from nvfp4_mx_quantize (TILED scales).
 * MX has no tensor scales, so the residue's K-tiles continue the same fp32
 * accumulation, Y = [A | R] [W | W]^T, written once.  Requirements and
 * conventions as nvfp4_mx_gemm; r_codes and r_scales must not be NULL. */
nvfp4_status nvfp4_mx_gemm_residue(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* r_codes,
                                   const uint8_t* r_scales, const uint8_t* w_codes, const uint8_t* w_scales,
                                   int64_t M, int64_t N, int64_t K, void* y, nvfp4_dtype out_dt, int64_t ldy,
                                   int* dev_status, void* stream);

/* Test support for the device-side bounded waits (failure detection around
 * the method; the pages have no counterpart).  Every mbarrier wait of the
 * tensor-core kernels (nvfp4_gemm, nvfp4_gemm_residue, the fused decode
 * linears, the MXFP4 GEMMs) gives up after limit_ns nanoseconds (default 4 s;
 * 0 restores it), records NVFP4_ERR_TIMEOUT in *dev_status and lets the launch
 * finish: each CTA first lets its own bulk copies and MMAs in flight and the
 * bytes its cluster peers send complete, then releases its tensor memory and
 * exits, so the context stays usable.  withhold != 0 makes those kernels skip
 * loading their weight tiles (the large-M GEMM: every operand tile), so that
 * their waits run out: a way to exercise the timeout path that faults nothing.
 * Output contents of a launch that timed out are unspecified.  The setting is
 * process wide, read when a launch is made, and meant for tests only. */
void nvfp4_test_wait_fault(uint64_t limit_ns, int withhold);

/* Human-readable name of a status code (static string). */
const char* nvfp4_status_string(nvfp4_status status);

/* Library version and target, e.g. "nvfp4 0.1 sm_100a" (static string). */
const char* nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
