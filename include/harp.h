/*
 * harp.h -- C ABI of libharp: HARP's structured orthogonal processor fused
 * with a group-wise low-bit quantizer, on one NVIDIA B200 (sm_100a).
 *
 * What it computes (the pages' titles and sections):
 *  - HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme
 *    LLM Quantization (gist.science, paper 2605.29843), section 2.1: a
 *    processor on R^d is a product of m stride stages with mixed radices
 *    b_0 .. b_{m-1}, prod b_t = d; stage t applies one b_t x b_t orthogonal
 *    block to each group of coordinates that a stride permutation separates.
 *    Section 2.2: blocks B = Q(theta) G_b, G_b a normalised Sylvester
 *    Hadamard (b = 2^k) or the Q factor of a fixed Gaussian; theta = 0 gives
 *    the fixed randomized Hadamard transform (random signs, then Hadamard).
 *    Sections 3 and 5: two-sided on weights (W' = U^T W V), one-sided on
 *    activations; an exact change of basis, undone by the transpose.
 *  - PolarQuant: Optimal Gaussian Weight Quantization via Hadamard Rotation
 *    for LLM Compression (gist.science, paper 2603.29078), section 2:
 *    rotated groups scaled to N(0,1) and coded with Lloyd-Max centroids;
 *    fp16 group scale, fp32 centroid table; section 1: the absmax uniform
 *    quantizer on [-alpha, alpha].
 *
 * Conventions fixed by this library where the pages leave them open:
 *  - Index convention. s_t = b_{t+1} * ... * b_{m-1} (s_{m-1} = 1). Stage t's
 *    group c = h*s_t + l (0 <= l < s_t) holds the coordinates
 *    h*b_t*s_t + k*s_t + l, k = 0 .. b_t-1, and
 *        y[h b s + k s + l] = sum_j B_{t,c}[k][j] * x[h b s + j s + l].
 *    The processor is M = B_{m-1} ... B_1 B_0 D_s: the sign vector first,
 *    then stage 0 (largest stride). Its inverse is D_s B_0^T ... B_{m-1}^T.
 *  - Sides. HARP_RIGHT maps every row r of a [rows x cols] matrix to M r
 *    (d = cols; X -> X V with V = M^T). HARP_LEFT maps every column w to M w
 *    (d = rows; W -> U^T W with U = M^T). Two-sided: W' = M_L W M_R^T.
 *  - Quantizer groups are `group` consecutive columns of a row of the rotated
 *    matrix. Lloyd-Max: s = sqrt(mean(x^2)) over the group (or, with
 *    HARP_SCALE_ABSMAX, max|x| / c_{K-1}); code = number of
 *    fp32 midpoints t_k (of neighbouring fp32 centroids) with x/s > t_k.
 *    Absmax: s = max|x| / (2^(b-1) - 1); code = clamp(rint(x/s), -qmax, qmax)
 *    + 2^(b-1), so 4-bit codes are 1..15. Scales are stored as IEEE fp16
 *    (round to nearest even, saturating at 65504) and codes are computed
 *    with the stored scale. A group whose stored scale is 0 gets the middle
 *    code (2^(b-1)) and dequantizes to 0.
 *  - Packing: code i of a row occupies bits [b*i, b*i + b) of that row's
 *    little-endian bitstream (first code in the low bits of byte 0); rows of
 *    `codes` are cols*b/8 bytes apart. Scales are a separate [rows x
 *    cols/group] fp16 array.
 *
 * Memory and errors:
 *  - All tensor pointers passed to compute calls are DEVICE pointers owned by
 *    the caller (e.g. torch tensors) unless a parameter says "host". Compute
 *    calls are asynchronous on the given CUDA stream (NULL = legacy default
 *    stream) and never synchronise; the library allocates no device memory
 *    after plan creation.
 *  - Every call returns a harp_status (0 = HARP_OK). Arguments are checked on
 *    the host before any launch; a rejected call launches nothing and leaves
 *    outputs untouched. A compute call on an empty matrix (rows or cols 0)
 *    checks its plan, codebook and shapes, then returns HARP_OK without
 *    touching any pointer. Kernels never trap or assert. HARP_ERR_CUDA reports a
 *    launch error (cudaGetLastError after the launch); asynchronous execution
 *    errors surface at the caller's next synchronisation.
 *  - There is no CPU fallback: without a CUDA device, plan creation returns
 *    HARP_ERR_CUDA.
 */
#ifndef HARP_H_
#define HARP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum harp_status {
    HARP_OK = 0,
    HARP_ERR_INVALID_ARG = 1,   /* NULL where a pointer is required, bad enum value */
    HARP_ERR_SHAPE = 2,         /* prod b_t != d, d != rows/cols, group does not divide cols, ... */
    HARP_ERR_UNSUPPORTED = 3,   /* radix outside [1, 64], more than 16 stages, bits not in {2,3,4,5} */
    HARP_ERR_ALIGNMENT = 4,     /* device pointer or leading dimension not aligned (see each call) */
    HARP_ERR_WORKSPACE = 5,     /* workspace NULL or smaller than harp_workspace_size() */
    HARP_ERR_CUDA = 6,          /* CUDA runtime error (no device, launch failure) */
    HARP_ERR_ALLOC = 7          /* host or device allocation failed at plan / codebook creation */
} harp_status;

enum harp_dtype { HARP_F32 = 0, HARP_BF16 = 1, HARP_F16 = 2 /* harp_requantize's restored weights only */ };
enum harp_side { HARP_RIGHT = 0, HARP_LEFT = 1 };
enum harp_dir { HARP_FWD = 0, HARP_INV = 1 };
enum harp_quant_kind { HARP_LLOYD_MAX = 0, HARP_ABSMAX = 1 };
enum harp_block_kind { HARP_BLOCKS_HADAMARD = 0, HARP_BLOCKS_QR = 1, HARP_BLOCKS_CAYLEY = 2 };

#define HARP_MAX_STAGES 16
#define HARP_MAX_RADIX 64

typedef struct harp_plan_s *harp_plan_t;
typedef struct harp_codebook_s *harp_codebook_t;

/* Human-readable name of a status code (static storage; never NULL). */
const char *harp_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int harp_version(void);

/* --------------------------------------------------------------- plan objects */

/* Create a processor plan on the current CUDA device  [HARP 2.1, 2.2].
 *  d      vector length the processor acts on (cols for HARP_RIGHT, rows for
 *         HARP_LEFT), 1 <= d <= 2^31 - 1.
 *  m      number of stages, 1 <= m <= HARP_MAX_STAGES.
 *  radix  host [m]; each b_t in [1, HARP_MAX_RADIX]; prod b_t must equal d.
 *  blocks host [m] pointers; blocks[t] points to d/b_t row-major b_t x b_t
 *         float blocks (block c at offset c*b_t*b_t, entry [k][j] = output
 *         k, input j). The blocks are used as given; forward and inverse are
 *         exact inverses only if they are orthogonal.
 *  signs  host [d] of +1/-1 (any float is accepted and multiplied in), or
 *         NULL for all +1.
 *  stream CUDA stream the copies to device memory are ordered on (NULL =
 *         legacy default stream).
 * The plan copies blocks and signs to device memory and owns that copy until
 * harp_plan_destroy. The copies run on `stream` and are complete when the
 * call returns (it synchronises that stream), so the caller may release its
 * host arrays at once and launches on any stream may use the plan. Errors:
 * INVALID_ARG (NULL out/radix/blocks), UNSUPPORTED, SHAPE, CUDA, ALLOC. */
int harp_plan_create(harp_plan_t *out, int64_t d, int m, const int32_t *radix,
                     const float *const *blocks, const float *signs, void *stream);

/* Release a plan and its device memory. NULL is accepted. The caller must
 * ensure no launch that uses the plan is still running. */
int harp_plan_destroy(harp_plan_t plan);

/* Read back a plan's shape: d, m and radix (host [HARP_MAX_STAGES]); any
 * output pointer may be NULL. */
int harp_plan_info(harp_plan_t plan, int64_t *d, int *m, int32_t *radix);

/* Build one stage's blocks from raw Gaussian draws, on the host, in double
 * precision, rounded to float  [HARP 2.1, 2.2]:
 *  HARP_BLOCKS_HADAMARD  every group gets the base mixer G_b: the normalised
 *                        Sylvester Hadamard if b is a power of two, else the
 *                        Q factor (positive R diagonal) of `base_gauss`.
 *  HARP_BLOCKS_QR        group c gets the Q factor (positive R diagonal) of
 *                        gauss[c] (a random orthogonal block).
 *  HARP_BLOCKS_CAYLEY    group c gets Q_c G_b, with Q_c the Cayley map
 *                        (I - A)^-1 (I + A) of A = skew_scale * S_c, S_c the
 *                        skew-symmetric matrix whose strict upper triangle is
 *                        gauss[c]'s; for b = 2, Q_c is the Givens rotation
 *                        [[cos a, -sin a], [sin a, cos a]], a =
 *                        skew_scale * gauss[c][0][1]. skew_scale = 0 gives
 *                        back G_b exactly.
 *  gauss      host [n_groups][b][b] doubles (ignored for HADAMARD), row-major.
 *  base_gauss host [b][b] doubles, needed only when b is not a power of two
 *             and kind != QR.
 *  out        host [n_groups][b][b] floats.
 * Errors: INVALID_ARG, UNSUPPORTED (b outside [1, 64]), SHAPE (singular
 * input). */
int harp_stage_blocks(int kind, int b, int64_t n_groups, const double *gauss,
                      const double *base_gauss, double skew_scale, float *out);

/* Build one stage's blocks on the device from int8-stored parameters
 * [HARP 2.2 (B = Q(theta) G_b; Givens for b = 2, Cayley for b > 2),
 *  HARP 2.4 (parameters stored in int8)]:
 *    B_c = Q(theta_c) G_b,  theta = theta_scale * q.
 *  b = 2: Q = [[cos a, -sin a], [sin a, cos a]], a = theta_c (one value).
 *  b > 2: Q = (I - A)^-1 (I + A), A skew-symmetric whose strict upper
 *         triangle, read row by row ((0,1), (0,2), ..., (0,b-1), (1,2), ...),
 *         is theta_c's b(b-1)/2 values.
 *  b = 1: B = [1].
 * Computed in double precision on the device, rounded once to float. Every q
 * = 0 gives G_b exactly.
 *  b            1..HARP_MAX_RADIX.
 *  theta        device int8 [n_groups][P], P = b(b-1)/2 (1 for b = 2, 0 for
 *               b = 1; may be NULL then).
 *  theta_scale  the stage's scale (finite).
 *  base         device float [b][b] row-major G_b, required when b is not a
 *               power of two; NULL = the normalised Sylvester matrix
 *               (-1)^popcount(k & j) / sqrt(b).
 *  out          device float [n_groups][b][b] row-major (out k, in j),
 *               4-byte aligned.
 * Stream-ordered and asynchronous. Errors: INVALID_ARG (NULL pointer,
 * non-finite scale, missing base), UNSUPPORTED (b outside [1, 64]),
 * ALIGNMENT, CUDA. */
int harp_theta_blocks(int b, int64_t n_groups, const int8_t *theta, float theta_scale,
                      const float *base, float *out, void *stream);

/* Replace stage `stage` of a plan with the blocks harp_theta_blocks builds
 * from (theta, theta_scale, base), on the device and in the plan's own
 * layouts (the plan's radix b = radix[stage], n_groups = d / b). Stream-
 * ordered: launches on `stream` before this call use the old blocks, later
 * ones the new; launches on other streams must be ordered by the caller. The
 * stage is afterwards applied by general block arithmetic (never the
 * Walsh-Hadamard butterfly), also when every q is 0.
 * Must be called with the plan's device current.
 * Errors: INVALID_ARG (NULL plan or pointer, stage outside [0, m), non-finite
 * scale, missing base, another device current), CUDA. */
int harp_plan_load_theta(harp_plan_t plan, int stage, const int8_t *theta, float theta_scale,
                         const float *base, void *stream);

/* Lloyd-Max centroids for N(0,1) with 2^bits levels  [PolarQuant 2], computed
 * on the host (double precision, rounded to float): ascending, odd-symmetric.
 * out: host [2^bits]. bits in {2, 3, 4, 5} (5 = PolarQuant's Q5). */
int harp_lloyd_max_centroids(int bits, float *out);

/* Create a quantizer description  [PolarQuant 1, 2].
 *  kind        HARP_LLOYD_MAX or HARP_ABSMAX.
 *  bits        2, 3, 4 or 5 (PolarQuant section 3 uses 5-bit Q5 codes).
 *  group       elements per scale group along a row: a positive multiple of
 *              32 (UNSUPPORTED otherwise); must divide cols at each call
 *              (group = cols gives one scale per row).
 *  scale_mode  how a Lloyd-Max group is scaled to N(0,1):
 *              HARP_SCALE_RMS (default): s = sqrt(mean(x^2)) over the group
 *              (PolarQuant section 2: l2-normalise, then scale to unit
 *              variance); HARP_SCALE_ABSMAX: s = max|x| / c_{K-1}, the
 *              group's largest magnitude onto the outermost centroid. Absmax
 *              codebooks always use s = max|x| / (2^(b-1) - 1) and accept
 *              either value.
 *  centroids   host [2^bits] ascending floats for HARP_LLOYD_MAX, or NULL
 *              for the built-in N(0,1) Lloyd-Max table; ignored for absmax.
 * Host-only object (no device memory); the tables travel as kernel arguments.
 * Errors: INVALID_ARG (NULL out, unknown kind or scale_mode, centroids not
 * strictly ascending, or a non-positive largest centroid with
 * HARP_SCALE_ABSMAX), UNSUPPORTED, ALLOC. */
enum harp_scale_mode { HARP_SCALE_RMS = 0, HARP_SCALE_ABSMAX = 1 };
int harp_codebook_create(harp_codebook_t *out, int kind, int bits, int64_t group, int scale_mode,
                         const float *centroids);
int harp_codebook_destroy(harp_codebook_t cb);

/* Copy a codebook's fp32 tables to host memory: centroids [2^bits] (absmax:
 * the integer levels code - 2^(b-1)) and thresholds [2^bits - 1]; either may
 * be NULL. */
int harp_codebook_tables(harp_codebook_t cb, float *centroids, float *thresholds);

/* Bytes of device workspace the fused two-sided calls need for a
 * [rows x cols] matrix: rows*cols*8 (two fp32 intermediates, between which
 * the passes of the two-sided path alternate) when `left` is not NULL,
 * else 0. */
int harp_workspace_size(harp_plan_t left, harp_plan_t right, int64_t rows, int64_t cols,
                        size_t *bytes);

/* ------------------------------------------------------------ compute calls */

/* Apply a processor to the rows (HARP_RIGHT, plan d = cols) or the columns
 * (HARP_LEFT, plan d = rows) of a row-major matrix, forward (M) or inverse
 * (M^T)  [HARP 2.1; 5].
 *  in, out      device; element [r][c] at r*ld + c; in_dtype / out_dtype are
 *               HARP_F32 or HARP_BF16 (bf16 output rounds to nearest even).
 *               in and out must not overlap.
 *  ld_in/ld_out leading dimensions in elements, >= cols, multiples of 4.
 *  Alignment: in and out 16-byte aligned.
 * Arithmetic is fp32 with fp32 blocks. */
int harp_rotate(harp_plan_t plan, int side, int dir, const void *in, int in_dtype,
                void *out, int out_dtype, int64_t rows, int64_t cols, int64_t ld_in,
                int64_t ld_out, void *stream);

/* Group-wise quantize an (already rotated) row-major matrix  [PolarQuant 2].
 *  in      device [rows x cols], leading dimension ld_in (multiple of 4).
 *  codes   device [rows x cols*bits/8] bytes (cols*bits % 8 == 0; packed as
 *          described above); scales device [rows x cols/group] fp16 bits.
 *  Alignment: in 16 bytes, codes 4 bytes, scales 2 bytes. */
int harp_quantize(harp_codebook_t cb, const void *in, int in_dtype, int64_t rows,
                  int64_t cols, int64_t ld_in, uint8_t *codes, uint16_t *scales,
                  void *stream);

/* Inverse of harp_quantize: out[r][c] = s * centroid[code] (Lloyd-Max) or
 * s * (code - 2^(b-1)) (absmax)  [PolarQuant 2]. out: device, ld_out >= cols,
 * multiple of 4, 16-byte aligned. */
int harp_dequantize(harp_codebook_t cb, const uint8_t *codes, const uint16_t *scales,
                    int64_t rows, int64_t cols, void *out, int out_dtype, int64_t ld_out,
                    void *stream);

/* Fused forward path: W' = M_L W M_R^T (left may be NULL for right-only),
 * then group-wise quantize and pack W'  [HARP 2.1, 3; PolarQuant 2].
 *  in           device [rows x cols], contiguous (ld = cols), F32 or BF16.
 *  codes/scales as in harp_quantize.
 *  rotated_out  optional device fp32 [rows x cols] copy of W' (NULL = none).
 *  workspace    device, >= harp_workspace_size bytes, 16-byte aligned
 *               (may be NULL when the size is 0).
 * right->d must equal cols and left->d rows. */
int harp_rotate_quantize(harp_plan_t left, harp_plan_t right, harp_codebook_t cb,
                         const void *in, int in_dtype, int64_t rows, int64_t cols,
                         uint8_t *codes, uint16_t *scales, float *rotated_out,
                         void *workspace, size_t ws_bytes, void *stream);

/* PolarQuant's two-stage codec, fused [PolarQuant 2 (codes, fp16 norm,
 * H^-1 = H), 3 (Q5 weights restored to FP16, then a downstream absmax INT4
 * quantizer)]: for every row,
 *     restored = round_mid( D_s B_0^T ... B_{m-1}^T dequant_in(codes_in) )
 *     (codes_out, scales_out) = quantize_out(restored)     (no rotation)
 * i.e. harp_dequantize_unrotate (right side only) into the storage type
 * `mid_dtype`, then harp_quantize with `cb_out`, in one pass over the matrix.
 *  right        the first stage's row processor; right->d == cols.
 *  cb_in        the first stage's codebook (any kind, 2..5 bits).
 *  codes_in, scales_in  device, laid out as harp_quantize writes them.
 *  mid_dtype    HARP_F32, HARP_BF16 or HARP_F16: each restored value is
 *               rounded to nearest even in this type (fp16 saturating at
 *               +-65504) before the second quantizer sees it.
 *  restored_out optional device [rows x cols] contiguous array of
 *               `mid_dtype` receiving the restored weights (NULL = none).
 *  cb_out       the second codebook (e.g. HARP_ABSMAX, 4 bits, group 128).
 *  codes_out, scales_out  device, as harp_quantize writes them for cb_out.
 * Both groups must divide cols. Alignment: codes 4 bytes, scales 2 bytes,
 * restored_out 16 bytes. Errors: INVALID_ARG, SHAPE, UNSUPPORTED (a row of
 * `cols` values does not fit the kernel's shared-memory tile), ALIGNMENT,
 * CUDA. */
int harp_requantize(harp_plan_t right, harp_codebook_t cb_in, const uint8_t *codes_in,
                    const uint16_t *scales_in, int64_t rows, int64_t cols, int mid_dtype,
                    void *restored_out, harp_codebook_t cb_out, uint8_t *codes_out,
                    uint16_t *scales_out, void *stream);

/* Fused inverse path: dequantize, then W = M_L^T W' M_R  [HARP 5;
 * PolarQuant 2]. out: device [rows x cols] contiguous, F32 or BF16.
 * Workspace as for harp_rotate_quantize. */
int harp_dequantize_unrotate(harp_plan_t left, harp_plan_t right, harp_codebook_t cb,
                             const uint8_t *codes, const uint16_t *scales, int64_t rows,
                             int64_t cols, void *out, int out_dtype, void *workspace,
                             size_t ws_bytes, void *stream);

/* ------------------------------------------------ host-buffer variants */

/* The fused calls for callers whose data live in host memory: each copies
 * its inputs from host buffers into a caller-provided device scratch,
 * runs the device call there, and copies its outputs back into host
 * buffers. Copies (one cudaMemcpyAsync per buffer) and kernels are ordered
 * on `stream` and the call returns once they are enqueued: the host buffers
 * must stay valid and unchanged until the stream has passed them
 * (synchronise the stream before reading the outputs). Pinned (page-locked)
 * host buffers make the copies asynchronous; pageable ones also work, with
 * the CUDA runtime's staging. Nothing is allocated.
 *
 * Scratch layout (each part 256-byte aligned): values (rows*cols elements
 * of the value dtype: the input of the forward, the output of the inverse),
 * packed codes, fp16 scales, then the workspace of harp_workspace_size.
 * harp_host_scratch_size gives the bytes for a call's shapes and value
 * dtype (HARP_BF16 or HARP_F32). Errors: those of the device call, plus
 * INVALID_ARG (NULL host buffer with rows, cols > 0; value dtype not bf16 /
 * f32) and WORKSPACE (dev_scratch NULL or smaller than the size). */
int harp_host_scratch_size(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int64_t rows,
                           int64_t cols, int value_dtype, size_t *bytes);

/* harp_rotate_quantize with host `in` (rows x cols, in_dtype, row-major) and
 * host outputs `codes` (rows * cols * bits / 8 bytes) and `scales`
 * (rows * cols / group fp16 values)  [HARP 3; PolarQuant 2]. */
int harp_rotate_quantize_host(harp_plan_t left, harp_plan_t right, harp_codebook_t cb,
                              const void *in, int in_dtype, int64_t rows, int64_t cols,
                              uint8_t *codes, uint16_t *scales, void *dev_scratch,
                              size_t scratch_bytes, void *stream);

/* harp_dequantize_unrotate with host `codes` and `scales` and host output
 * `out` (rows x cols, out_dtype HARP_BF16 or HARP_F32)  [PolarQuant 2;
 * HARP 5]. */
int harp_dequantize_unrotate_host(harp_plan_t left, harp_plan_t right, harp_codebook_t cb,
                                  const uint8_t *codes, const uint16_t *scales, int64_t rows,
                                  int64_t cols, void *out, int out_dtype, void *dev_scratch,
                                  size_t scratch_bytes, void *stream);

/* ------------------------------------------------------------ timing hooks */

/* Number of kernel launches (passes) harp_rotate_quantize and
 * harp_dequantize_unrotate make for this pair of processors and codebook
 * when both sides are given; 0 when they fall back to one launch per side.
 * Host-only. */
int harp_pass_count(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int *passes);

/* FMAs per matrix element that pass `pass` (0-based, forward order) of the
 * two-sided plan spends: the sum of the radices of the stages it applies
 * (pass np-1-k of the inverse call applies the same stages). Host-only.
 * Errors: INVALID_ARG (NULL argument, no pass plan, pass out of range). */
int harp_pass_fma(harp_plan_t left, harp_plan_t right, harp_codebook_t cb, int pass, int *fma);

/* Register CUDA events (cudaEvent_t handles, owned by the caller and kept
 * alive while registered) for timing the passes of the fused two-sided
 * calls made afterwards by the calling thread: each such call records
 * events[0] on its stream before its first pass and events[k+1] after pass k
 * (for k + 1 < n). n = 0 unregisters. No effect on results. Errors:
 * INVALID_ARG (n < 0, or NULL events with n > 0). */
int harp_set_pass_events(void *const *events, int n);

/* ------------------------------------------------------------ diagnostics */

/* Which arithmetic the two-sided calls' block stages use (process-wide; a
 * tuning and testing switch, results agree within the fp32 tolerance):
 *  HARP_BLOCK_STAGES_AUTO  per pass, tensor cores (tcgen05.mma kind::tf32
 *                          with split operands, "3xTF32": each product
 *                          x*b as x_hi*b_hi + x_lo*b_hi + x_hi*b_lo in fp32)
 *                          when a block of the pass is wider than 32, else
 *                          fp32 FMAs (the faster of the two measured on the
 *                          B200 for each width);
 *  HARP_BLOCK_STAGES_TC    tensor cores for every block stage;
 *  HARP_BLOCK_STAGES_FFMA  fp32 FMAs for every block stage.
 * Stages whose blocks are all normalised Sylvester matrices always run as
 * Walsh-Hadamard butterflies. Takes effect for calls made afterwards.
 * Errors: INVALID_ARG (unknown mode). */
enum harp_block_stages { HARP_BLOCK_STAGES_AUTO = 0, HARP_BLOCK_STAGES_TC = 1, HARP_BLOCK_STAGES_FFMA = 2 };
int harp_set_block_stages(int mode);

/* Every wait inside the library's kernels is bounded (the tensor-core stages
 * of the two-sided kernels wait for their MMA batches for about half a
 * second at most); a wait that runs out abandons the launch without trapping
 * and is recorded per device. This call returns that record for the current
 * device in *flags and clears it: 0 = no wait ran out; bit 0 = a tensor-core
 * batch of a two-sided call did not complete; bit 1 = a bulk copy of a
 * two-sided call's operand blocks or input did not arrive; bit 2 = a row
 * tile of a right-only call did not arrive (those calls' outputs are
 * incomplete). Synchronous (it waits for the device's pending work).
 * Errors: INVALID_ARG (NULL flags), CUDA. */
int harp_fault_status(unsigned int *flags);

/* ------------------------------------------- variant that allocates nothing */

/* Capacity of the library-owned scratch used by harp_rotate_quantize_static:
 * 32 MiB, i.e. a two-sided matrix of up to 4,194,304 elements (for example
 * 2048 x 2048 or 1024 x 4096; harp_workspace_size gives the need). */
#define HARP_STATIC_WORKSPACE_BYTES ((size_t)32 << 20)

/* harp_rotate_quantize without a caller workspace. The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory: code hosted by a framework that owns every device byte (a pool
 * reserved at start-up that rejects further requests) and code on a
 * latency-critical path where cudaMalloc, which may synchronise the device,
 * is not allowed. Such callers still pass their own input and outputs.
 *
 * Arguments and results are those of harp_rotate_quantize (same checks, same
 * kernels, identical output); the fp32 intermediate of the two-sided path
 * lives instead in a file-scope device array of HARP_STATIC_WORKSPACE_BYTES
 * inside the library, which every device that loads the library holds until
 * the process exits. The call allocates no memory (no cudaMalloc / cudaFree,
 * no allocating library routine).
 *  - Size limit: a workspace need (harp_workspace_size, rows*cols*8 bytes) above
 *    HARP_STATIC_WORKSPACE_BYTES returns HARP_ERR_WORKSPACE before anything
 *    is launched. Right-only calls (left = NULL) need no scratch.
 *  - Set-up: the first two-sided call on a device looks up the array's
 *    device address (cudaGetSymbolAddress, with that device current) and
 *    caches it; make that first call before any stream capture.
 *  - Sharing: every call on a device uses the same array, which keeps the
 *    last call's contents. Each call overwrites every element it reads
 *    before reading it, so nothing needs clearing, but calls that can
 *    overlap on the GPU (different streams, no ordering between them) race
 *    on the array and corrupt each other's results: serialise them.
 * Errors: those of harp_rotate_quantize, plus HARP_ERR_WORKSPACE (too large),
 * HARP_ERR_CUDA (no device, address lookup failed) and HARP_ERR_UNSUPPORTED
 * (device ordinal above 63). */
int harp_rotate_quantize_static(harp_plan_t left, harp_plan_t right, harp_codebook_t cb,
                                const void *in, int in_dtype, int64_t rows, int64_t cols,
                                uint8_t *codes, uint16_t *scales, float *rotated_out,
                                void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HARP_H_ */
