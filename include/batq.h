/*
 * libbatq -- BATQuant W4A4 MXFP4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The method: BATQuant (arXiv 2603.16590), "BATQuant: Outlier-resilient MXFP4
 * Quantization via Learnable Block-wise Optimization".  Before every linear
 * layer each 32-element MXFP block x_i of a token is transformed by a
 * block-wise affine matrix P_i = B_i (x) A (Global-Private Kronecker
 * decomposition: one 8x8 A shared by all blocks, one private 4x4 B_i per
 * block), clipped to [sigma(a_i_min) min, sigma(a_i_max) max] and quantized to
 * MXFP4; the weight-side inverse transform is fused into the weights offline.
 *   - block-wise affine transform, GPK: daily-arxiv summary page
 *     (zhaoyang97.github.io), sections "块仿射变换 (BAT)" and "GPK 分解";
 *     gist.science technical summary, sections 2.A and 2.B.
 *   - clip: daily-arxiv summary, section "块级可学习裁剪"; gist.science 2.C.
 *   - weights fused offline, activation transform + clip online:
 *     thelatestinai.com page, Figure 3 caption; gist.science 2.D.
 *   - cost of the activation transform O(SN(g1+g2)): thelatestinai.com
 *     page, Table 1.
 *   - MXFP4 rules (E8M0 shared scale 2^(floor(log2 amax) - 2), E2M1 elements
 *     rounded to nearest even and saturated at +-6): OCP Microscaling
 *     Formats v1.0; the pages state the 32-element shared E8M0 scale and the
 *     divide-then-round order (thelatestinai.com page, Figure 2 caption).
 *
 * Conventions for every call:
 *   - All pointers named *_dev, and X / W / codes / scales / out / workspace,
 *     are DEVICE pointers owned by the caller.  The library never allocates
 *     device memory and never synchronises on the compute calls.
 *   - Pointers named *_host are host pointers, read during the call only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Compute calls are asynchronous and stream-ordered.
 *   - Every call returns a batq_status.  Argument, shape, alignment and
 *     architecture errors are reported before anything is launched; a failed
 *     launch returns BATQ_ERR_CUDA.  No call aborts or prints.
 *   - Matrices are row-major.  S = tokens, N = in-features (= K), M =
 *     out-features, k = N / 32 blocks per row.
 *   - Codes: two E2M1 codes per byte, element 2j in the low nibble; code =
 *     sign << 3 | magnitude (0, 0.5, 1, 1.5, 2, 3, 4, 6).  A row of N
 *     elements takes N/2 bytes; rows are packed (row stride N/2 bytes).
 *   - Scales: one E8M0 byte (2^(byte - 127)) per row and 32-block.
 *     BATQ_SCALES_LINEAR: rows x k bytes, row-major.
 *     BATQ_SCALES_MMA: the tiled layout the block-scaled tensor-core MMA
 *     consumes: rows padded to a multiple of 128 and k to a multiple of 4;
 *     byte (r, c) at ((r/128)*(kpad/4) + c/4)*512 + (r%32)*16 + ((r/32)%4)*4
 *     + c%4.  Padding bytes are written as 0x7F.
 *   - An all-zero block gets scale byte 0x00; a block holding a non-finite
 *     transformed value gets 0xFF and zero codes.
 */
#ifndef BATQ_H
#define BATQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BATQ_API __attribute__((visibility("default")))
#else
#define BATQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BATQ_OK = 0,
  BATQ_ERR_INVALID_ARG = 1, /* null pointer, bad enum, negative size */
  BATQ_ERR_SHAPE = 2,       /* N % 64 != 0, S < 1, M % 16 != 0, ld < row length, rows x N/32 >= 2^31 */
  BATQ_ERR_ALIGNMENT = 3,   /* a device pointer or row stride not 16-byte aligned */
  BATQ_ERR_SINGULAR = 4,    /* A or some B_i singular / condition number > 1e8 */
  BATQ_ERR_ARCH = 5,        /* current device is not sm_100 */
  BATQ_ERR_CUDA = 6,        /* a CUDA runtime / driver call failed */
  BATQ_ERR_TIMEOUT = 7,     /* a kernel gave up waiting on a barrier (device error word set) */
  BATQ_ERR_WORKSPACE = 8,   /* workspace too small */
  BATQ_ERR_SCRATCH_LIMIT = 9 /* problem needs more scratch than batq_linear_no_alloc's fixed array */
} batq_status;

/* Size of the fixed device scratch array used by batq_linear_no_alloc (16 MiB). */
#define BATQ_NO_ALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

typedef enum { BATQ_F32 = 0, BATQ_BF16 = 1 } batq_dtype;

typedef enum { BATQ_SCALES_LINEAR = 0, BATQ_SCALES_MMA = 1 } batq_scale_layout;

/* Text for a status code (static storage). */
BATQ_API const char* batq_status_string(batq_status status);

/* Library version, major*10000 + minor*100 + patch. */
BATQ_API int batq_version(void);

/*
 * Bytes needed for the MXFP4 codes and scales of a rows x N matrix in the
 * given scale layout (same for activations, rows = S, and weights, rows = M).
 * Host only; no CUDA call.
 */
BATQ_API batq_status batq_act_buffer_sizes(int rows, int N, batq_scale_layout layout,
                                  size_t* code_bytes, size_t* scale_bytes);

/*
 * Clip ratios sigma(alpha) = 1 / (1 + exp(-alpha)) per block column
 * (daily-arxiv summary, section "块级可学习裁剪": the sigmoid keeps the
 * ratios in (0, 1)).  Evaluated in double precision and rounded to fp32 once.
 * alpha_min_host, alpha_max_host: k floats each.  ratios_out_host: 2k floats,
 * interleaved {r_min_0, r_max_0, r_min_1, ...}.  Host only; no CUDA call.
 */
BATQ_API batq_status batq_clip_ratios(const float* alpha_min_host, const float* alpha_max_host, int k,
                             float* ratios_out_host);

/*
 * Online activation path (daily-arxiv summary, "块仿射变换 (BAT)", "GPK 分解",
 * "块级可学习裁剪"; thelatestinai.com page, Figure 2 caption): for every token
 * s and block i, with X_si the row-major 4x8 view of the 32 inputs,
 *   Y = B_i^T X_si A                       (= x . (B_i (x) A), fp32)
 *   lo = r_min_i * min(Y), hi = r_max_i * max(Y), Y_hat = min(max(Y, lo), hi)
 *   e = clamp(floor(log2 max|Y_hat|) - 2, -127, 127), scale byte e + 127
 *   codes = E2M1_RNE_satfinite(Y_hat * 2^-e)
 *
 * X: device, S rows of N elements (x_dtype), row stride ldx elements
 *    (ldx >= N, ldx * elem_size a multiple of 16, X 16-byte aligned).
 * A_host: host, 8x8 fp32 row-major (A[a][b] at a*8+b); copied into the launch.
 * B_dev: device, k x 16 fp32, 16-byte aligned; B_i row-major (B_i[r][c] at
 *    16i + 4r + c).
 * ratios_dev: device, 2k fp32 from batq_clip_ratios (16-byte aligned), or NULL
 *    for no clip.
 * codes: device, S x N/2 bytes, 16-byte aligned.
 * scales: device, batq_act_buffer_sizes(S, N, layout) bytes.
 * y_debug: device S x N fp32 or NULL; receives the pre-clip Y (tests only).
 * Errors: BATQ_ERR_SHAPE, BATQ_ERR_ALIGNMENT, BATQ_ERR_ARCH, BATQ_ERR_CUDA.
 */
BATQ_API batq_status batq_quant_act(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                           const float* A_host, const float* B_dev, const float* ratios_dev,
                           uint8_t* codes, uint8_t* scales, batq_scale_layout layout,
                           float* y_debug, void* stream);

/* Device workspace bytes batq_prepare_weights needs for N in-features. Host only. */
BATQ_API batq_status batq_prepare_workspace_size(int N, size_t* bytes);

/*
 * Offline weight side (thelatestinai.com page, Figure 3 caption: weight-side
 * transforms fused offline into the linear layers).  Since
 * y = x W^T = (x P)(P^-1 W^T), the fused weights are W' = W P^-T, i.e. per
 * row and block W'_mat = B_i^-1 W_mat A^-T.  The inverses of A and every B_i
 * are computed on the host in double precision (partial-pivot Gauss-Jordan);
 * W' is formed on the device in fp32 and quantized to MXFP4 along K by
 * round-to-nearest, without clipping.
 *
 * W: device, M x N (w_dtype), row stride ldw elements (16-byte aligned rows).
 * A_host: 8x8 fp32; B_host: k x 16 fp32 (host).
 * w_codes: device M x N/2 bytes; w_scales: batq_act_buffer_sizes(M, N, layout).
 * workspace: device, batq_prepare_workspace_size(N) bytes.
 * Errors: as batq_quant_act, plus BATQ_ERR_SINGULAR (condition number of A or
 * some B_i above 1e8) and BATQ_ERR_WORKSPACE.  Uses a pageable host->device
 * copy, so it must not be called during stream capture.
 */
BATQ_API batq_status batq_prepare_weights(const void* W, batq_dtype w_dtype, int M, int N, int ldw,
                                 const float* A_host, const float* B_host,
                                 uint8_t* w_codes, uint8_t* w_scales, batq_scale_layout layout,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * W4A4 MXFP4 x MXFP4 block-scaled GEMM on the tcgen05 tensor cores with fp32
 * accumulation in tensor memory:
 *   out[s][m] = sum_n deq(a)[s][n] * deq(w)[m][n],  deq = E2M1 value * 2^(scale - 127).
 * a_codes: S x N/2, a_scales: MMA layout for S rows; w_codes: M x N/2,
 * w_scales: MMA layout for M rows (all device, 16-byte aligned, K-major).
 * out: device S x M of out_dtype (fp32 or bf16), row stride ldo elements.
 * Errors: BATQ_ERR_SHAPE (N % 64, M % 16), BATQ_ERR_ALIGNMENT, BATQ_ERR_ARCH,
 * BATQ_ERR_CUDA.
 */
BATQ_API batq_status batq_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                            const uint8_t* w_codes, const uint8_t* w_scales,
                            int S, int M, int N, batq_dtype out_dtype, void* out, int ldo,
                            void* stream);

/* Device workspace bytes batq_linear needs (activation codes + MMA-layout scales). Host only. */
BATQ_API batq_status batq_linear_workspace_size(int S, int N, size_t* bytes);

/*
 * Whole W4A4 linear: batq_quant_act (MMA scale layout, into the workspace)
 * followed by batq_gemm_mxfp4 on the same stream.  Arguments as in those
 * two calls; w_codes / w_scales come from batq_prepare_weights with
 * BATQ_SCALES_MMA.
 */
BATQ_API batq_status batq_linear(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                        const float* A_host, const float* B_dev, const float* ratios_dev,
                        const uint8_t* w_codes, const uint8_t* w_scales, int M,
                        void* workspace, size_t workspace_bytes,
                        batq_dtype out_dtype, void* out, int ldo, void* stream);

/*
 * One linear of a group: the arguments of batq_linear, with the same meaning,
 * layout and ownership (A_host: 64 floats on the host, read during the call).
 */
typedef struct batq_linear_args {
  const void* X;
  batq_dtype x_dtype;
  int S, N, ldx;
  const float* A_host;
  const float* B_dev;
  const float* ratios_dev;
  const uint8_t* w_codes;
  const uint8_t* w_scales;
  int M;
  batq_dtype out_dtype;
  void* out;
  int ldo;
} batq_linear_args;

#define BATQ_MAX_LINEAR_GROUP 8

/* One activation of a quantiser group: the arguments of batq_quant_act. */
typedef struct batq_quant_args {
  const void* X;
  batq_dtype x_dtype;
  int S, N, ldx;
  const float* A_host;
  const float* B_dev;
  const float* ratios_dev;
  uint8_t* codes;
  uint8_t* scales;
  batq_scale_layout layout;
} batq_quant_args;

/*
 * `count` (1..8) independent batq_quant_act calls (no y_debug) on one stream.
 * Each activation takes the kernel its own call would take: those for the
 * tensor-core transform (bf16, at least six 128 x 128 tiles per SM) share one
 * launch (their tiles form one list); the others get their own launches of
 * the CUDA-core kernel, which start side by side (each waits for the launch
 * before it only before finishing).  Codes and scales equal batq_quant_act's
 * bit for bit.  Outputs must not overlap one another or any input.
 * Errors: as batq_quant_act for each (the first failing check's code),
 * BATQ_ERR_INVALID_ARG for count out of range; nothing is launched when a
 * check fails.
 */
BATQ_API batq_status batq_quant_act_grouped(const batq_quant_args* acts, int count, void* stream);

/* One product of a GEMM group: the arguments of batq_gemm_mxfp4. */
typedef struct batq_gemm_args {
  const uint8_t* a_codes;
  const uint8_t* a_scales;
  const uint8_t* w_codes;
  const uint8_t* w_scales;
  int S, M, N;
  batq_dtype out_dtype;
  void* out;
  int ldo;
} batq_gemm_args;

/*
 * `count` (1..8) independent batq_gemm_mxfp4 calls on one stream.  When every
 * S > 128 and every out_dtype is the same, one launch of the CTA-pair GEMM
 * covers all of them; when every S <= 128 falls in the same tile
 * configuration (S <= 16, <= 32, <= 64 or <= 128; decode batches) with one
 * out_dtype, one launch of the single-CTA GEMM does; otherwise they run one
 * after another.  Results equal
 * batq_gemm_mxfp4's bit for bit.  Outputs must not overlap one another or any
 * input.  Errors: as batq_gemm_mxfp4 for each, BATQ_ERR_INVALID_ARG for count
 * out of range; nothing is launched when a check fails.
 */
BATQ_API batq_status batq_gemm_mxfp4_grouped(const batq_gemm_args* gemms, int count, void* stream);

/*
 * Workspace bytes batq_linear_grouped needs for `count` (1..8) linears: each
 * linear's batq_linear_workspace_size rounded up to 256 bytes, summed.  Host
 * only.  Errors: BATQ_ERR_INVALID_ARG (null pointers, count out of range), BATQ_ERR_SHAPE.
 */
BATQ_API batq_status batq_linear_grouped_workspace_size(const batq_linear_args* linears, int count,
                                                        size_t* bytes);

/*
 * `count` (1..8) independent linears on one stream, each computing what
 * batq_linear computes with its own arguments (BATQuant thelatestinai.com page,
 * Figure 2: transform, clip and quantise each linear's activations, then the
 * W4A4 product).  Linear i's codes and scales go to its 256-byte-aligned part
 * of the workspace, in order.  The activations are quantised as by
 * batq_quant_act_grouped; when the products qualify (see
 * batq_gemm_mxfp4_grouped: every S > 128, or every S <= 128 in one tile
 * configuration, with one out_dtype), one GEMM launch covers them all, which
 * saves the per-launch fill and drain of 2 x (count - 1) launches.  Otherwise
 * the GEMMs run one after another.  The outputs must not overlap one another
 * or any input.  Codes, scales and outputs equal batq_linear's bit for bit.
 * Errors: as batq_linear for each linear (the first failing
 * check's code), BATQ_ERR_INVALID_ARG for count out of range.  Nothing is
 * launched when a check fails.
 */
BATQ_API batq_status batq_linear_grouped(const batq_linear_args* linears, int count, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------ W4A8 variant
 * The pages' second setting (BATQuant thelatestinai.com page, abstract and
 * Table 2, W4A8 rows): the same transform and clip with MXFP8 activations,
 * E4M3 elements under the E8M0 shared scale 2^(floor(log2 amax) - 8) (OCP MX
 * v1.0), round to nearest even, magnitudes above 448 saturated to 448.  The
 * weights stay MXFP4 (same values and scales as batq_prepare_weights); for the
 * E4M3 x E4M3 block-scaled MMA (tcgen05 kind::mxf8f6f4) each E2M1 weight code
 * is held in one E4M3 byte of the same value.
 */

/* Bytes of MXFP8 codes (rows x N, one per element) and of scales. Host only. */
BATQ_API batq_status batq_mxfp8_buffer_sizes(int rows, int N, batq_scale_layout layout, size_t* code_bytes,
                                    size_t* scale_bytes);

/*
 * As batq_quant_act, but the codes are E4M3 bytes: codes is device S x N
 * bytes (16-byte aligned), element n of row s at s * N + n.  Scales as in
 * batq_quant_act.  Errors as batq_quant_act.
 */
BATQ_API batq_status batq_quant_act_mxfp8(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                 const float* A_host, const float* B_dev, const float* ratios_dev,
                                 uint8_t* codes, uint8_t* scales, batq_scale_layout layout,
                                 float* y_debug, void* stream);

/* Device workspace bytes batq_prepare_weights_w4a8 needs. Host only. */
BATQ_API batq_status batq_prepare_weights_w4a8_workspace_size(int M, int N, size_t* bytes);

/*
 * batq_prepare_weights, then each E2M1 code widened to the E4M3 byte of the
 * same value: w_codes8 is device M x N bytes (16-byte aligned); w_scales as in
 * batq_prepare_weights.  workspace: batq_prepare_weights_w4a8_workspace_size
 * bytes (it also holds the packed MXFP4 codes on the way).  Errors as
 * batq_prepare_weights.
 */
BATQ_API batq_status batq_prepare_weights_w4a8(const void* W, batq_dtype w_dtype, int M, int N, int ldw,
                                      const float* A_host, const float* B_host,
                                      uint8_t* w_codes8, uint8_t* w_scales, batq_scale_layout layout,
                                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * W4A8 block-scaled GEMM: out = deq(a) deq(w)^T with E4M3 codes on both sides
 * (a_codes8 S x N from batq_quant_act_mxfp8, w_codes8 M x N from
 * batq_prepare_weights_w4a8), MMA-layout scales, fp32 accumulation in tensor
 * memory.  Shapes, alignment and errors as batq_gemm_mxfp4.
 */
BATQ_API batq_status batq_gemm_w4a8(const uint8_t* a_codes8, const uint8_t* a_scales,
                           const uint8_t* w_codes8, const uint8_t* w_scales,
                           int S, int M, int N, batq_dtype out_dtype, void* out, int ldo,
                           void* stream);

/* Device workspace bytes batq_linear_w4a8 needs (E4M3 codes + MMA-layout scales). Host only. */
BATQ_API batq_status batq_linear_w4a8_workspace_size(int S, int N, size_t* bytes);

/*
 * Whole W4A8 linear: batq_quant_act_mxfp8 (MMA scale layout, into the
 * workspace) followed by batq_gemm_w4a8 on the same stream.  Arguments as
 * batq_linear, with the weights from batq_prepare_weights_w4a8.
 */
BATQ_API batq_status batq_linear_w4a8(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                             const float* A_host, const float* B_dev, const float* ratios_dev,
                             const uint8_t* w_codes8, const uint8_t* w_scales, int M,
                             void* workspace, size_t workspace_bytes,
                             batq_dtype out_dtype, void* out, int ldo, void* stream);

/* ------------------------------------------------------------------------
 * NVFP4 output variant.  The format is the one the ARCQuant page names
 * (section "背景：为什么 W4A4 在 NVFP4 上很难"): 16 E2M1 elements share one
 * E4M3 scale.  The transform and the clip stay on the method's 32-element
 * blocks (BATQuant daily-arxiv summary, "块仿射变换" and "块级可学习裁剪");
 * each clipped block is stored as two 16-element groups.  A per-tensor fp32
 * encode scale gs (decoded value = code x group scale / gs) widens the range
 * of the E4M3 group scales; gs = 1 is the format with no tensor scale.
 * Every step is an IEEE fp32 operation:
 *   group scale  s = E4M3(fp32(fp32(amax_group * gs) / 6)), nearest even,
 *                saturating at 448 (amax of the clipped group);
 *   element      q = fp32(y_hat * fp32(gs / s)) (multiplier 0 when s = 0),
 *                then E2M1 nearest even, saturating at 6, sign kept on zero.
 * A 32-block holding a non-finite value gets scale byte 0x7F (E4M3 NaN) in
 * both groups and zero codes.  Codes are packed as in batq_quant_act.  Scales
 * are one byte per row and group: LINEAR layout rows x N/16, row-major; MMA
 * layout the 128-row x 4-column tiles of batq_quant_act with N/16 columns
 * (N/16 is a multiple of 4) and rows padded to 128 with the byte 0x38 (1.0).
 * All scale pointers must be 16-byte aligned, gs pointers 4-byte aligned.
 * ------------------------------------------------------------------------ */

/* Sizes of an NVFP4 operand: rows x N/2 code bytes; scale bytes as above. Host only. */
BATQ_API batq_status batq_nvfp4_buffer_sizes(int rows, int N, batq_scale_layout layout, size_t* code_bytes,
                                    size_t* scale_bytes);

/*
 * As batq_quant_act with NVFP4 output.  gs_dev: device float holding the
 * per-tensor encode scale (finite and > 0; a static calibration value), or
 * NULL for 1.  It is read after the preceding grid in the stream finishes.
 * Errors as batq_quant_act; BATQ_ERR_ALIGNMENT also for a misaligned scales
 * or gs_dev pointer.
 */
BATQ_API batq_status batq_quant_act_nvfp4(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                 const float* A_host, const float* B_dev, const float* ratios_dev,
                                 const float* gs_dev, uint8_t* codes, uint8_t* scales,
                                 batq_scale_layout layout, float* y_debug, void* stream);

/* Device workspace bytes batq_prepare_weights_nvfp4 needs. Host only. */
BATQ_API batq_status batq_prepare_weights_nvfp4_workspace_size(int N, size_t* bytes);

/*
 * Offline weight side with NVFP4 output: the fused weights W' = W P^-T
 * (as batq_prepare_weights) are measured once for their largest magnitude
 * amax, then quantised (no clip) with gs = fp32(448 * 6 / amax) (1 for
 * all-zero weights), which is written to the device float *gs_out_dev for the
 * GEMM.  Two kernel launches and a 4-byte memset on `stream`, nothing
 * synchronised.  Errors as batq_prepare_weights (BATQ_ERR_INVALID_ARG also
 * for a NULL gs_out_dev).
 */
BATQ_API batq_status batq_prepare_weights_nvfp4(const void* W, batq_dtype w_dtype, int M, int N, int ldw,
                                       const float* A_host, const float* B_host, uint8_t* w_codes,
                                       uint8_t* w_scales, batq_scale_layout layout, float* gs_out_dev,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * NVFP4 block-scaled GEMM (tcgen05 kind::mxf4nvf4, one E4M3 scale per 16 K):
 * out = fp32(1 / fp32(gs_a * gs_w)) x sum_n (code_a s_a)(code_w s_w), fp32
 * accumulation in tensor memory.  a_gs_dev / w_gs_dev: device floats (NULL
 * for 1), read after the preceding grid finishes.  Scales in MMA layout.
 * Shapes and errors as batq_gemm_mxfp4.
 */
BATQ_API batq_status batq_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_gs_dev,
                            const uint8_t* w_codes, const uint8_t* w_scales, const float* w_gs_dev,
                            int S, int M, int N, batq_dtype out_dtype, void* out, int ldo, void* stream);

/* Device workspace bytes batq_linear_nvfp4 needs (codes + MMA-layout scales). Host only. */
BATQ_API batq_status batq_linear_nvfp4_workspace_size(int S, int N, size_t* bytes);

/*
 * Whole NVFP4 linear: batq_quant_act_nvfp4 (gs from a_gs_dev, MMA layout,
 * into the workspace) followed by batq_gemm_nvfp4 on the same stream, with
 * the weights and w_gs_dev from batq_prepare_weights_nvfp4.  Other arguments
 * and errors as batq_linear.
 */
BATQ_API batq_status batq_linear_nvfp4(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                              const float* A_host, const float* B_dev, const float* ratios_dev,
                              const float* a_gs_dev, const uint8_t* w_codes, const uint8_t* w_scales,
                              const float* w_gs_dev, int M, void* workspace, size_t workspace_bytes,
                              batq_dtype out_dtype, void* out, int ldo, void* stream);

/* ------------------------------------------------------------------------
 * Naive Kronecker decomposition (BATQuant thelatestinai.com page, Table 1,
 * middle row: P_i = B_i (x) A_i with an 8x8 A_i per block, k (g1^2 + g2^2)
 * parameters, 10,240 at N = 4096, against GPK's shared A).  The same path as
 * batq_quant_act / batq_prepare_weights / batq_linear with MXFP4 output,
 * except that A is replaced by one 8x8 row-major A_i per block column:
 * A_blocks k x 64 floats (device, 16-byte aligned, for the activation calls;
 * host for the weight preparation, which inverts every A_i in fp64 and returns
 * BATQ_ERR_SINGULAR as batq_prepare_weights does).
 * ------------------------------------------------------------------------ */

/*
 * As batq_quant_act (MXFP4 codes, scales in either layout, optional y_debug)
 * with A_blocks_dev (device, k x 64 floats, A_i row-major at 64 i, 16-byte
 * aligned) in place of the shared A.  Errors as batq_quant_act;
 * BATQ_ERR_INVALID_ARG for a NULL A_blocks_dev, BATQ_ERR_ALIGNMENT for a
 * misaligned one.
 */
BATQ_API batq_status batq_quant_act_kron(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                const float* A_blocks_dev, const float* B_dev, const float* ratios_dev,
                                uint8_t* codes, uint8_t* scales, batq_scale_layout layout, float* y_debug,
                                void* stream);

/* Device workspace bytes batq_prepare_weights_kron needs (B'_i and A'_i). Host only. */
BATQ_API batq_status batq_prepare_weights_kron_workspace_size(int N, size_t* bytes);

/*
 * As batq_prepare_weights with A_blocks_host (host, k x 64 floats) in place
 * of A: W'_mat = B_i^-1 W_mat A_i^-T per block, MXFP4 without clip.  The fp64
 * inverses of every A_i and B_i are formed on the host (BATQ_ERR_SINGULAR if
 * any is singular or has 1-norm condition number above 1e8) and copied into
 * `workspace` (batq_prepare_weights_kron_workspace_size bytes, device,
 * 16-byte aligned) before the quantiser runs.  Other errors as
 * batq_prepare_weights.
 */
BATQ_API batq_status batq_prepare_weights_kron(const void* W, batq_dtype w_dtype, int M, int N, int ldw,
                                      const float* A_blocks_host, const float* B_host, uint8_t* w_codes,
                                      uint8_t* w_scales, batq_scale_layout layout, void* workspace,
                                      size_t workspace_bytes, void* stream);

/*
 * Whole linear with per-block A_i: batq_quant_act_kron into the workspace
 * (batq_linear_workspace_size bytes) followed by the MXFP4 GEMM on the same
 * stream, with the weights from batq_prepare_weights_kron.  Arguments and
 * errors otherwise as batq_linear.
 */
BATQ_API batq_status batq_linear_kron(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                             const float* A_blocks_dev, const float* B_dev, const float* ratios_dev,
                             const uint8_t* w_codes, const uint8_t* w_scales, int M, void* workspace,
                             size_t workspace_bytes, batq_dtype out_dtype, void* out, int ldo, void* stream);

/* ------------------------------------------------------------------------
 * BAT on the KV cache (the pages' KV8 / KV4 settings: BATQuant thelatestinai.com
 * page, Table 2 caption, W4A8KV8 and W4A8KV4; gist.science summary, §2.D: the
 * transforms also apply to the KV cache).  New key (or value) rows -- N =
 * kv_heads x head_dim elements per token, N % 64 == 0 -- go through the same
 * block transform, clip and MX quantisation as batq_quant_act (A, B_i and the
 * clip ratios are the cache's own) and are written into a paged cache at the
 * rows slot_mapping names.  The attention side (the inverse transform folded
 * into the queries or the output projection) is not part of this call.
 * ------------------------------------------------------------------------ */

typedef enum {
  BATQ_KV_MXFP4 = 0, /* KV4: packed E2M1 codes, num_slots x N/2 bytes */
  BATQ_KV_MXFP8 = 1  /* KV8: E4M3 codes, num_slots x N bytes */
} batq_kv_format;

/*
 * slot_mapping_dev: device int32[S], the cache row of each new token; tokens
 * with a negative slot, or one >= num_slots, are skipped (padding tokens); two
 * tokens must not share a slot.  cache_codes: device num_slots x (N/2 or N)
 * bytes, 16-byte aligned; cache_scales: device num_slots x N/32 E8M0 bytes
 * (LINEAR layout).  Rows not named are left as they were.  Stream-ordered,
 * asynchronous.  Errors: BATQ_ERR_INVALID_ARG (null pointers, num_slots < 1,
 * unknown format), BATQ_ERR_SHAPE, BATQ_ERR_ALIGNMENT, BATQ_ERR_ARCH,
 * BATQ_ERR_CUDA.
 */
BATQ_API batq_status batq_quant_kv_cache(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                const float* A_host, const float* B_dev, const float* ratios_dev,
                                const int* slot_mapping_dev, int num_slots, batq_kv_format kv_format,
                                uint8_t* cache_codes, uint8_t* cache_scales, void* stream);

/* ------------------------------------------------------------------------
 * RMSNorm fused ahead of the activation path (the step before every linear:
 * BATQuant transforms the activations online before each linear,
 * thelatestinai.com page, Figure 3 caption; the pages' only kernel design,
 * ARCQuant's reading notes, section "融合核函数设计", fuses RMSNorm with the
 * quantisation).  Per token s: z = x_s / sqrt(mean_j x_sj^2 + eps) * gamma,
 * then y = z P_i, the clip and MXFP4 exactly as batq_quant_act.  z never
 * leaves the library's kernels and is not rounded to bf16: a first kernel
 * computes each token's 1 / sqrt(mean x^2 + eps) (sum of squares in fp64,
 * rounded to fp32 once) into the workspace, and the quantiser applies gamma
 * to the elements and that factor to the transformed values.
 * ------------------------------------------------------------------------ */

/* Device workspace bytes batq_rmsnorm_quant_act needs (S floats, rounded up to 256). Host only. */
BATQ_API batq_status batq_rmsnorm_workspace_size(int S, size_t* bytes);

/*
 * As batq_quant_act (MXFP4 codes, scales in either layout, optional y_debug:
 * the transformed values of z) with the RMSNorm ahead of the transform.
 * gamma_dev: device, N floats, 16-byte aligned; eps: finite, >= 0.
 * workspace: device, >= batq_rmsnorm_workspace_size(S) bytes, 16-byte
 * aligned; it receives the per-token factors (the caller owns it).  Errors as
 * batq_quant_act, plus BATQ_ERR_INVALID_ARG (NULL gamma or workspace, eps
 * negative or not finite), BATQ_ERR_WORKSPACE, BATQ_ERR_ALIGNMENT.
 */
BATQ_API batq_status batq_rmsnorm_quant_act(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                            const float* gamma_dev, float eps, const float* A_host,
                                            const float* B_dev, const float* ratios_dev, uint8_t* codes,
                                            uint8_t* scales, batq_scale_layout layout, void* workspace,
                                            size_t workspace_bytes, float* y_debug, void* stream);

/* Device workspace bytes batq_rmsnorm_linear needs: batq_linear's plus the per-token factors. Host only. */
BATQ_API batq_status batq_rmsnorm_linear_workspace_size(int S, int N, size_t* bytes);

/*
 * Whole linear with the RMSNorm ahead of the transform: batq_rmsnorm_quant_act
 * into the workspace (codes and MMA scales laid out as for batq_linear, the
 * per-token factors after them) followed by the MXFP4 GEMM against weights
 * prepared by batq_prepare_weights, on the same stream.  Arguments and errors
 * otherwise as batq_linear and batq_rmsnorm_quant_act.
 */
BATQ_API batq_status batq_rmsnorm_linear(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                         const float* gamma_dev, float eps, const float* A_host,
                                         const float* B_dev, const float* ratios_dev, const uint8_t* w_codes,
                                         const uint8_t* w_scales, int M, void* workspace, size_t workspace_bytes,
                                         batq_dtype out_dtype, void* out, int ldo, void* stream);

/*
 * batq_linear without a caller-provided workspace, for callers that cannot
 * allocate device memory (for example a plugin running in a process whose
 * device memory is fully reserved by another allocator, or a path where the
 * device synchronisation cudaMalloc / cudaFree may cause is not allowed).  The
 * method has no counterpart of this call: it only changes where the scratch
 * lives.  Arguments, results and errors are those of batq_linear.
 *
 * The scratch is a fixed array of BATQ_NO_ALLOC_SCRATCH_BYTES in the
 * library's own device memory; every GPU that loads the library holds it
 * until the process exits.  Problems whose batq_linear_workspace_size exceeds
 * it return BATQ_ERR_SCRATCH_LIMIT before anything is launched (for N = 4096,
 * up to 7704 tokens fit).  The call allocates nothing itself, but CUDA
 * creates the array on a device when it loads the library's device code there,
 * which with the default lazy module loading happens at the first call on
 * that device (or at any earlier libbatq call that ran there).  A process
 * whose device memory another allocator reserves up front should therefore
 * make one small, valid batq_linear_no_alloc call on each device before that
 * allocator reserves the memory (a call refused with BATQ_ERR_SCRATCH_LIMIT
 * returns before touching the device and does not create it), or set
 * CUDA_MODULE_LOADING=EAGER so the array is created when the CUDA context is.
 * The first call on a device also looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  All calls
 * share the one array and it keeps the last call's contents (every byte the
 * GEMM reads is rewritten by each call, so stale contents are never used), so
 * calls that can overlap on the GPU (different streams, or several host
 * threads) race on it and must be serialised by the caller.
 */
BATQ_API batq_status batq_linear_no_alloc(const void* X, batq_dtype x_dtype, int S, int N, int ldx,
                                          const float* A_host, const float* B_dev, const float* ratios_dev,
                                          const uint8_t* w_codes, const uint8_t* w_scales, int M,
                                          batq_dtype out_dtype, void* out, int ldo, void* stream);

/*
 * Failure-path self-test: launches a one-thread kernel that waits on a
 * barrier nothing ever arrives on, with a bounded wait of `limit_us`
 * microseconds (1 .. 1e6) -- the same bounded wait every libbatq kernel uses
 * for its pipeline barriers.  The wait expires, the kernel sets bit 0 of the
 * device error word and returns; the context stays usable.  Follow with
 * batq_device_error to read (and clear) the word.  The method has no
 * counterpart of this call.  Errors: BATQ_ERR_INVALID_ARG, BATQ_ERR_ARCH,
 * BATQ_ERR_CUDA.
 */
BATQ_API batq_status batq_selftest_wait_timeout(unsigned int limit_us, void* stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word.  Kernels set bits there when a bounded wait on a barrier gives up
 * (bit 0: data never arrived; bit 1: a stage was never released; bit 2: an
 * MMA never completed; bit 3: the accumulator was never drained).
 * *flags_out receives the word; returns BATQ_ERR_TIMEOUT if it was non-zero.
 */
BATQ_API batq_status batq_device_error(void* stream, unsigned int* flags_out);

#ifdef __cplusplus
}
#endif

#endif /* BATQ_H */
