/*
 * kq.h -- C ABI of the KroQuant online activation quantizer (sm_100a).
 *
 * Method.  "KroQuant: Kronecker-Structured Block Transforms for Efficient
 * Post-Training Quantization of Diffusion Transformers" (Abstract; research
 * summary, method paragraph): before a W4A4 linear layer, every 32-channel
 * block j of an activation row is multiplied by a learned invertible matrix
 * T_j = A_j1 (x) A_j2 (x) A_j3 (x) A_j4 (x) A_j5, a Kronecker product of five
 * 2x2 unit-determinant LU factors, and the result is quantised to MXFP4; the
 * inverse transform is folded into the weights offline.
 *
 * Parameters (15 floats per block, fp32, layout [nb][15], nb = d / 32):
 *   factor m = 0..4 is (a, b, u) at [3m], [3m+1], [3m+2] and equals
 *   A = L U, L = [[1, 0], [a, 1]], U = [[u, b], [0, 1/u]]  (det A = 1).
 *   u must be non-zero and a, b, u finite.  Every kernel that reads the
 *   parameters checks this on the device: a violation sets
 *   KQ_DEVSTAT_BAD_PARAMS in the status word (kq_device_status) and the
 *   outputs of that call are unspecified; nothing faults.
 *   Factor m acts on bit (4 - m) of the channel index inside the block
 *   (factor 0 on the most significant bit: the standard Kronecker index map).
 *   Channel c = 32 j + i; y_j = T_j x_j for each token (column vector).
 *
 * MXFP4 output (OCP Microscaling Formats v1.0):
 *   scales  uint8 [M][nb] row-major, E8M0: value 2^(byte - 127), 0xFF = NaN.
 *           byte = clamp(floor(log2(amax_j)) - 2 + 127, 0, 254) where amax_j is
 *           the largest |y| of the block; a block holding NaN or Inf gets 0xFF
 *           and unspecified codes.
 *   codes   uint8 [M][d/2] row-major, E2M1 nibbles of r = y / 2^(byte - 127),
 *           rounded to nearest (ties to even), saturated to +-6, sign bit 3
 *           (a negative value that rounds to zero gives 0x8).  Element 2i of
 *           a row is the low nibble of byte i, element 2i+1 the high nibble.
 *
 * Conventions for every call:
 *   - every array pointer is a DEVICE pointer to memory the caller owns; the
 *     library allocates nothing and keeps no per-call state;
 *   - rows are contiguous (leading dimension = d);
 *   - work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = the
 *     legacy default stream) and the call returns after the launch; results
 *     are ready when the stream reaches that point;
 *   - arguments are checked on the host before anything is launched; a
 *     non-zero return means nothing was enqueued (KQ_ERR_CUDA: the launch
 *     itself failed; kq_last_error() has the CUDA message);
 *   - M == 0 (or N == 0) is a no-op that returns KQ_OK once the shape and
 *     dtype are valid; its pointers are not looked at and may be NULL;
 *   - the functions are thread-safe.
 *
 * Device waits.  The streaming kernels wait on shared-memory barriers for
 * their tensor-memory-access (TMA) loads.  Every wait is bounded (about one
 * second); a wait that runs out stops its thread block and sets a bit in a
 * per-device status word, read with kq_device_status().  In correct
 * operation this never happens.
 */
#ifndef KQ_H
#define KQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes --------------------------------------------------- */
#define KQ_OK               0
#define KQ_ERR_INVALID_ARG  1  /* NULL pointer, M < 0, d <= 0, d % 32 != 0   */
#define KQ_ERR_ALIGNMENT    2  /* a pointer lacks the alignment stated below */
#define KQ_ERR_DTYPE        3  /* x_dtype is not KQ_DTYPE_BF16 / KQ_DTYPE_F32 */
#define KQ_ERR_UNSUPPORTED  4  /* size beyond a documented limit             */
#define KQ_ERR_CUDA         5  /* a CUDA call failed; see kq_last_error()    */

/* ---- input element types -------------------------------------------- */
#define KQ_DTYPE_BF16 0   /* bfloat16, 2 bytes per element */
#define KQ_DTYPE_F32  1   /* float32, 4 bytes per element  */

/* Largest channel count the streaming kernels take (their per-block
 * coefficient tables live in shared memory). */
#define KQ_MAX_D 32768

/* ---- device status bits (kq_device_status) -------------------------- */
#define KQ_DEVSTAT_WAIT_TIMEOUT 0x1u   /* a bounded barrier wait ran out */
#define KQ_DEVSTAT_BAD_PARAMS   0x2u   /* an LU factor had u == 0 or a non-finite a, b or u */

/*
 * kq_quantize -- the online quantizer (the hot path).
 *   x       [M][d] activations, bf16 or fp32 (x_dtype); 16-byte aligned.
 *   params  [d/32][15] fp32 LU parameters (layout above); 4-byte aligned.
 *   codes   [M][d/2] uint8 output; 16-byte aligned.
 *   scales  [M][d/32] uint8 output; any alignment.
 * For each token row and block j: y = T_j x_j in fp32 arithmetic, then MXFP4
 * (the abstract: transform the activations, then quantise; W4A4 in MXFP4).
 * Limits: d <= KQ_MAX_D; M * d / 32 < 2^31; M < 2^30 (KQ_ERR_UNSUPPORTED).
 */
int kq_quantize(const void* x, int x_dtype, int64_t M, int64_t d,
                const float* params, uint8_t* codes, uint8_t* scales,
                void* stream);

/*
 * kq_quantize_tc -- the same operation as kq_quantize, computed the way the
 * method's own kernel does it ("small tensor-core GEMMs", Abstract): each
 * 32 x 32 block transform runs on the tcgen05 tensor cores (T_j expanded in
 * fp32 and split into three bf16 terms, fp32 accumulation in tensor memory)
 * and the SIMT warps only encode.  bf16 input only (KQ_ERR_DTYPE otherwise);
 * other arguments, layouts, limits and tolerances as kq_quantize.  On B200 at
 * DiT shapes it is slower than kq_quantize's packed-FP32 shear butterfly; it
 * is kept for that comparison.
 */
int kq_quantize_tc(const void* x, int x_dtype, int64_t M, int64_t d,
                   const float* params, uint8_t* codes, uint8_t* scales,
                   void* stream);

/*
 * kq_quantize_sf_tiled -- kq_quantize with the scale bytes written straight
 * into the blocked layout of kq_sf_tile (the operand format of
 * kq_gemm_mxfp4), saving that pass in a layer step; codes as kq_quantize.
 *   scales_tiled [ceil(M/128)][d/128][512] uint8; its bytes for rows past M
 *   are not written.  d a multiple of 128; other arguments as kq_quantize.
 */
int kq_quantize_sf_tiled(const void* x, int x_dtype, int64_t M, int64_t d,
                         const float* params, uint8_t* codes, uint8_t* scales_tiled,
                         void* stream);

/*
 * kq_quantize_centered -- the centring variant (a per-token-mean variant of
 * the online quantizer on the pages, from a different method): each token is
 * shifted by its own offset before the transform, MXFP4(T (x - mu 1)); the
 * GEMM restores the offset in full precision (kq_gemm_mxfp4_rank1).
 *   mu [M] fp32 (4-byte aligned), normally the per-token mean (kq_row_sum
 *   with scale 1/d); x - mu is formed in fp32.  Other arguments as kq_quantize.
 */
int kq_quantize_centered(const void* x, int x_dtype, int64_t M, int64_t d,
                         const float* params, const float* mu, uint8_t* codes,
                         uint8_t* scales, void* stream);

/*
 * kq_row_sum -- out[m] = scale * sum_k x[m][k], fp32 accumulation: the
 * per-token means of the centring variant (scale = 1/d) and the row sums W 1
 * of the weights its GEMM needs (scale = 1).
 *   x [M][d] bf16 or fp32 (16-byte aligned), out [M] fp32 (4-byte aligned).
 */
int kq_row_sum(const void* x, int x_dtype, int64_t M, int64_t d, float scale, float* out,
               void* stream);

/*
 * kq_transform -- the transform stage alone: y = blockdiag(T_j) x in fp32
 * (the abstract: an invertible linear transform applied to the activations,
 * block by block over 32 channels; research summary, method paragraph: each
 * block's matrix is the Kronecker product of five 2x2 LU factors).
 * Same arguments and limits as kq_quantize; y [M][d] fp32, 16-byte aligned.
 * It runs the same transform code as kq_quantize, so kq_quantize's codes are
 * the MXFP4 encoding of exactly these values.
 */
int kq_transform(const void* x, int x_dtype, int64_t M, int64_t d,
                 const float* params, float* y, void* stream);

/*
 * sq_quantize -- the comparison quantizer: per-channel scaling (the
 * abstract's SmoothQuant option) followed by the same MXFP4 encoding.
 *   inv_s [d] fp32 = 1 / s_c (4-byte aligned); y_c = x_c * inv_s[c] in fp32.
 * Other arguments and limits as kq_quantize.
 */
int sq_quantize(const void* x, int x_dtype, int64_t M, int64_t d,
                const float* inv_s, uint8_t* codes, uint8_t* scales,
                void* stream);

/*
 * kq_expand_params -- the dense blocks of the transform (research summary,
 * method paragraph: each 32-element block's matrix is the Kronecker product
 * of five 2x2 unit-determinant LU factors; the abstract: 15 parameters per
 * block, fewer than half of per-channel scaling's 32).
 *   params [nb][15] fp32 -> T [nb][32][32] fp32, row-major:
 *   T[j][i][k] = prod_m A_jm[bit(i, 4-m)][bit(k, 4-m)]  (y_i = sum_k T[i][k] x_k).
 *   d = 32 * nb.  T 4-byte aligned.
 */
int kq_expand_params(const float* params, int64_t d, float* T, void* stream);

/*
 * kq_fold_weights -- the inverse transform folded into the weights (done
 * offline; the abstract: the inverse goes to the weights).
 *   W [N][d] fp32 (nn.Linear layout, layer output = W x), params [d/32][15].
 *   W_out [N][d] fp32 = W blockdiag(T_j)^(-1), so W_out (T x) = W x.
 *   W_out may equal W (in place); otherwise the two must not overlap.
 *   fp32 arithmetic; T_j^(-1) = (x)_m A_jm^(-1), A^(-1) = [[ab+1/u, -b], [-au, u]].
 *   W and W_out 16-byte aligned.  Limit: N * d / 32 < 2^31.
 */
int kq_fold_weights(const float* W, int64_t N, int64_t d, const float* params,
                    float* W_out, void* stream);

/*
 * kq_quantize_weights -- the weight side of the W4A4 layer, done offline:
 * the inverse transform folded into the weights (the abstract: the inverse
 * goes to the weights) and the result quantised to MXFP4 like the
 * activations, in 32-element blocks along d (the GEMM's reduction
 * dimension, so weight and activation blocks line up).
 *   W [N][d] fp32 (nn.Linear layout), params [d/32][15] as above.
 *   codes [N][d/2] and scales [N][d/32]: the MXFP4 encoding (same rules as
 *   kq_quantize) of W' = W blockdiag(T_j)^(-1), evaluated in fp32 exactly as
 *   kq_fold_weights evaluates it; W' itself is never written.
 *   W and codes 16-byte aligned, params 4-byte aligned.  Limit: N * d / 32 < 2^31.
 */
int kq_quantize_weights(const float* W, int64_t N, int64_t d, const float* params,
                        uint8_t* codes, uint8_t* scales, void* stream);

/*
 * kq_sf_tile -- scale bytes in the blocked layout the tensor cores read them
 * from (the operand format of kq_gemm_mxfp4; no page counterpart: a layout
 * of the hardware).
 *   scales [R][K/32] uint8 row-major (as written by kq_quantize or
 *   kq_quantize_weights) -> tiled [ceil(R/128)][K/128][512] uint8: row r and
 *   scale column s at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + s % 4 of
 *   block (r / 128, s / 4); rows past R are zero.  K a multiple of 128.
 */
int kq_sf_tile(const uint8_t* scales, int64_t R, int64_t K, uint8_t* tiled, void* stream);

/*
 * kq_gemm_mxfp4 -- the W4A4 linear layer on the quantised operands (the step
 * after the quantizer: "before quantizing both" weights and activations to 4
 * bits, the abstract):
 *   Y[m][n] = sum_k a[m][k] * b[n][k], a = the MXFP4 activations (codes
 *   [M][K/2] from kq_quantize, scales tiled by kq_sf_tile), b = the MXFP4
 *   folded weights (codes [N][K/2] from kq_quantize_weights, scales tiled).
 *   Y [M][N] fp32 row-major.  Products on the tensor cores with the
 *   block-scaled FP4 MMA, fp32 accumulation in tensor memory.  When M and K
 *   are multiples of 256 and N of 256 (or else of 192) the work runs on pairs
 *   of SMs (256 x 256 or 256 x 192 tiles, one MMA over both SMs' shared
 *   memory); the result does not depend on which kernel ran.
 *   K a multiple of 128; all pointers 16-byte aligned; M, N < 2^31.
 */
int kq_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_sf_tiled, const uint8_t* b_codes,
                  const uint8_t* b_sf_tiled, int64_t M, int64_t N, int64_t K, float* Y,
                  void* stream);

/*
 * kq_gemm_mxfp4_bf16 -- kq_gemm_mxfp4 with Y written as bf16 (the dtype the
 * next op of a DiT layer takes): each fp32 sum rounded to bf16, nearest even.
 *   Y [M][N] bf16 row-major, 16-byte aligned; other arguments and limits as
 *   kq_gemm_mxfp4.
 */
int kq_gemm_mxfp4_bf16(const uint8_t* a_codes, const uint8_t* a_sf_tiled, const uint8_t* b_codes,
                       const uint8_t* b_sf_tiled, int64_t M, int64_t N, int64_t K, void* Y,
                       void* stream);

/*
 * kq_gemm_mxfp4_rank1 -- kq_gemm_mxfp4 plus the rank-1 term that restores
 * the centring variant's offsets: Y = MXFP4(A) MXFP4(B)^T + mu wsum^T, with
 * mu [M] the offsets given to kq_quantize_centered and wsum [N] = W 1 the
 * row sums of the unfolded weights (both fp32, 4-byte aligned); the term is
 * added in fp32 in the epilogue.  Other arguments as kq_gemm_mxfp4.
 */
int kq_gemm_mxfp4_rank1(const uint8_t* a_codes, const uint8_t* a_sf_tiled, const uint8_t* b_codes,
                        const uint8_t* b_sf_tiled, int64_t M, int64_t N, int64_t K,
                        const float* mu, const float* wsum, float* Y, void* stream);

/*
 * kq_dequant -- MXFP4 back to fp32, for checking (the abstract: W4A4 in
 * MXFP4; the element value is the E2M1 code times the block's E8M0 scale,
 * as the OCP Microscaling v1.0 format defines it):
 *   out[m][c] = E2M1(code) * 2^(scale - 127); scale 0xFF gives NaN.
 *   codes [M][d/2] (16-byte aligned), scales [M][d/32], out [M][d] fp32
 *   (16-byte aligned).  Values beyond the fp32 range (scale bytes 253, 254
 *   with large codes) become +-Inf; scale byte 0 gives fp32 subnormals.
 *   Limit: M * d / 32 < 2^31.
 */
int kq_dequant(const uint8_t* codes, const uint8_t* scales, int64_t M, int64_t d,
               float* out, void* stream);

/*
 * kq_device_status -- read the status word of the CURRENT device
 * (KQ_DEVSTAT_* bits set by kernels since it was last cleared) into *flags;
 * clear it when `clear` is non-zero.  Synchronous: it waits for all work on
 * the device.  Returns KQ_OK or KQ_ERR_CUDA.
 */
int kq_device_status(uint32_t* flags, int clear);

/*
 * kq_selftest_bounded_wait -- failure-detection self-test.  Enqueues a kernel
 * whose one thread waits, through the same bounded wait the streaming
 * kernels use, on a shared-memory barrier that nothing arrives on.  After
 * limit_us microseconds (1 .. 1e6) the wait gives up, the kernel sets
 * KQ_DEVSTAT_WAIT_TIMEOUT in the device status word and returns; nothing
 * faults and the context stays usable.  Read and clear the bit with
 * kq_device_status().  Not part of the method (no page describes it).
 */
int kq_selftest_bounded_wait(uint32_t limit_us, void* stream);

/* Static text for a status code (never NULL). */
const char* kq_status_string(int status);

/* Detail of the last failure on the calling thread ("" if none). */
const char* kq_last_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int kq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KQ_H */
