/*
 * kroquant.h -- C ABI of the KroQuant online activation quantizer for
 * NVIDIA B200 (sm_100a), with the SmoothQuant and plain-MXFP4 baselines.
 *
 * What is computed ("KroQuant: Kronecker-Structured Block Transforms for
 * Efficient Post-Training Quantization of Diffusion Transformers",
 * arXiv 2607.21446, abstract and section 3.2, Eq. (4) as summarised by the
 * Pith review of the paper): every token row of a bf16 activation X[M, d] is
 * cut into d/32 blocks of 32 consecutive channels; block j of every row is
 * multiplied by the 32x32 matrix K^(j) = G1 (x) G2 (x) G3 (x) G4 (x) G5, a
 * Kronecker product of five 2x2 factors; the result y is quantized to MXFP4:
 *
 *   amax  = max_i |y_i|                                  (fp32)
 *   e     = clamp(floor(log2(amax)) - 2, -127, 127)      (amax = 0 -> -127)
 *   scale = byte e + 127 (E8M0), one per block
 *   code  = FP4 E2M1 of y_i * 2^-e, round-to-nearest-even, saturating at +-6,
 *           sign bit = sign of y_i (a negative value that rounds to zero is 0x8)
 *
 * (the scale rule and element format are the OCP Microscaling Formats v1.0
 * MXFP4 conversion, section 6.3).
 *
 * Layouts (all row-major, contiguous, no strides):
 *   act      bf16 [M][d]              d a positive multiple of 32
 *   factors  float32 [d/32][5][2][2]   factors[j][k] is G_(k+1) of column block
 *                                      j, stored [row][col]; G1 acts on bit 4
 *                                      (the MSB) of the in-block index, G5 on
 *                                      bit 0 (the textbook Kronecker order).
 *                                      Shared mode: one set [5][2][2] for every
 *                                      column block.
 *   codes    uint8 [M][d/2]           element 2i in the low nibble of byte i,
 *                                      element 2i+1 in the high nibble.
 *   scales   uint8 [M][d/32]          E8M0 byte of each block.
 *
 * Conventions shared by every entry point:
 *   - Every pointer is a DEVICE pointer owned by the caller.  The library never
 *     allocates, frees or synchronises; work is enqueued on `stream` (NULL =
 *     the legacy default stream) and runs asynchronously.
 *   - The returned status covers argument checks and launch errors only;
 *     asynchronous execution errors surface at the caller's next synchronising
 *     CUDA call.  On any non-OK status kq_last_error() describes it.
 *   - M == 0 (or N == 0) is a no-op that returns KQ_OK without touching the GPU.
 *   - Argument checks run before any CUDA call, in this order: negative sizes
 *     or d % 32 != 0 -> KQ_ERR_SHAPE; NULL pointer with nonzero size ->
 *     KQ_ERR_NULL; misalignment -> KQ_ERR_ALIGN.
 *   - Alignment: act, out_codes, out_y, W, W_out 16 bytes; factors and mult
 *     16 bytes; out_scales 1 byte.
 *   - Input with a non-finite value (inf/NaN) is outside the contract: such a
 *     block's outputs are unspecified (but written in bounds).
 *   - Work runs on the calling thread's current CUDA device: every pointer and
 *     `stream` must belong to it.  Device properties the launches need (SM
 *     count, occupancy, shared-memory opt-ins, tile choices) are looked up
 *     once per device and kept in thread-safe process-wide caches.
 *   - Calls on different streams that write the same output race; besides
 *     those caches and the bounded-wait counter (kq_wait_timeouts), nothing is
 *     shared between calls.  Calls may come from several host threads.
 */
#ifndef KROQUANT_H
#define KROQUANT_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's stream handle (same definition as cuda_runtime_api.h). */
typedef struct CUstream_st *cudaStream_t;

typedef enum {
    KQ_OK = 0,
    KQ_ERR_NULL = -1,    /* a required pointer is NULL */
    KQ_ERR_SHAPE = -2,   /* M < 0, N < 0, d <= 0, d % 32 != 0, or size overflow */
    KQ_ERR_ALIGN = -3,   /* a pointer is not aligned as documented above */
    KQ_ERR_CUDA = -4,    /* a CUDA runtime call failed (launch, attribute query) */
    KQ_ERR_VARIANT = -5  /* kq_quantize_variant: unknown or unavailable variant */
} kq_status;

/* KroQuant quantizer, one factor set per column block ([d/32][5][2][2]).
 * Reads act once, writes codes and scales once, in one fused kernel. */
int kq_quantize(const void *act_bf16, const float *factors,
                uint8_t *out_codes, uint8_t *out_scales,
                int64_t M, int64_t d, cudaStream_t stream);

/* KroQuant quantizer with one factor set ([5][2][2]) shared by every column
 * block (the shared-parameter mode of the SANA-shaped layers). */
int kq_quantize_shared(const void *act_bf16, const float *factors,
                       uint8_t *out_codes, uint8_t *out_scales,
                       int64_t M, int64_t d, cudaStream_t stream);

/* SmoothQuant baseline ("KroQuant ...", abstract: per-channel scaling): y_c =
 * fp32(x_c * mult[c]) with mult[c] = 1/s_c given (float32 [d]), then the MXFP4
 * block quantizer above. */
int sq_quantize(const void *act_bf16, const float *mult,
                uint8_t *out_codes, uint8_t *out_scales,
                int64_t M, int64_t d, cudaStream_t stream);

/* Plain MXFP4 baseline: the block quantizer above applied to x itself. */
int mx_quantize(const void *act_bf16,
                uint8_t *out_codes, uint8_t *out_scales,
                int64_t M, int64_t d, cudaStream_t stream);

/* KroQuant quantizer from the LU parametrisation of each factor (KroQuant
 * section 3.2, Eq. (6) as summarised by the Pith review): G_k = L_k U_k with
 * U_k = [[a_k, b_k], [0, -1/a_k]] and L_k = [[1, 0], [c_k, 1]] (L unit lower
 * triangular: a reading, the pages print only U), i.e.
 * G_k = [[a_k, b_k], [c_k a_k, c_k b_k - 1/a_k]], det G_k = -1.
 * lu_params: float32 [d/32][5][3] = (a, b, c) of G1..G5 per column block, 15
 * scalars per block; shared != 0: one set [5][3] for every block.  Every
 * a_k must be nonzero.  The factors are expanded in-kernel (the paper's
 * on-the-fly "K2" kernel), then as kq_quantize.  lu_params: 4-byte aligned. */
int kq_quantize_lu(const void *act_bf16, const float *lu_params, int shared,
                   uint8_t *out_codes, uint8_t *out_scales,
                   int64_t M, int64_t d, cudaStream_t stream);

/* The KroQuant quantizer fused with the normalisation that produces its input
 * ("KroQuant ...", abstract: normalisation layers between blocks force the
 * transform online).  For every token row h (bf16 [M][d]):
 *   x_mod = LayerNorm(h) * (1 + gamma[b]) + beta[b]
 * with LayerNorm without affine (mean and biased variance over the d
 * channels, eps inside the square root) and AdaLN modulation by per-sample
 * vectors gamma, beta (float32 [nsamples][d]; row r belongs to sample
 * r / (M / nsamples)); then kq_quantize on x_mod, which stays in fp32 and is
 * never written out.  Needs M % nsamples == 0 and d <= 16384.  h, gamma, beta,
 * factors, out_codes: 16-byte aligned. */
int norm_kq_quantize(const void *h_bf16, const float *gamma, const float *beta,
                     int64_t nsamples, float eps, const float *factors, int shared,
                     uint8_t *out_codes, uint8_t *out_scales,
                     int64_t M, int64_t d, cudaStream_t stream);

/* Test export: norm_kq_quantize through a chosen kernel (the same result up
 * to the rounding of the row statistics, within the transform tolerance):
 *   0  the default (3 from 192 block columns up, else 1 where it fits, else 2),
 *   1  one warp per row, rows streamed once into shared-memory row buffers
 *      beside a per-column coefficient table (falls to 2 where none fits),
 *   2  one warp per row, the row read twice (statistics, then transform),
 *   3  one CTA per row, one thread per block column: coefficients in
 *      registers, rows streamed once through a per-thread cp.async ring,
 *      row statistics by a CTA reduction.
 * Other values return KQ_ERR_VARIANT. */
int norm_kq_quantize_variant(int variant, const void *h_bf16, const float *gamma, const float *beta,
                             int64_t nsamples, float eps, const float *factors, int shared,
                             uint8_t *out_codes, uint8_t *out_scales,
                             int64_t M, int64_t d, cudaStream_t stream);

/* Fixed-Hadamard baseline (the pages' comparison point for the on-the-fly
 * kernel, a fast Walsh-Hadamard transform): y = H_H x / sqrt(H) on every H
 * consecutive channels of a row, H_H the Sylvester Hadamard matrix, H a
 * power of two in [32, 1024] dividing d; then the MXFP4 block quantizer above
 * on each 32-block.  H outside that set or d % H != 0 -> KQ_ERR_SHAPE. */
int fwht_quantize(const void *act_bf16, int64_t H,
                  uint8_t *out_codes, uint8_t *out_scales,
                  int64_t M, int64_t d, cudaStream_t stream);

/* Offline fold of the inverse transform into weights (Pith review, "key
 * machinery": the inverse is folded into the weights offline), used to check
 * invertibility: W_out = W T^-1, i.e. for every row n and column block j,
 * W_out[n, blk j] = W[n, blk j] (K^(j))^-1, so that
 * X W^T == (X T^T)(W_out)^T.  W, W_out: float32 [N][d] (may not alias).
 * shared != 0 selects one factor set for all blocks.  Every factor must be
 * invertible (det != 0); a zero determinant yields inf/NaN outputs. */
int kq_fold_weights(const float *W, const float *factors, int shared,
                    float *W_out, int64_t N, int64_t d, cudaStream_t stream);

/* Inverse transform, x = T^-1 y per 32-block (y, x_out float32 [M][d], may not
 * alias): the Kronecker product of the factor inverses G_k^-1 applied as
 * butterflies.  With mx_dequantize it gives the round trip x -> codes/scales
 * -> x^ used to measure quantisation error.  Every factor must be invertible. */
int kq_inverse_f32(const float *y, const float *factors, int shared,
                   float *x_out, int64_t M, int64_t d, cudaStream_t stream);

/* MXFP4 decode: out[r][32j + i] = E2M1(code) * 2^(scale - 127) (float32
 * [M][d]; exact in fp32; scale byte 0xFF gives NaN).  codes and out 16-byte
 * aligned. */
int mx_dequantize(const uint8_t *codes, const uint8_t *scales, float *out,
                  int64_t M, int64_t d, cudaStream_t stream);

/* ---- W4A4 consumer: the linear layer on the quantized operands ----------
 *
 * Scale-factor layout ("sf"): the E8M0 scales of a [rows][d] MXFP4 matrix as
 * the block-scaled tensor-core MMA reads them (NVIDIA PTX ISA, tcgen05.mma
 * block scaling, the scale-factor operand).  With nb = d/32 block columns,
 * the scales of 128 consecutive rows x 4 consecutive block columns form one
 * 512-byte unit; the scale of row r, block column j sits at byte
 *   ((r / 128) * ceil(nb / 4) + j / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + j % 4.
 * A buffer holds kq_sf_bytes(rows, d) bytes (whole units: rows rounded up to
 * 128, block columns to 4).  The writers below fill every real scale and,
 * when nb is odd, the byte of block column nb (set to 0x00): mxf4_gemm reads
 * it beside column nb-1.  Other padding bytes are left untouched and are
 * never read for an output element. */
#define KQ_SCALES_ROWMAJOR 0
#define KQ_SCALES_SF 1

/* Bytes of a scale-factor-layout buffer for a [rows][d] matrix; -1 for
 * rows < 0 or d not a positive multiple of 32.  Host only, no CUDA call. */
int64_t kq_sf_bytes(int64_t rows, int64_t d);

/* kq_quantize (shared != 0: kq_quantize_shared) with the scales written in
 * the scale-factor layout to out_sf (kq_sf_bytes(M, d) bytes, 1-byte
 * aligned); codes exactly as kq_quantize. */
int kq_quantize_sf(const void *act_bf16, const float *factors, int shared,
                   uint8_t *out_codes, uint8_t *out_sf,
                   int64_t M, int64_t d, cudaStream_t stream);

/* The plain MXFP4 quantizer on float32 input x [M][d] (for the folded weights
 * W T^-1 from kq_fold_weights, which are fp32): the block rule above on the
 * fp32 values.  scale_layout KQ_SCALES_ROWMAJOR writes out_scales [M][d/32],
 * KQ_SCALES_SF the scale-factor layout (kq_sf_bytes(M, d) bytes); any other
 * value -> KQ_ERR_SHAPE.  x and out_codes 16-byte aligned. */
int mx_quantize_f32(const float *x, uint8_t *out_codes, uint8_t *out_scales,
                    int scale_layout, int64_t M, int64_t d, cudaStream_t stream);

/* norm_kq_quantize with the scales written in the scale-factor layout to
 * out_sf (kq_sf_bytes(M, d) bytes, 1-byte aligned); codes exactly as
 * norm_kq_quantize.  With mxf4_gemm this is the whole W4A4 layer input path:
 * residual stream h -> LayerNorm + AdaLN -> transform -> MXFP4 -> product,
 * with no intermediate written in bf16 and no scale relayout. */
int norm_kq_quantize_sf(const void *h_bf16, const float *gamma, const float *beta,
                        int64_t nsamples, float eps, const float *factors, int shared,
                        uint8_t *out_codes, uint8_t *out_sf,
                        int64_t M, int64_t d, cudaStream_t stream);

/* Row-major scales [M][d/32] (from any quantizer here) -> the scale-factor
 * layout (kq_sf_bytes(M, d) bytes; the buffers may not overlap). */
int mx_scales_to_sf(const uint8_t *scales, uint8_t *out_sf,
                    int64_t M, int64_t d, cudaStream_t stream);

/* The W4A4 linear layer ("KroQuant ...", abstract: W4A4 at MXFP4; section
 * 3.2, Eq. (4): the inverse folded into the weights, so that
 * X W^T = (X T^T)(W T^-1)^T):
 *   out[m][n] = sum_k a[m][k] * b[n][k]
 * with a the decoded MXFP4 activation (a_codes [M][K/2], a_sf its scales in
 * the scale-factor layout, kq_sf_bytes(M, K) bytes) and b the decoded MXFP4
 * weight (b_codes [N][K/2], b_sf, kq_sf_bytes(N, K) bytes).  Products are
 * exact and accumulate in fp32 on the tensor cores (tcgen05 block-scaled
 * MMA); out is bf16 (out_f32 == 0, rounded to nearest even) or float32,
 * [M][N] row-major.  Needs K a positive multiple of 32, N a multiple of 8,
 * M, N, K < 2^31; every pointer 16-byte aligned; out may not overlap the
 * inputs.  A scale byte 0xFF (NaN) makes the outputs it reaches NaN. */
int mxf4_gemm(const uint8_t *a_codes, const uint8_t *a_sf,
              const uint8_t *b_codes, const uint8_t *b_sf,
              void *out, int out_f32, int64_t M, int64_t N, int64_t K,
              cudaStream_t stream);

/* Test export: mxf4_gemm through a chosen tile configuration (128 x 256
 * output tiles unless stated, one CTA per SM; a k-chunk is CB bytes of codes
 * per row):
 *   0  the default (what mxf4_gemm runs): above 128 rows 7, or 8 where
 *      256-column tiles fill the last wave of SM pairs badly; up to 128 rows
 *      4, or 6 where 256-column tiles fill the last wave of SMs badly,
 *   1  CB = 128, 4 stages, epilogue stores from registers,
 *   2  CB = 64, 6 stages, bf16 epilogue through shared memory and TMA stores,
 *   3  CB = 64, 4 stages, TMA stores,
 *   4  CB = 128, 3 stages, TMA stores,
 *   5  CB = 64, 8 stages, stores from registers,
 *   6  as 4 with 192-column tiles,
 *   7  SM pairs: clusters of two CTAs on two SMs, 256 x 256 tiles, one
 *      M256 MMA (tcgen05 .cta_group::2) per K step for both SMs, CB = 128,
 *      4 stages, TMA stores,
 *   8  as 7 with 256 x 192 tiles and two accumulators.
 * Same results for every configuration (the K order of the MMAs is the same).
 * Other values return KQ_ERR_VARIANT. */
int mxf4_gemm_variant(int variant, const uint8_t *a_codes, const uint8_t *a_sf,
                      const uint8_t *b_codes, const uint8_t *b_sf,
                      void *out, int out_f32, int64_t M, int64_t N, int64_t K,
                      cudaStream_t stream);

/* Test export: the fp32 transform y = T x (float32 [M][d]) exactly as the
 * quantizer computes it before the amax, for the transform-accuracy check. */
int kq_transform_f32(const void *act_bf16, const float *factors, int shared,
                     float *out_y, int64_t M, int64_t d, cudaStream_t stream);

/* Test export: the KroQuant quantizer through a chosen kernel variant:
 *   0  the default (what kq_quantize runs: 2),
 *   1  one block per thread, direct 2x2 stages, 16-byte loads,
 *   2  packed f32x2 pairs with the unit-diagonal split of each factor,
 *      register prefetch,
 *   3  the arithmetic of 2 on input staged through shared memory by TMA,
 *   4  the block transform on the tcgen05 tensor cores: Y_j = X_j K_j^T with
 *      K_j expanded in fp32 and split into three bf16 parts stacked along N
 *      (one MMA per block and k-step; bf16 x bf16 products are exact), the
 *      three fp32 partial results summed by the epilogue; TMA-fed,
 *      accumulators in tensor memory,
 *   9  the operations of 2 on two rows of a column at once (every stage a
 *      packed f32x2 FMA), input staged through shared memory by TMA, one
 *      CTA per SM; shapes whose block-column count does not fit its grid
 *      rule (and the fp32 export) run 2.
 * Variants 2, 3 and 9 give identical results.  Every variant emits a block
 * whose transformed values are not finite as the scale byte 0xFF with zero
 * codes; a unit-diagonal block that overflows only in its intermediates is
 * recomputed in the direct form.  Other values (5-8 were retired) return
 * KQ_ERR_VARIANT. */
int kq_quantize_variant(int variant, const void *act_bf16, const float *factors,
                        int shared, uint8_t *out_codes, uint8_t *out_scales,
                        int64_t M, int64_t d, cudaStream_t stream);

/* Test export: kq_transform_f32 through a chosen kernel variant (as above). */
int kq_transform_f32_variant(int variant, const void *act_bf16, const float *factors, int shared,
                             float *out_y, int64_t M, int64_t d, cudaStream_t stream);

/* Test exports: the baselines through a chosen kernel variant: 1 =
 * register-prefetch kernel, 2 = TMA-staged kernel, 0 = the default (SQ: 2,
 * MX: 1, the faster of the two on the benchmark shapes). */
int sq_quantize_variant(int variant, const void *act_bf16, const float *mult,
                        uint8_t *out_codes, uint8_t *out_scales,
                        int64_t M, int64_t d, cudaStream_t stream);
int mx_quantize_variant(int variant, const void *act_bf16,
                        uint8_t *out_codes, uint8_t *out_scales,
                        int64_t M, int64_t d, cudaStream_t stream);

/* Diagnostics of the bounded waits (no counterpart on the pages).  The
 * TMA-staged kernels wait on shared-memory barriers; every wait gives up after
 * about a second of clock cycles, adds 1 to a device counter per giving-up
 * thread, drains its copies in flight and returns, so the context stays
 * usable.  kq_wait_timeouts copies the counter to *count (synchronising the
 * device) and zeroes it if reset != 0.  The counter is one device-global int
 * of the library, shared by every call on that device: calls that overlap on
 * the GPU (several streams or threads) add to the same count, and a reset
 * clears theirs too.  kq_selftest_bounded_wait launches one staged CTA whose
 * producer issues no copies, so its waits run out after about a millisecond;
 * its operand is a fixed 80 KB device array of the library (1280 blocks of
 * 64 bytes, shared by all its calls), and it reads and writes no memory other
 * than that array and the counter (in fact only the counter). */
int kq_wait_timeouts(int *count, int reset);
int kq_selftest_bounded_wait(cudaStream_t stream);

/* Message for the last non-OK status returned on the calling thread (a static
 * thread-local buffer, valid until the thread's next call).  "" if none. */
const char *kq_last_error(void);

/* Library ABI version (this header: 1). */
int kq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KROQUANT_H */
