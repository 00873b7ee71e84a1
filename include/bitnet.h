/*
 * bitnet.h -- C ABI of libbitnet_b200.so: the BitLinear / H-BitLinear forward (BitNet b1.58,
 * BitNet v2) on one NVIDIA B200 (sm_100a).
 *
 * The forward has four steps:
 *   1. the latent weights W are ternarised with absmean (one scale gamma = mean|W| per tensor)
 *      and packed two bits per weight        ["The Era of 1-bit LLMs" summary page,
 *                                              sections 方法论 and 方法详解; BitNet b1.58 2B4T
 *                                              article, section 一.2 (BitLinear, W1.58A8)];
 *   2. in H-BitLinear every token row gets an online Hadamard transform  [BitNet v2 write-up,
 *      paragraphs on H-BitLinear; BitNet v2 abstract];
 *   3. every token row is quantised, with absmax to INT8 or with absmean to INT4  [2B4T
 *      article, 一.2; BitNet v2 write-up, 8-bit / 4-bit activation paragraph];
 *   4. a ternary x integer product accumulates in int32 and is rescaled to bf16
 *      [2B4T article, 一.2: multiplying by 1 adds, by -1 subtracts, by 0 skips].
 *
 * Conventions shared by every entry point
 *   - Pointers named *_dev are device pointers the caller owns; the library never allocates,
 *     frees or keeps them.  Every device pointer must be 16-byte aligned.
 *   - Matrices are row-major.  X and Y are bf16 (passed as void*), W is bf16.
 *   - Calls are asynchronous on `stream` (0 = the legacy default stream).  A return value of
 *     BITNET_OK means the work was enqueued.  Any other return means nothing was launched,
 *     except BITNET_ERR_CUDA (a launch failed part-way).  Faults of kernels that already ran,
 *     and device-side wait time-outs, are reported by bitnet_sync_status().
 *   - Shape rules: M >= 1 tokens; K >= 128 input features with K % 128 == 0; N >= 8 output
 *     features with N % 8 == 0.  H-BitLinear also needs K to be a power of two, 128..32768
 *     (else BITNET_ERR_UNSUPPORTED).  act_bits is 8 or 4.
 *   - bitnet_last_error() returns a text description of the last failure on this host thread.
 */
#ifndef BITNET_B200_H
#define BITNET_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including the CUDA headers. */
typedef struct CUstream_st *bitnet_stream_t;

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_INVALID = -1,     /* null or misaligned pointer, bad size, bad act_bits */
    BITNET_ERR_UNSUPPORTED = -2, /* valid arguments the library does not handle (e.g. K not a
                                    power of two for H-BitLinear, not an sm_100 device) */
    BITNET_ERR_CUDA = -3,        /* a CUDA runtime call or kernel launch failed */
    BITNET_ERR_TIMEOUT = -4,     /* a kernel gave up a bounded device-side wait (reported by
                                    bitnet_sync_status) */
    BITNET_ERR_WORKSPACE = -5    /* workspace smaller than the size query returned */
} bitnet_status;

/* Text for a status code (static storage). */
const char *bitnet_status_string(int status);

/* Detail of the last failure returned on the calling host thread (thread-local storage). */
const char *bitnet_last_error(void);

/* ---------------------------------------------------------------------------------------- */
/* Step 1: weight ternarisation and packing                                                  */
/* ---------------------------------------------------------------------------------------- */

/* Bytes of packed weights for an [N, K] matrix: N * K / 4. */
size_t bitnet_packed_weight_bytes(int64_t N, int64_t K);

/* Bytes of device workspace bitnet_quantize_pack_weights needs (partial sums of |w|). */
size_t bitnet_weight_workspace_bytes(int64_t N, int64_t K);

/*
 * absmean ternarisation ["The Era of 1-bit LLMs" summary, 方法论 / 方法详解]:
 *   gamma = fp32(max(mean |W|, 1e-5)), the mean taken in double over all N*K weights in a
 *   fixed order (the result does not depend on the launch);
 *   q = clip(round_half_even(w / gamma), -1, 1), the division IEEE fp32.
 * W_dev     bf16 [N, K] latent weights (read only).
 * Wp_dev    out: packed weights, N*K/4 bytes.  Row n is K/16 little-endian 32-bit words; word
 *           g holds k = 16g .. 16g+15 as offset codes u = q + 1 in {0, 1, 2}, weight
 *           k = 16g + 4p + j (p, j in 0..3) at bits 8j + 2p.
 * gamma_dev out: one float.
 * ws_dev    scratch of ws_bytes >= bitnet_weight_workspace_bytes(N, K); contents undefined
 *           afterwards.
 */
int bitnet_quantize_pack_weights(const void *W_dev, int64_t N, int64_t K, void *Wp_dev,
                                 float *gamma_dev, void *ws_dev, size_t ws_bytes,
                                 bitnet_stream_t stream);

/*
 * bitnet_quantize_pack_weights without a workspace argument, for callers that cannot allocate
 * device memory themselves -- for example a runtime that hands the library only the tensors it
 * already owns, or code running where cudaMalloc is not allowed.  (The pages have no counterpart:
 * this is a convenience of the library, not a step of the method.)
 * Same inputs, outputs and results as bitnet_quantize_pack_weights; the partial sums of |w| go
 * to a fixed scratch array inside the library (9472 bytes on every device that loads it, held
 * until the process exits).  Maximum: the weight count is split into at most 1184 partial sums,
 * which always fit, so every shape accepted by bitnet_quantize_pack_weights is accepted here;
 * a shape that needed more scratch would be rejected with BITNET_ERR_UNSUPPORTED.
 * The first call on a device looks up the scratch address (cudaGetSymbolAddress) with that
 * device current; make that first call before capturing a stream into a CUDA graph.
 * All calls share the one scratch array, which keeps the last call's contents (every entry is
 * rewritten before it is read, so nothing needs clearing): calls that overlap on the GPU --
 * on different streams without ordering between them -- race and give wrong gamma values.
 * The call allocates and frees nothing.
 */
int bitnet_quantize_pack_weights_noalloc(const void *W_dev, int64_t N, int64_t K, void *Wp_dev,
                                         float *gamma_dev, bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* Steps 2 and 3: online Hadamard transform and per-token activation quantisation            */
/* ---------------------------------------------------------------------------------------- */

/* Bytes of activation codes for M tokens: M*K (INT8) or M*K/2 (INT4). */
size_t bitnet_act_codes_bytes(int64_t M, int64_t K, int act_bits);

/*
 * Per token row m (BitNet v2 write-up, H-BitLinear; 2B4T article, 一.2):
 *   z = (1/sqrt(K)) H_K x  when hadamard != 0 (H_K in Sylvester order, H_2n = [[H,H],[H,-H]],
 *       computed in fp32 by a fast Walsh-Hadamard transform), else z = x;
 *   act_bits 8 (absmax; 2B4T article, 一.2): mx = max(max_k |z_k|, 1e-5); s = 127 / mx (IEEE
 *       fp32); codes = round_half_even(z * s); scales[m] = mx / 127;
 *   act_bits 4 (absmean; the BitNet v2 write-up gives INT8 and INT4 each their own strategy,
 *       formulas not printed, and the pages' other quantisation function is absmean):
 *       g = fp32(max(mean_k |z_k|, 1e-5)) (sum in double); s = sqrt7 / g with sqrt7 the fp32
 *       value of sqrt(7) (the mean magnitude maps to code sqrt 7, so a Gaussian row spans the
 *       4-bit range to about 2.3 standard deviations); codes = clip(round_half_even(z * s),
 *       -8, 7); scales[m] = g / sqrt7;
 *   rowsum[m] = sum_k codes.
 * X_dev       bf16 [M, K].
 * codes_dev   out: int8 [M, K] (act_bits 8) or [M, K/2] bytes (act_bits 4: every 8 codes
 *             k0..k0+7 fill 4 bytes, byte j = code k0+j in the low nibble and k0+4+j in the
 *             high nibble, two's complement).
 * scales_dev  out: float [M], the dequantisation step of each token.
 * rowsum_dev  out: int32 [M], the sum of each token's codes (used by the product kernels to
 *             remove the +1 offset of the stored weight codes).
 */
int bitnet_act_quant(const void *X_dev, int64_t M, int64_t K, int hadamard, int act_bits,
                     void *codes_dev, float *scales_dev, int32_t *rowsum_dev,
                     bitnet_stream_t stream);

/* Debug / parity entry: Z = (1/sqrt(K)) H_K X per row in fp32, X bf16 [M, K], Z float [M, K].
 * Same transform code as bitnet_act_quant. */
int bitnet_fwht_f32(const void *X_dev, int64_t M, int64_t K, float *Z_dev,
                    bitnet_stream_t stream);

/*
 * RMS normalisation fused in front of steps 2 and 3.  The pages name this normalisation without a
 * formula: BitNet b1.58 2B4T article, section 一.3 (subln normalisation in place of LayerNorm);
 * BitNet v2 write-up (RMS normalisation among the model's LLaMA-like components).  Per token row:
 *   y = (x * rinv) * g,  rinv = 1 / sqrt(sum_k x_k^2 / K + eps)   (each an IEEE fp32 operation),
 * then exactly bitnet_act_quant on y (hadamard != 0: z = (1/sqrt(K)) H_K y).
 * norm_gain_dev  bf16 [K] per-feature gain, 16-byte aligned, or NULL for unit gain.
 * eps            finite and > 0, else BITNET_ERR_INVALID.
 * Other arguments, layouts and errors as bitnet_act_quant.
 */
int bitnet_act_quant_norm(const void *X_dev, int64_t M, int64_t K, const void *norm_gain_dev,
                          float eps, int hadamard, int act_bits, void *codes_dev,
                          float *scales_dev, int32_t *rowsum_dev, bitnet_stream_t stream);

/* Debug / parity entry: Z = y (hadamard == 0) or (1/sqrt(K)) H_K y (hadamard != 0), float
 * [M, K], with y the normalised rows of bitnet_act_quant_norm (same kernels and arithmetic). */
int bitnet_norm_transform_f32(const void *X_dev, int64_t M, int64_t K, const void *norm_gain_dev,
                              float eps, int hadamard, float *Z_dev, bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* Step 4: ternary x integer product and rescale                                             */
/* ---------------------------------------------------------------------------------------- */

/*
 * acc[m, n] = sum_k codes[m, k] * q[n, k]            (exact, int32)
 * Y[m, n]   = bf16_rn(float(acc[m, n]) * (scales[m] * gamma))   (fp32 product)
 * codes/scales/rowsum as written by bitnet_act_quant; Wp/gamma as written by
 * bitnet_quantize_pack_weights.  acc_dev (int32 [M, N]) and Y_dev (bf16 [M, N]) are each
 * optional (NULL to skip); at least one must be given.  Three kernels serve the product, by token count: a weight-streaming kernel (M <= 8), a
 * tensor-core kernel with the weights on the MMA's M side and K split across a cluster of SMs
 * (9 <= M <= 64), and a tensor-core kernel over 256 x 256 output tiles (M > 64).  None keeps
 * state between calls or uses memory other than its arguments: calls on different streams may
 * run concurrently.
 */
int bitnet_ternary_gemm(const void *codes_dev, const float *scales_dev,
                        const int32_t *rowsum_dev, int64_t M, int64_t K, const void *Wp_dev,
                        const float *gamma_dev, int64_t N, int act_bits, int32_t *acc_dev,
                        void *Y_dev, bitnet_stream_t stream);

/*
 * Which kernel the product of an M x K by N x K shape takes on the current device (a query of
 * the library; the pages have no counterpart).  Every path gives the same integers.
 *   *path    BITNET_PATH_DECODE    weight-streaming kernel on the CUDA cores (M <= 8 tokens);
 *            BITNET_PATH_TC        tensor-core kernel (M > 64; INT8, or INT4 with K < 8192),
 *                                  one pass over K per 256 x 256 tile, both operands in shared
 *                                  memory;
 *            BITNET_PATH_TC_TMEM   tensor-core kernel (M > 64, INT4, K >= 8192), one pass over K
 *                                  per 256-feature x 256-token tile, the unpacked weights in
 *                                  tensor memory (the MMA's A operand);
 *            BITNET_PATH_TC_SKINNY tensor-core kernel for 9 <= M <= 64: 128 output features per
 *                                  CTA, K cut into *k_split chunks over a cluster of CTAs.
 *   *k_split chunks of K per output feature block (1 unless BITNET_PATH_TC_SKINNY).
 * Shape and act_bits rules and errors as bitnet_ternary_gemm; enqueues nothing.
 */
typedef enum {
    BITNET_PATH_DECODE = 1,
    BITNET_PATH_TC = 2,
    BITNET_PATH_TC_SKINNY = 3,
    BITNET_PATH_TC_TMEM = 4
} bitnet_product_path;

int bitnet_product_plan(int64_t M, int64_t K, int64_t N, int act_bits, int *path, int *k_split);

/*
 * Which kernel quantises the activations of a K-wide row (a query of the library, host only: it
 * touches no device and enqueues nothing; the pages have no counterpart).  Every path gives the
 * same codes up to the near-tie flips the activation entries document.
 *   *path  BITNET_QUANT_PLAIN        per-token absmax / absmean rule on the raw row (hadamard 0);
 *          BITNET_QUANT_FWHT         fast Walsh-Hadamard transform in registers, then the rule;
 *          BITNET_QUANT_HADAMARD_TC  H_K = H_128 (x) H_(K/128) with the H_128 factor as bf16
 *                                    tensor-core products (K = 8192 or 16384, no RMS norm).
 * hadamard, norm: as the activation entries (norm != 0 for the bitnet_act_quant_norm family).
 * Errors: BITNET_ERR_INVALID for K not a positive multiple of 128 or a null path,
 * BITNET_ERR_UNSUPPORTED for hadamard != 0 with K not a power of two in [128, 32768].
 */
typedef enum {
    BITNET_QUANT_PLAIN = 1,
    BITNET_QUANT_FWHT = 2,
    BITNET_QUANT_HADAMARD_TC = 3
} bitnet_quant_path;

int bitnet_act_quant_plan(int64_t K, int hadamard, int norm, int *path);

/*
 * Activations fused into the product's epilogue, for the up / gate projections that feed the
 * FFN (BitNet b1.58 2B4T article, section 一.3: squared ReLU; BitNet v2 write-up: SwishGLU).
 * With y = float(acc) * (scales[m] * gamma) as in bitnet_ternary_gemm:
 *   BITNET_ACT_RELU2   Y[m, n] = bf16_rn(max(y, 0) * max(y, 0))                Y bf16 [M, N]
 *   BITNET_ACT_SWIGLU  Y[m, j] = bf16_rn(silu(y[m, 2j]) * y[m, 2j + 1])         Y bf16 [M, N/2]
 * silu(x) = x / (1 + exp(-x)).  For SwiGLU the weight rows are interleaved: feature 2j is the
 * gate projection and 2j + 1 the up projection of output j, and N % 16 == 0.  Other arguments
 * as bitnet_ternary_gemm (only the bf16 output); an unknown activation is BITNET_ERR_INVALID.
 */
typedef enum { BITNET_ACT_RELU2 = 1, BITNET_ACT_SWIGLU = 2 } bitnet_activation;

int bitnet_ternary_gemm_act(const void *codes_dev, const float *scales_dev,
                            const int32_t *rowsum_dev, int64_t M, int64_t K, const void *Wp_dev,
                            const float *gamma_dev, int64_t N, int act_bits, int activation,
                            void *Y_dev, bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* The whole layer                                                                          */
/* ---------------------------------------------------------------------------------------- */

/* Bytes of workspace the two forward calls need: codes + scales + rowsums, 256-byte aligned. */
size_t bitnet_workspace_bytes(int64_t M, int64_t K, int64_t N, int act_bits);

/*
 * Y = BitLinear(X): per-token absmax quantisation of X (no transform), then the ternary
 * product with Wp and the rescale to bf16.  X_dev bf16 [M, K], Y_dev bf16 [M, N],
 * ws_dev scratch of ws_bytes >= bitnet_workspace_bytes(M, K, N, act_bits).
 */
int bitnet_bitlinear_forward(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                             const float *gamma_dev, int64_t N, int act_bits, void *Y_dev,
                             void *ws_dev, size_t ws_bytes, bitnet_stream_t stream);

/* Y = H-BitLinear(X): as bitnet_bitlinear_forward with the online Hadamard transform before
 * the quantisation (BitNet v2 write-up: used for the attention output projection Wo and the
 * FFN down projection Wdown).  K must be a power of two. */
int bitnet_hbitlinear_forward(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                              const float *gamma_dev, int64_t N, int act_bits, void *Y_dev,
                              void *ws_dev, size_t ws_bytes, bitnet_stream_t stream);

/* Y = BitLinear(RMSNorm(X)) (hadamard == 0) or H-BitLinear(RMSNorm(X)) (hadamard != 0): the
 * layer with the normalisation of bitnet_act_quant_norm fused into its quantiser.  Arguments
 * as bitnet_act_quant_norm and bitnet_bitlinear_forward; the same workspace size. */
int bitnet_norm_bitlinear_forward(const void *X_dev, int64_t M, int64_t K,
                                  const void *norm_gain_dev, float eps, int hadamard,
                                  const void *Wp_dev, const float *gamma_dev, int64_t N,
                                  int act_bits, void *Y_dev, void *ws_dev, size_t ws_bytes,
                                  bitnet_stream_t stream);

/* Y = act(BitLinear(X)) (hadamard == 0) or act(H-BitLinear(X)): the layer with the activation of
 * bitnet_ternary_gemm_act in its epilogue.  Y is bf16 [M, N] or [M, N/2] (SwiGLU). */
int bitnet_bitlinear_forward_act(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                                 const float *gamma_dev, int64_t N, int act_bits, int hadamard,
                                 int activation, void *Y_dev, void *ws_dev, size_t ws_bytes,
                                 bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* Variant: weight + activation Hadamard rotation                                            */
/* ---------------------------------------------------------------------------------------- */

/*
 * The BitNet v2 write-up's ablation rotates the weights as well as the activations (Hadamard
 * rotation of weights + activations, or of activations only).  With the orthonormal, symmetric
 * H' = H_K / sqrt(K) (Sylvester order), W x = (W H')(H' x): the activation half is
 * bitnet_hbitlinear_forward unchanged, and this call prepares the weight half.  Per weight row:
 *   w' = H' w computed in fp32 by the transform of bitnet_fwht_f32 (the same kernel), then
 *   gamma = fp32(max(mean |w'|, 1e-5)) (sum in double), q = RoundClip(w' / gamma, -1, 1) with an
 *   IEEE fp32 division and round-half-to-even, packed as bitnet_quantize_pack_weights.
 * K must be a power of two in [128, 32768] (else BITNET_ERR_UNSUPPORTED) and N a multiple of 8.
 * ws_dev: ws_bytes >= bitnet_weight_workspace_bytes_rotated(N, K) (the fp32 rotated rows, 4NK
 * bytes, then the partial sums); contents undefined afterwards.  Use the result with
 * bitnet_hbitlinear_forward.
 */
size_t bitnet_weight_workspace_bytes_rotated(int64_t N, int64_t K);

int bitnet_quantize_pack_weights_rotated(const void *W_dev, int64_t N, int64_t K, void *Wp_dev,
                                         float *gamma_dev, void *ws_dev, size_t ws_bytes,
                                         bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* Variant INT4 quantiser with an absmax scale                                               */
/* ---------------------------------------------------------------------------------------- */

/*
 * The INT4 path (act_bits 4) uses the absmean rule above.  This variant quantises to INT4 with
 * absmax instead, the INT8 rule with Q = 7 (the BitNet v2 write-up names absmax for the 4-bit
 * activations of the post-training baselines it compares against).  Per token row, with
 * z = (1/sqrt(K)) H_K x (hadamard != 0) or z = x:
 *   mx = max(max_k |z_k|, 1e-5); s = 7 / mx (IEEE fp32); codes = round_half_even(z * s) in
 *   [-7, 7]; scales[m] = mx / 7; rowsum[m] = sum_k codes.
 * Outputs in the INT4 layout of bitnet_act_quant (act_bits 4), so bitnet_ternary_gemm with
 * act_bits 4 consumes them.  Shapes, alignment and errors as bitnet_act_quant.
 */
int bitnet_act_quant_absmax4(const void *X_dev, int64_t M, int64_t K, int hadamard,
                             void *codes_dev, float *scales_dev, int32_t *rowsum_dev,
                             bitnet_stream_t stream);

/* The whole layer with this quantiser: bitnet_act_quant_absmax4, then the product with act_bits
 * 4.  ws_bytes >= bitnet_workspace_bytes(M, K, N, 4); other arguments as
 * bitnet_bitlinear_forward. */
int bitnet_bitlinear_forward_absmax4(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                                     const float *gamma_dev, int64_t N, int hadamard, void *Y_dev,
                                     void *ws_dev, size_t ws_bytes, bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* Base-3 weights for decode                                                                */
/* ---------------------------------------------------------------------------------------- */

/*
 * Five ternary weights in one byte (BitNet b1.58 2B4T article, section 一.1: 3^5 = 243 <= 256,
 * 1.6 bits a weight instead of 2), for the weight-streaming product of a few tokens, which is
 * bound by the bytes of weights it reads.
 * Layout: row n is ceil(K/20) little-endian 32-bit words; byte i (0..3) of word w holds the
 * offset codes u = q + 1 of weights k = 20w + 5i .. 20w + 5i + 4 as the base-3 number
 * u0*81 + u1*27 + u2*9 + u3*3 + u4, the first weight most significant (the article's example:
 * codes 2,0,1,2,1 -> byte 178).  Weights k >= K (the last word of a row) are stored as u = 1.
 */

/* Bytes of base-3 weights for an [N, K] matrix: N * 4 * ceil(K / 20). */
size_t bitnet_base3_weight_bytes(int64_t N, int64_t K);

/*
 * absmean ternarisation exactly as bitnet_quantize_pack_weights (same gamma, same q for every
 * weight), stored in the base-3 layout above.  Wp3_dev out: bitnet_base3_weight_bytes(N, K)
 * bytes; other arguments, shapes and errors as bitnet_quantize_pack_weights.
 */
int bitnet_quantize_pack_weights_base3(const void *W_dev, int64_t N, int64_t K, void *Wp3_dev,
                                       float *gamma_dev, void *ws_dev, size_t ws_bytes,
                                       bitnet_stream_t stream);

/*
 * The product of bitnet_ternary_gemm / bitnet_ternary_gemm_act on base-3 weights, for
 * M <= 8 tokens (else BITNET_ERR_UNSUPPORTED) and INT8 codes (as written by bitnet_act_quant
 * with act_bits 8).  activation: 0 (none), BITNET_ACT_RELU2 or BITNET_ACT_SWIGLU, with the
 * outputs of bitnet_ternary_gemm_act; acc_dev (int32 [M, N], exact) only with activation 0.
 * acc_dev and Y_dev are each optional; at least one must be given.  A byte above 242 in Wp3 is
 * not a valid store and gives unspecified (but in-bounds) results.
 */
int bitnet_ternary_gemv_base3(const void *codes_dev, const float *scales_dev,
                              const int32_t *rowsum_dev, int64_t M, int64_t K,
                              const void *Wp3_dev, const float *gamma_dev, int64_t N,
                              int activation, int32_t *acc_dev, void *Y_dev,
                              bitnet_stream_t stream);

/*
 * The whole layer on base-3 weights for M <= 8 tokens: INT8 per-token quantisation (with the
 * online Hadamard transform when hadamard != 0, as bitnet_hbitlinear_forward), then
 * bitnet_ternary_gemv_base3 with the given activation (0 for none) into Y_dev (bf16 [M, N], or
 * [M, N/2] for SwiGLU).  ws_dev: ws_bytes >= bitnet_workspace_bytes(M, K, N, 8).
 */
int bitnet_bitlinear_forward_base3(const void *X_dev, int64_t M, int64_t K, const void *Wp3_dev,
                                   const float *gamma_dev, int64_t N, int hadamard,
                                   int activation, void *Y_dev, void *ws_dev, size_t ws_bytes,
                                   bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* Low-bit Q / K / V states                                                                 */
/* ---------------------------------------------------------------------------------------- */

/*
 * The BitNet v2 write-up's Tables 2 and 3 vary the bit width of the attention's Q, K and V states
 * (a 3-bit KV cache matches full precision); the quantiser's formula is not printed.  This is the
 * activations' absmax rule applied per token (group = C) or per head (group = head_dim):
 *   per row m and group j of `group` consecutive features:
 *   mx = max(max |x| over the group, 1e-5);  s = Q / mx (IEEE fp32), Q = 2^(bits-1) - 1;
 *   codes = clip(round_half_even(fl32(x * s)), -Q-1, Q);  scales[m * (C / group) + j] = mx / Q.
 * X_dev       bf16 [M, C] states (e.g. the Q, K or V projection's output), 16-byte aligned.
 * codes_dev   out: bitnet_state_codes_bytes(M, C, bits) bytes; row m is a little-endian bit
 *             stream of C two's complement fields, code k in bits bits*k .. bits*k + bits - 1
 *             (bits = 3: eight codes in three bytes).  16-byte aligned.
 * scales_dev  out: float [M, C / group].
 * group % 32 == 0, C % group == 0, 2 <= bits <= 8, else BITNET_ERR_INVALID.
 */
size_t bitnet_state_codes_bytes(int64_t M, int64_t C, int bits);

int bitnet_quant_states(const void *X_dev, int64_t M, int64_t C, int64_t group, int bits,
                        void *codes_dev, float *scales_dev, bitnet_stream_t stream);

/* ---------------------------------------------------------------------------------------- */
/* Status                                                                                   */
/* ---------------------------------------------------------------------------------------- */

/* Synchronises `stream`, then returns BITNET_ERR_CUDA if the stream reported a fault,
 * BITNET_ERR_TIMEOUT if a kernel of this library on the current device gave up a bounded
 * wait since the last call (the flag is cleared), else BITNET_OK. */
int bitnet_sync_status(bitnet_stream_t stream);

/*
 * Self-test of the failure detection (a library facility; the pages have no counterpart).
 * Every wait inside the library's kernels is bounded: a phase that does not complete within
 * ~1 s makes the kernel record BITNET_ERR_TIMEOUT, wind down and return, and the next
 * bitnet_sync_status() reports it.  This call enqueues one small kernel that runs that same
 * bounded wait on a barrier nothing ever arrives on, giving up after limit_cycles SM clock cycles
 * (1 .. 2e9, else BITNET_ERR_INVALID).  It neither faults nor hangs the GPU; afterwards
 * bitnet_sync_status(stream) returns BITNET_ERR_TIMEOUT once and the context stays usable.
 */
int bitnet_selftest_wait_timeout(int64_t limit_cycles, bitnet_stream_t stream);

/* Number of kernel launches this library has issued in this process (all devices). */
uint64_t bitnet_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* BITNET_B200_H */
