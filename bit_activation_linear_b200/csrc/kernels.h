// kernels.h -- internal launchers of libbitnet_b200.so (not part of the C ABI).
// Every launcher enqueues on `stream` and returns the cudaError_t of its launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bitnet {

// ---- step 1: weights (weights.cu) ----
int absmean_num_partials(int64_t n);
cudaError_t launch_absmean_partials(const void *W, int64_t n, double *partials, int P,
                                    cudaStream_t stream);
cudaError_t launch_ternarize_pack(const void *W, int64_t n, const double *partials, int P,
                                  uint32_t *Wp, float *gamma, cudaStream_t stream);
// absmean ternarisation and 2-bit pack of fp32 weights (the Hadamard-rotated rows): two
// launches, the partial sums into partials[P].
cudaError_t launch_ternarize_pack_f32(const float *W, int64_t n, double *partials, int P,
                                      uint32_t *Wp, float *gamma, cudaStream_t stream);

// Base-3 rows (five weights per byte, ceil(K/20) 32-bit words per row) for the decode product.
cudaError_t launch_ternarize_pack_base3(const void *W, int64_t N, int64_t K,
                                        const double *partials, int P, uint32_t *Wp3,
                                        float *gamma, cudaStream_t stream);
// Device address (current device) and size of the library's fixed partial-sum scratch.
cudaError_t noalloc_partials_address(double **ptr, size_t *bytes);

// ---- steps 2-3: activations (actquant.cu) ----
// Optional RMS normalisation of each row before the transform / quantisation:
// y = (x * rinv) * g, rinv = 1 / sqrt(sum(x^2) / K + eps), g bf16 [K] (nullptr: unit gain).
struct NormArgs {
    bool on = false;
    const void *gain = nullptr;
    float eps = 0.f;
};
// Hadamard + quantise (or z output when zout != nullptr).  K = 2^logk, 7 <= logk <= 15.
cudaError_t launch_fwht_quant(const void *X, int64_t M, int logk, int act_bits,
                              const NormArgs &nrm, void *codes, float *scales, int32_t *rowsum,
                              float *zout, int *status, cudaStream_t stream);
// act_bits 8: absmax INT8; act_bits 4: absmean INT4 (the mean |z| of a token maps to code
// sqrt(7), clipped to [-8, 7]).  kActInt4Absmax selects the variant absmax INT4 quantiser (Q = 7;
// INT4 codes, layout as act_bits 4); the launchers reject it together with a norm or a z output.
constexpr int kActInt4Absmax = 0x204;

// The transform with its first seven butterfly levels as a tensor-core product (hadamard_tc.cu),
// for K = 2^logk with hadamard_tc_supported(logk) and no norm: the same outputs as
// launch_fwht_quant (codes, scales, rowsum; or z when zout != nullptr).  encode is
// cuTensorMapEncodeTiled.
bool hadamard_tc_supported(int logk);
cudaError_t launch_hadamard_tc(const void *X, int64_t M, int logk, int act_bits, void *codes,
                               float *scales, int32_t *rowsum, float *zout, int *status,
                               void *encode_fn, int num_sms, cudaStream_t stream);

// Quantise without a transform; K % 128 == 0.  zout != nullptr (with nrm.on) writes the
// normalised rows in fp32 instead of codes.
cudaError_t launch_act_quant_plain(const void *X, int64_t M, int64_t K, int act_bits,
                                   const NormArgs &nrm, void *codes, float *scales,
                                   int32_t *rowsum, float *zout, cudaStream_t stream);

// ---- step 4: product (gemv.cu, gemm_tc.cu) ----
struct GemmArgs {
    const void *codes;      // int8 [M][K] or packed int4 [M][K/2]
    const float *scales;    // [M]
    const int32_t *rowsum;  // [M]
    const uint32_t *Wp;     // [N][K/16]
    const float *gamma;     // [1]
    int64_t M, N, K;
    int act_bits;
    int32_t *acc;           // optional int32 [M][N]
    void *Y;                // optional bf16 [M][N]
    int *status;            // device status word
    // The packed weights were complete before the kernel that precedes this launch in the
    // stream started (true when the library's own quantiser runs in between, as in the forward
    // entries): the decode kernel may then load them before waiting for that kernel.
    bool early_weights = false;
    // 0: Y = rescaled output; 1: squared ReLU of it; 2: SwiGLU over interleaved gate/up
    // features (Y has N/2 columns)
    int activation = 0;
};

// Weight-streaming kernel for few tokens (decode).
constexpr int kGemvMaxTokens = 8;
cudaError_t launch_ternary_gemv(const GemmArgs &a, cudaStream_t stream);

// Weight-streaming kernel on base-3 rows (INT8 codes, M <= kGemvMaxTokens); a.Wp points at the
// base-3 words.
cudaError_t launch_ternary_gemv_base3(const GemmArgs &a, cudaStream_t stream);

// tcgen05 tensor-core kernel (prefill), one pass over K per 256 x 256 tile.  encode is
// cuTensorMapEncodeTiled.
cudaError_t launch_ternary_gemm_tc(const GemmArgs &a, void *encode_fn, int num_sms,
                                   cudaStream_t stream, int *launches = nullptr);

// tcgen05 tensor-core kernel (prefill) on CTA pairs with the unpacked weights in tensor memory
// (operand A) and 256-feature x 192-token tiles (gemm_pair_ts.cu).
cudaError_t launch_ternary_gemm_pair_ts(const GemmArgs &a, void *encode_fn, int num_sms,
                                        cudaStream_t stream, int *launches = nullptr);
// The product of INT4 codes with K >= kPairTsMinK takes it: its single accumulator makes a
// tile's MMAs wait for the previous tile's epilogue, which short K axes cannot hide (measured on
// B200: slower than the shared-memory kernel at K <= 4096, faster from K = 8192).
constexpr int64_t kPairTsMinK = 8192;
inline bool use_pair_ts(int act_bits, int64_t K) { return act_bits == 4 && K >= kPairTsMinK; }

// tcgen05 tensor-core kernel for kGemvMaxTokens < M <= kSkinnyMaxTokens: weights on the MMA's M
// side, streamed once, K split over a cluster (gemm_skinny.cu).  One launch.
constexpr int kSkinnyMaxTokens = 64;
cudaError_t launch_ternary_gemm_skinny(const GemmArgs &a, void *encode_fn, cudaStream_t stream);
// CTAs per cluster (K chunks per feature block) that launch takes on the current device.
int ternary_gemm_skinny_split(int64_t N, int64_t K);

// 2-D tiled tensor map over a row-major array (no interleave, 256-byte L2 promotion, zero fill).
CUresult encode_tmap_2d(void *encode_fn, CUtensorMap *map, CUtensorMapDataType dt,
                        const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                        uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

// ---- low-bit Q / K / V states (states.cu) ----
// Per (token, group) absmax codes of `bits` bits (2..8) as little-endian row bit streams, one
// fp32 scale per group.  group % 32 == 0, C % group == 0.
cudaError_t launch_quant_states(const void *X, int64_t M, int64_t C, int64_t group, int bits,
                                void *codes, float *scales, cudaStream_t stream);

// ---- failure detection self-test (selftest.cu) ----
cudaError_t launch_selftest_wait_timeout(long long limit_cycles, int *status,
                                         cudaStream_t stream);

}  // namespace bitnet
