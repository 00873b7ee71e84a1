// gemv.cu -- step 4 for a handful of tokens (decode): the ternary x integer product streamed
// straight from the packed weights, bound by HBM bandwidth on the 2-bit weight stream.
//
// 2B4T article, section 一.2: with ternary weights the matrix product is additions and
// subtractions only.  Here the weights stay as the stored offset codes u = q + 1 in {0,1,2}:
// one shift-and-mask turns 16 packed weights into four words of four bytes, and dp4a against
// the matching four activation codes accumulates sum_k u * c exactly; the per-token code sum
// written by the quantiser removes the offset: sum_k q * c = sum_k u * c - sum_k c.
//
// A warp owns R consecutive output features (R = 2 from four tokens up, so that each code load
// serves two rows).  The K axis is walked in steps of 512 weights: in a step lane l takes the
// packed word 32s + l of each row (weights k = 512s + 16l .. +15, one coalesced 128-byte load per
// warp and row) and the 16 matching codes of each token (one coalesced 16-byte load per lane).
// The weight words of eight steps are loaded before any is used, so every warp keeps 8R loads
// in flight and the weight stream is requested at full rate.  Activation codes (at most eight
// tokens) are read through L1, where every warp of the SM finds them.
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

constexpr int kGemvSteps = 16;      // 512-weight steps whose weight loads are in flight together
constexpr int kGemvWarps = 4;       // warps per CTA

// Reduce the lanes' partial sums, remove the weight offset with the code sums and write the
// results: lane r*T + t stores (row n0 + r, token t).  ACT: 0 rescaled output, 1 squared ReLU of
// it, 2 SwiGLU over the warp's two rows (gate, up = features 2j, 2j+1; output column j; R == 2).
template <int T, int R, int ACT>
__device__ __forceinline__ void gemv_epilogue(const int (&acc)[R][T], int lane, int n0, int M,
                                              int N, const float *__restrict__ scales,
                                              const int32_t *__restrict__ rowsum, float gamma,
                                              int32_t *__restrict__ acc_out,
                                              __nv_bfloat16 *__restrict__ Y) {
    static_assert(ACT != 2 || R == 2, "SwiGLU needs the gate and up rows in one warp");
    int sums[R][T];  // full sums, the same in every lane
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < T; ++t) {
            int s = acc[r][t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
            sums[r][t] = s;
        }
#pragma unroll
    for (int t = 0; t < T; ++t) {
        if (t >= M) break;
        const float sc = scales[t] * gamma;
        if constexpr (ACT == 2) {
            if (lane == t && n0 + 1 < N) {
                const float g = (float)(sums[0][t] - rowsum[t]) * sc;
                const float u = (float)(sums[1][t] - rowsum[t]) * sc;
                Y[(int64_t)t * (N / 2) + n0 / 2] = __float2bfloat16_rn(__fdiv_rn(g, 1.f + expf(-g)) * u);
            }
        } else {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int n = n0 + r;
                if (lane == r * T + t && n < N) {
                    const int a = sums[r][t] - rowsum[t];
                    if (acc_out) acc_out[(int64_t)t * N + n] = a;
                    if (Y) {
                        float y = (float)a * sc;
                        if constexpr (ACT == 1) y = y > 0.f ? y * y : 0.f;
                        Y[(int64_t)t * N + n] = __float2bfloat16_rn(y);
                    }
                }
            }
        }
    }
}

// ACT as in gemv_epilogue.
template <int BITS, int T, int R, int ACT>
__global__ void __launch_bounds__(kGemvWarps * 32)
    ternary_gemv_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales,
                        const int32_t *__restrict__ rowsum, int M, int K,
                        const uint32_t *__restrict__ wp, const float *__restrict__ gamma_ptr,
                        int N, int32_t *__restrict__ acc_out, __nv_bfloat16 *__restrict__ Y,
                        int early_weights) {
    if (!early_weights) pdl_wait();
    const int lane = threadIdx.x & 31;
    const int n0 = (blockIdx.x * kGemvWarps + (threadIdx.x >> 5)) * R;
    if (n0 >= N) return;  // whole warp leaves together (nothing of its own to wait for)
    const int words = K / 16;  // packed words per row
    const int steps = (words + 31) / 32;  // the last step may be partial (K % 512 != 0)
    int acc[R][T];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < T; ++t) acc[r][t] = 0;

    for (int s0 = 0; s0 < steps; s0 += kGemvSteps) {
        uint32_t w[R][kGemvSteps];
#pragma unroll
        for (int j = 0; j < kGemvSteps; ++j)
#pragma unroll
            for (int r = 0; r < R; ++r)
                w[r][j] = (32 * (s0 + j) + lane < words && n0 + r < N)
                              ? __ldg(wp + (int64_t)(n0 + r) * words + 32 * (s0 + j) + lane)
                              : 0u;
        // With early_weights the packed weights were complete before the kernel that wrote the
        // codes started, so they are loaded before waiting for that kernel (programmatic
        // dependent launch); the codes, scales and code sums are always read after the wait.
        if (early_weights && s0 == 0) pdl_wait();
#pragma unroll
        for (int j = 0; j < kGemvSteps; ++j) {
            if (s0 + j >= steps) break;
            const int k0 = 512 * (s0 + j) + 16 * lane;
            const bool k_in = k0 < K;  // lanes past the end of a partial step add zero
            // codes k0 .. k0+15 of every token as four words of four int8 (word p = k0+4p .. +3),
            // all loaded before the dot products (tokens t >= M read nothing and add zero)
            uint32_t xs[T][4];
#pragma unroll
            for (int t = 0; t < T; ++t) {
                uint32_t *x = xs[t];
                if (!k_in || t >= M) {
                    x[0] = x[1] = x[2] = x[3] = 0u;
                } else if constexpr (BITS == 8) {
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(codes + (int64_t)t * K + k0));
                    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
                } else {
                    // nibble storage: each word holds codes k..k+3 (low nibbles), k+4..k+7 (high)
                    const uint2 v =
                        __ldg(reinterpret_cast<const uint2 *>(codes + (int64_t)t * (K / 2) + k0 / 2));
                    x[0] = sext_nibbles(v.x & 0x0F0F0F0Fu);
                    x[1] = sext_nibbles((v.x >> 4) & 0x0F0F0F0Fu);
                    x[2] = sext_nibbles(v.y & 0x0F0F0F0Fu);
                    x[3] = sext_nibbles((v.y >> 4) & 0x0F0F0F0Fu);
                }
            }
            // packed word: weight k0 + 4p + j at bits 8j + 2p, as offset codes u = q + 1
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int u = (int)((w[r][j] >> (2 * p)) & 0x03030303u);
#pragma unroll
                    for (int t = 0; t < T; ++t) acc[r][t] = __dp4a(u, (int)xs[t][p], acc[r][t]);
                }
        }
    }
    gemv_epilogue<T, R, ACT>(acc, lane, n0, M, N, scales, rowsum, *gamma_ptr, acc_out, Y);
}

template <int BITS, int T, int R, int ACT>
static cudaError_t launch_gemv_t(const GemmArgs &a, cudaStream_t stream) {
    static_assert(R * T <= 32, "one lane per (row, token) result");
    const int64_t warps = (a.N + R - 1) / R;
    const unsigned blocks = (unsigned)((warps + kGemvWarps - 1) / kGemvWarps);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3(kGemvWarps * 32, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ternary_gemv_kernel<BITS, T, R, ACT>,
                              reinterpret_cast<const uint8_t *>(a.codes), a.scales, a.rowsum,
                              (int)a.M, (int)a.K, a.Wp, a.gamma, (int)a.N, a.acc,
                              reinterpret_cast<__nv_bfloat16 *>(a.Y), a.early_weights ? 1 : 0);
}

template <int BITS, int ACT>
static cudaError_t launch_gemv_a(const GemmArgs &a, cudaStream_t stream) {
    constexpr int R_SMALL = ACT == 2 ? 2 : 1;  // SwiGLU keeps the row pair in one warp
    if (a.M <= 1) return launch_gemv_t<BITS, 1, R_SMALL, ACT>(a, stream);
    if (a.M <= 2) return launch_gemv_t<BITS, 2, R_SMALL, ACT>(a, stream);
    if (a.M <= 4) return launch_gemv_t<BITS, 4, 2, ACT>(a, stream);
    return launch_gemv_t<BITS, 8, 2, ACT>(a, stream);
}

template <int BITS>
static cudaError_t launch_gemv_b(const GemmArgs &a, cudaStream_t stream) {
    if (a.acc || a.activation == 0) return launch_gemv_a<BITS, 0>(a, stream);
    return a.activation == 1 ? launch_gemv_a<BITS, 1>(a, stream)
                             : launch_gemv_a<BITS, 2>(a, stream);
}

cudaError_t launch_ternary_gemv(const GemmArgs &a, cudaStream_t stream) {
    if (a.M > kGemvMaxTokens) return cudaErrorInvalidValue;
    return a.act_bits == 4 ? launch_gemv_b<4>(a, stream) : launch_gemv_b<8>(a, stream);
}

// ------------------------------------------------------------------------------------------
// Base-3 weights (2B4T article, section 一.1: five ternary weights in one byte, 1.6 bits a
// weight).  Row n is ceil(K/20) 32-bit words; byte i of word w is the base-3 number of the offset
// codes of weights 20w + 5i .. +4, first weight most significant.  A 256-entry table in shared
// memory turns a byte into its five offset codes, one per byte of a 64-bit entry; the four entries
// of a word are spliced into five dp4a words of four codes each, matching the 20 activation codes
// k = 20w .. 20w + 19.  Same K walk as the 2-bit kernel with steps of 640 weights: lane l takes
// word 32s + l of each row.  INT8 codes only (the 20-code groups do not fall on the 8-code
// groups of the INT4 nibble layout).

template <int T, int R, int ACT>
__global__ void __launch_bounds__(kGemvWarps * 32)
    ternary_gemv_base3_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales,
                              const int32_t *__restrict__ rowsum, int M, int K,
                              const uint32_t *__restrict__ wp3, const float *__restrict__ gamma_ptr,
                              int N, int32_t *__restrict__ acc_out, __nv_bfloat16 *__restrict__ Y,
                              int early_weights) {
    __shared__ unsigned long long digits[256];
    for (int v = threadIdx.x; v < 256; v += kGemvWarps * 32) {
        // byte 4 - j of the entry = base-3 digit j of v (digit 0 least significant); bytes
        // 243..255 never occur in a stored row
        unsigned long long e = 0;
        int x = v;
#pragma unroll
        for (int b = 4; b >= 0; --b) {
            e |= (unsigned long long)(x % 3) << (8 * b);
            x /= 3;
        }
        digits[v] = e;
    }
    __syncthreads();
    if (!early_weights) pdl_wait();
    const int lane = threadIdx.x & 31;
    const int n0 = (blockIdx.x * kGemvWarps + (threadIdx.x >> 5)) * R;
    if (n0 >= N) return;  // whole warp leaves together (after the block's only barrier)
    const int words = (K + 19) / 20;
    const int steps = (words + 31) / 32;
    int acc[R][T];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < T; ++t) acc[r][t] = 0;

    for (int s0 = 0; s0 < steps; s0 += kGemvSteps) {
        uint32_t w[R][kGemvSteps];
#pragma unroll
        for (int j = 0; j < kGemvSteps; ++j)
#pragma unroll
            for (int r = 0; r < R; ++r)
                w[r][j] = (32 * (s0 + j) + lane < words && n0 + r < N)
                              ? __ldg(wp3 + (int64_t)(n0 + r) * words + 32 * (s0 + j) + lane)
                              : 0u;  // byte 0 decodes to u = 0: adds nothing
        if (early_weights && s0 == 0) pdl_wait();
#pragma unroll
        for (int j = 0; j < kGemvSteps; ++j) {
            if (s0 + j >= steps) break;
            const int k0 = 20 * (32 * (s0 + j) + lane);
            // codes k0 + 4p .. +3 of every token (K % 4 == 0: a group is wholly in or out)
            uint32_t xs[T][5];
#pragma unroll
            for (int t = 0; t < T; ++t)
#pragma unroll
                for (int p = 0; p < 5; ++p)
                    xs[t][p] = (t < M && k0 + 4 * p < K)
                                   ? __ldg(reinterpret_cast<const uint32_t *>(
                                         codes + (int64_t)t * K + k0 + 4 * p))
                                   : 0u;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const uint32_t v = w[r][j];
                const unsigned long long L0 = digits[v & 0xFFu], L1 = digits[(v >> 8) & 0xFFu],
                                         L2 = digits[(v >> 16) & 0xFFu], L3 = digits[v >> 24];
                // offset codes of weights k0 .. k0+19, four per word in k order
                const uint32_t u[5] = {(uint32_t)L0,
                                       (uint32_t)(L0 >> 32) | (uint32_t)(L1 << 8),
                                       (uint32_t)(L1 >> 24) | (uint32_t)(L2 << 16),
                                       (uint32_t)(L2 >> 16) | (uint32_t)(L3 << 24),
                                       (uint32_t)(L3 >> 8)};
#pragma unroll
                for (int p = 0; p < 5; ++p)
#pragma unroll
                    for (int t = 0; t < T; ++t)
                        acc[r][t] = __dp4a((int)u[p], (int)xs[t][p], acc[r][t]);
            }
        }
    }
    gemv_epilogue<T, R, ACT>(acc, lane, n0, M, N, scales, rowsum, *gamma_ptr, acc_out, Y);
}

template <int T, int R, int ACT>
static cudaError_t launch_gemv3_t(const GemmArgs &a, cudaStream_t stream) {
    static_assert(R * T <= 32, "one lane per (row, token) result");
    const int64_t warps = (a.N + R - 1) / R;
    const unsigned blocks = (unsigned)((warps + kGemvWarps - 1) / kGemvWarps);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3(kGemvWarps * 32, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ternary_gemv_base3_kernel<T, R, ACT>,
                              reinterpret_cast<const uint8_t *>(a.codes), a.scales, a.rowsum,
                              (int)a.M, (int)a.K, a.Wp, a.gamma, (int)a.N, a.acc,
                              reinterpret_cast<__nv_bfloat16 *>(a.Y), a.early_weights ? 1 : 0);
}

template <int ACT>
static cudaError_t launch_gemv3_a(const GemmArgs &a, cudaStream_t stream) {
    constexpr int R_SMALL = ACT == 2 ? 2 : 1;
    if (a.M <= 1) return launch_gemv3_t<1, R_SMALL, ACT>(a, stream);
    if (a.M <= 2) return launch_gemv3_t<2, R_SMALL, ACT>(a, stream);
    if (a.M <= 4) return launch_gemv3_t<4, 2, ACT>(a, stream);
    return launch_gemv3_t<8, 2, ACT>(a, stream);
}

cudaError_t launch_ternary_gemv_base3(const GemmArgs &a, cudaStream_t stream) {
    if (a.M > kGemvMaxTokens || a.act_bits != 8) return cudaErrorInvalidValue;
    if (a.acc || a.activation == 0) return launch_gemv3_a<0>(a, stream);
    return a.activation == 1 ? launch_gemv3_a<1>(a, stream) : launch_gemv3_a<2>(a, stream);
}

}  // namespace bitnet
