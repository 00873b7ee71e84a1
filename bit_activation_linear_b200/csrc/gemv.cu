// gemv.cu -- step 4 for a handful of tokens (decode): the ternary x integer product streamed
// straight from the packed weights, bound by HBM bandwidth on the weight stream.
//
// 2B4T article, section 一.2: with ternary weights the matrix product is additions and
// subtractions only.  Here the weights stay as the stored offset codes u = q + 1 in {0,1,2}:
// one shift-and-mask turns 16 packed weights into four words of four bytes, and dp4a against
// the matching four activation codes accumulates sum_k u * c exactly; the per-token code sum
// written by the quantiser removes the offset: sum_k q * c = sum_k u * c - sum_k c.
//
// A row group of R consecutive output features is owned by KS warps of one CTA (KS = 1, 2 or
// 4: when a matrix has few row groups, long rows are split so that it still fills the GPU).  The
// K axis is walked in steps of 512 weights, step s going to warp s mod KS of the group: in a step
// lane l takes the packed word 32s + l of each row (weights k = 512s + 16l .. +15, one coalesced
// 128-byte load per warp and row) and the 16 matching codes of each token (one coalesced 16-byte
// load per lane).  The weight words of S steps are loaded before any is used, so every warp keeps
// S*R loads in flight and the weight stream is requested at full rate.  Every code is loaded once
// per R rows, so R grows with the token count (1 row for 1-2 tokens, 2 for 3-8, and 4 for 5-8
// tokens when N >= 8192) to keep the L1 traffic of the code loads down.  Activation codes (at
// most eight tokens) are read through L1, where every warp of the SM finds them.  The lanes'
// partial sums are reduced with shuffles, then across the group's warps through shared memory,
// and the group's first warp writes the results.
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

constexpr int kGemvWarps = 4;  // warps per CTA

// d = c + sum_j a.u8[j] * b.s8[j]: unsigned bytes of a against signed bytes of b
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Reduce the lanes' partial sums (shuffles), then the KS warps' partial sums of the row group
// (shared memory, one barrier for the whole CTA), remove the weight offset with the code sums and
// write the results from the group's first warp: lane r*T + t stores (row n0 + r, token t).
// ACT: 0 rescaled output, 1 squared ReLU of it, 2 SwiGLU over row pairs (gate, up = features
// 2j, 2j+1 = rows n0 + 2p, n0 + 2p + 1; output column j = n0/2 + p, written by lane p*T + t).
// Every thread of the CTA must call it (it contains __syncthreads when KS > 1).
template <int T, int R, int KS, int ACT>
__device__ __forceinline__ void gemv_finish(const int (&acc)[R][T], int (*red)[R * T],
                                            bool active, int lane, int n0, int M, int N,
                                            const float *__restrict__ scales,
                                            const int32_t *__restrict__ rowsum,
                                            const float *__restrict__ gamma_ptr,
                                            int32_t *__restrict__ acc_out,
                                            __nv_bfloat16 *__restrict__ Y) {
    static_assert(ACT != 2 || R % 2 == 0, "SwiGLU needs the gate and up rows in one group");
    const int warp = threadIdx.x >> 5;
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
    if constexpr (KS > 1) {
        if (lane == 0)
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int t = 0; t < T; ++t) red[warp][r * T + t] = sums[r][t];
        __syncthreads();
        if (warp % KS != 0) return;
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < T; ++t) {
                int s = sums[r][t];
#pragma unroll
                for (int w = 1; w < KS; ++w) s += red[warp + w][r * T + t];
                sums[r][t] = s;
            }
    }
    if (!active) return;
    const float gamma = *gamma_ptr;
#pragma unroll
    for (int t = 0; t < T; ++t) {
        if (t >= M) break;
        const float sc = scales[t] * gamma;
        if constexpr (ACT == 2) {
#pragma unroll
            for (int p = 0; p < R / 2; ++p) {
                if (lane == p * T + t && n0 + 2 * p + 1 < N) {
                    const float g = (float)(sums[2 * p][t] - rowsum[t]) * sc;
                    const float u = (float)(sums[2 * p + 1][t] - rowsum[t]) * sc;
                    Y[(int64_t)t * (N / 2) + n0 / 2 + p] =
                        __float2bfloat16_rn(__fdiv_rn(g, 1.f + expf(-g)) * u);
                }
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

// Warps per row group.  With 1024 or more row groups the GPU has enough warps and a split only
// adds CTAs and a barrier (measured slower); with fewer, long rows are split so that every warp
// still walks at least ~4 steps.
static int gemv_split(int64_t groups, int steps) {
    if (groups >= 1024) return 1;
    return steps >= 16 ? 4 : steps >= 8 ? 2 : 1;
}

// ACT as in gemv_finish; S = steps whose weight loads are in flight together.
template <int BITS, int T, int R, int S, int KS, int ACT>
__global__ void __launch_bounds__(kGemvWarps * 32)
    ternary_gemv_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales,
                        const int32_t *__restrict__ rowsum, int M, int K,
                        const uint32_t *__restrict__ wp, const float *__restrict__ gamma_ptr,
                        int N, int32_t *__restrict__ acc_out, __nv_bfloat16 *__restrict__ Y,
                        int early_weights) {
    __shared__ int red[kGemvWarps][R * T];
    if (!early_weights) pdl_wait();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ks = warp % KS;
    const int n0 = (blockIdx.x * (kGemvWarps / KS) + warp / KS) * R;
    const bool active = n0 < N;
    const int words = K / 16;             // packed words per row
    const int steps = (words + 31) / 32;  // the last step may be partial (K % 512 != 0)
    const int mine = active && steps > ks ? (steps - ks + KS - 1) / KS : 0;  // this warp's steps
    int acc[R][T];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < T; ++t) acc[r][t] = 0;
    // With few (row, token) pairs, each 2-bit field p of a word is masked in place instead of
    // shifted down: byte j of w & (0x03030303 << 2p) holds 4^p u, so its dot product is 4^p
    // times the field's, kept in a sum of its own and scaled back (an exact shift: every term is
    // a multiple of 4^p) once per batch of S steps: a batch adds S * 4 terms of at most
    // 64 * 2 * 128 in magnitude to a field sum, far below 2^31.
    // One mask instead of a shift and a mask per field and dot product.
    constexpr bool FIELD_SUMS = R * T <= 4;
    int fs[FIELD_SUMS ? R : 1][FIELD_SUMS ? T : 1][4];

    for (int b0 = 0; b0 < mine; b0 += S) {
        if constexpr (FIELD_SUMS) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int t = 0; t < T; ++t)
#pragma unroll
                    for (int p = 0; p < 4; ++p) fs[r][t][p] = 0;
        }
        uint32_t w[R][S];
#pragma unroll
        for (int j = 0; j < S; ++j) {
            const int wi = 32 * (ks + KS * (b0 + j)) + lane;
#pragma unroll
            for (int r = 0; r < R; ++r)
                w[r][j] = (b0 + j < mine && wi < words && n0 + r < N)
                              ? __ldg(wp + (int64_t)(n0 + r) * words + wi)
                              : 0u;
        }
        // With early_weights the packed weights were complete before the kernel that wrote the
        // codes started, so they are loaded before waiting for that kernel (programmatic
        // dependent launch); the codes, scales and code sums are always read after the wait.
        if (early_weights && b0 == 0) pdl_wait();
#pragma unroll
        for (int j = 0; j < S; ++j) {
            if (b0 + j >= mine) break;
            const int k0 = 512 * (ks + KS * (b0 + j)) + 16 * lane;
            const bool k_in = k0 < K;  // lanes past the end of a partial step add zero
            // codes k0 .. k0+15 of every token as four words of four int8 (word p = k0+4p .. +3)
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
                    if constexpr (FIELD_SUMS) {
                        const uint32_t um = w[r][j] & (0x03030303u << (2 * p));
#pragma unroll
                        for (int t = 0; t < T; ++t) fs[r][t][p] = dp4a_us(um, xs[t][p], fs[r][t][p]);
                    } else {
                        const int u = (int)((w[r][j] >> (2 * p)) & 0x03030303u);
#pragma unroll
                        for (int t = 0; t < T; ++t) acc[r][t] = __dp4a(u, (int)xs[t][p], acc[r][t]);
                    }
                }
        }
        if constexpr (FIELD_SUMS) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int t = 0; t < T; ++t)
                    acc[r][t] += fs[r][t][0] + (fs[r][t][1] >> 2) + (fs[r][t][2] >> 4) +
                                 (fs[r][t][3] >> 6);
        }
    }
    // the scales and code sums are read below: make sure this warp has waited
    if (early_weights && mine == 0) pdl_wait();
    gemv_finish<T, R, KS, ACT>(acc, red, active, lane, n0, M, N, scales, rowsum, gamma_ptr,
                               acc_out, Y);
}

// CTAs of kGemvWarps warps, row groups of R rows owned by KS warps each.
template <int R, int KS, typename Kern>
static cudaError_t launch_gemv_kernel(Kern kern, const GemmArgs &a, cudaStream_t stream) {
    const int64_t groups = (a.N + R - 1) / R;
    constexpr int per_cta = kGemvWarps / KS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((groups + per_cta - 1) / per_cta), 1, 1);
    cfg.blockDim = dim3(kGemvWarps * 32, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, reinterpret_cast<const uint8_t *>(a.codes), a.scales,
                              a.rowsum, (int)a.M, (int)a.K, a.Wp, a.gamma, (int)a.N, a.acc,
                              reinterpret_cast<__nv_bfloat16 *>(a.Y), a.early_weights ? 1 : 0);
}

template <int BITS, int T, int R, int S, int ACT>
static cudaError_t launch_gemv_t(const GemmArgs &a, cudaStream_t stream) {
    static_assert(R * T <= 32, "one lane per (row, token) result");
    switch (gemv_split((a.N + R - 1) / R, (int)((a.K / 16 + 31) / 32))) {
        case 4: return launch_gemv_kernel<R, 4>(ternary_gemv_kernel<BITS, T, R, S, 4, ACT>, a, stream);
        case 2: return launch_gemv_kernel<R, 2>(ternary_gemv_kernel<BITS, T, R, S, 2, ACT>, a, stream);
        default: return launch_gemv_kernel<R, 1>(ternary_gemv_kernel<BITS, T, R, S, 1, ACT>, a, stream);
    }
}

// Rows per group by token count: the codes of T tokens are loaded once per R rows.  Four rows
// per group only from N = 8192 up, where the groups still give every SM many warps.
template <int BITS, int ACT>
static cudaError_t launch_gemv_a(const GemmArgs &a, cudaStream_t stream) {
    constexpr int R_SMALL = ACT == 2 ? 2 : 1;  // SwiGLU keeps each row pair in one group
    if (a.M <= 1) return launch_gemv_t<BITS, 1, R_SMALL, 16, ACT>(a, stream);
    if (a.M <= 2) return launch_gemv_t<BITS, 2, R_SMALL, 16, ACT>(a, stream);
    if (a.M <= 4) return launch_gemv_t<BITS, 4, 2, 16, ACT>(a, stream);
    if (a.N >= 8192) return launch_gemv_t<BITS, 8, 4, 8, ACT>(a, stream);
    return launch_gemv_t<BITS, 8, 2, 16, ACT>(a, stream);
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
// k = 20w .. 20w + 19.  Same row groups, K split and finish as the 2-bit kernel, with steps of 640
// weights: lane l takes word 32s + l of each row.  INT8 codes only (the 20-code groups do not fall
// on the 8-code groups of the INT4 nibble layout).

template <int T, int R, int S, int KS, int ACT>
__global__ void __launch_bounds__(kGemvWarps * 32)
    ternary_gemv_base3_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales,
                              const int32_t *__restrict__ rowsum, int M, int K,
                              const uint32_t *__restrict__ wp3, const float *__restrict__ gamma_ptr,
                              int N, int32_t *__restrict__ acc_out, __nv_bfloat16 *__restrict__ Y,
                              int early_weights) {
    __shared__ int red[kGemvWarps][R * T];
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
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int ks = warp % KS;
    const int n0 = (blockIdx.x * (kGemvWarps / KS) + warp / KS) * R;
    const bool active = n0 < N;
    const int words = (K + 19) / 20;
    const int steps = (words + 31) / 32;
    const int mine = active && steps > ks ? (steps - ks + KS - 1) / KS : 0;
    int acc[R][T];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int t = 0; t < T; ++t) acc[r][t] = 0;
    // With few (row, token) pairs, each 2-bit field p of a word is masked in place instead of
    // shifted down: byte j of w & (0x03030303 << 2p) holds 4^p u, so its dot product is 4^p
    // times the field's, kept in a sum of its own and scaled back (an exact shift: every term is
    // a multiple of 4^p) once per batch of S steps: a batch adds S * 4 terms of at most
    // 64 * 2 * 128 in magnitude to a field sum, far below 2^31.
    // One mask instead of a shift and a mask per field and dot product.
    constexpr bool FIELD_SUMS = R * T <= 4;
    int fs[FIELD_SUMS ? R : 1][FIELD_SUMS ? T : 1][4];

    for (int b0 = 0; b0 < mine; b0 += S) {
        if constexpr (FIELD_SUMS) {
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int t = 0; t < T; ++t)
#pragma unroll
                    for (int p = 0; p < 4; ++p) fs[r][t][p] = 0;
        }
        uint32_t w[R][S];
#pragma unroll
        for (int j = 0; j < S; ++j) {
            const int wi = 32 * (ks + KS * (b0 + j)) + lane;
#pragma unroll
            for (int r = 0; r < R; ++r)
                w[r][j] = (b0 + j < mine && wi < words && n0 + r < N)
                              ? __ldg(wp3 + (int64_t)(n0 + r) * words + wi)
                              : 0u;  // byte 0 decodes to u = 0: adds nothing
        }
        if (early_weights && b0 == 0) pdl_wait();
#pragma unroll
        for (int j = 0; j < S; ++j) {
            if (b0 + j >= mine) break;
            const int k0 = 20 * (32 * (ks + KS * (b0 + j)) + lane);
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
    if (early_weights && mine == 0) pdl_wait();
    gemv_finish<T, R, KS, ACT>(acc, red, active, lane, n0, M, N, scales, rowsum, gamma_ptr,
                               acc_out, Y);
}

template <int T, int R, int S, int ACT>
static cudaError_t launch_gemv3_t(const GemmArgs &a, cudaStream_t stream) {
    static_assert(R * T <= 32, "one lane per (row, token) result");
    switch (gemv_split((a.N + R - 1) / R, (int)(((a.K + 19) / 20 + 31) / 32))) {
        case 4: return launch_gemv_kernel<R, 4>(ternary_gemv_base3_kernel<T, R, S, 4, ACT>, a, stream);
        case 2: return launch_gemv_kernel<R, 2>(ternary_gemv_base3_kernel<T, R, S, 2, ACT>, a, stream);
        default: return launch_gemv_kernel<R, 1>(ternary_gemv_base3_kernel<T, R, S, 1, ACT>, a, stream);
    }
}

template <int ACT>
static cudaError_t launch_gemv3_a(const GemmArgs &a, cudaStream_t stream) {
    constexpr int R_SMALL = ACT == 2 ? 2 : 1;
    if (a.M <= 1) return launch_gemv3_t<1, R_SMALL, 16, ACT>(a, stream);
    if (a.M <= 2) return launch_gemv3_t<2, R_SMALL, 16, ACT>(a, stream);
    if (a.M <= 4) return launch_gemv3_t<4, 2, 16, ACT>(a, stream);
    if (a.N >= 8192) return launch_gemv3_t<8, 4, 8, ACT>(a, stream);
    return launch_gemv3_t<8, 2, 16, ACT>(a, stream);
}

cudaError_t launch_ternary_gemv_base3(const GemmArgs &a, cudaStream_t stream) {
    if (a.M > kGemvMaxTokens || a.act_bits != 8) return cudaErrorInvalidValue;
    if (a.acc || a.activation == 0) return launch_gemv3_a<0>(a, stream);
    return a.activation == 1 ? launch_gemv3_a<1>(a, stream) : launch_gemv3_a<2>(a, stream);
}

}  // namespace bitnet
