// gemv.cu -- step 4 for a handful of tokens (decode): the ternary x integer product streamed
// straight from the packed weights, bound by HBM bandwidth on the 2-bit weight stream.
//
// 2B4T article, section 一.2: with ternary weights the matrix product is additions and
// subtractions only.  Here the weights stay as the stored offset codes u = q + 1 in {0,1,2}:
// one shift-and-mask turns 16 packed weights into four words of four bytes, and dp4a against
// the matching four activation codes accumulates sum_k u * c exactly; the per-token code sum
// written by the quantiser removes the offset: sum_k q * c = sum_k u * c - sum_k c.
//
// One warp per output feature n; each lane streams 64 weights (one 16-byte load) per step, so a
// warp reads 2 KB of consecutive packed weights per step.  Activation codes (at most 8 tokens,
// a few KB) stay in L1/L2.
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

template <int BITS, int T>
__global__ void __launch_bounds__(256)
    ternary_gemv_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales,
                        const int32_t *__restrict__ rowsum, int M, int K,
                        const uint4 *__restrict__ wp, const float *__restrict__ gamma_ptr, int N,
                        int32_t *__restrict__ acc_out, __nv_bfloat16 *__restrict__ Y) {
    const int lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (n >= N) return;
    const uint4 *wrow = wp + (int64_t)n * (K / 64);  // 64 weights per uint4
    int acc[T];
#pragma unroll
    for (int t = 0; t < T; ++t) acc[t] = 0;

    for (int c = lane; c < K / 64; c += 32) {
        const uint4 w4 = ldg_nc_v4(wrow + c);
        const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
        // unpacked offset codes: u[4g + p] holds weights 64c + 16g + 4p .. +3
        uint32_t u[16];
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
            for (int p = 0; p < 4; ++p) u[4 * g + p] = (ww[g] >> (2 * p)) & 0x03030303u;
#pragma unroll
        for (int t = 0; t < T; ++t) {
            if (t >= M) break;
            if constexpr (BITS == 8) {
                const uint4 *xr = reinterpret_cast<const uint4 *>(codes + (int64_t)t * K) + 4 * c;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint4 x = __ldg(xr + g);
                    acc[t] = __dp4a((int)u[4 * g + 0], (int)x.x, acc[t]);
                    acc[t] = __dp4a((int)u[4 * g + 1], (int)x.y, acc[t]);
                    acc[t] = __dp4a((int)u[4 * g + 2], (int)x.z, acc[t]);
                    acc[t] = __dp4a((int)u[4 * g + 3], (int)x.w, acc[t]);
                }
            } else {
                // nibble storage: each 32-bit word holds codes k0..k0+3 (low nibbles) and
                // k0+4..k0+7 (high nibbles)
                const uint4 *xr =
                    reinterpret_cast<const uint4 *>(codes + (int64_t)t * (K / 2)) + 2 * c;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint4 x = __ldg(xr + h);
                    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int word = 4 * h + i;  // codes 8*word .. 8*word+7 of this 64
                        uint32_t lo = sext_nibbles(xw[i] & 0x0F0F0F0Fu);
                        uint32_t hi = sext_nibbles((xw[i] >> 4) & 0x0F0F0F0Fu);
                        acc[t] = __dp4a((int)u[2 * word], (int)lo, acc[t]);
                        acc[t] = __dp4a((int)u[2 * word + 1], (int)hi, acc[t]);
                    }
                }
            }
        }
    }
    const float gamma = *gamma_ptr;
#pragma unroll
    for (int t = 0; t < T; ++t) {
        if (t >= M) break;
        int s = acc[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
        if (lane == t) {
            const int a = s - rowsum[t];
            if (acc_out) acc_out[(int64_t)t * N + n] = a;
            if (Y) Y[(int64_t)t * N + n] = __float2bfloat16_rn((float)a * (scales[t] * gamma));
        }
    }
}

template <int BITS, int T>
static cudaError_t launch_gemv_t(const GemmArgs &a, cudaStream_t stream) {
    const unsigned blocks = (unsigned)((a.N + 7) / 8);
    ternary_gemv_kernel<BITS, T><<<blocks, 256, 0, stream>>>(
        reinterpret_cast<const uint8_t *>(a.codes), a.scales, a.rowsum, (int)a.M, (int)a.K,
        reinterpret_cast<const uint4 *>(a.Wp), a.gamma, (int)a.N, a.acc,
        reinterpret_cast<__nv_bfloat16 *>(a.Y));
    return cudaGetLastError();
}

template <int BITS>
static cudaError_t launch_gemv_b(const GemmArgs &a, cudaStream_t stream) {
    if (a.M <= 1) return launch_gemv_t<BITS, 1>(a, stream);
    if (a.M <= 2) return launch_gemv_t<BITS, 2>(a, stream);
    if (a.M <= 4) return launch_gemv_t<BITS, 4>(a, stream);
    return launch_gemv_t<BITS, 8>(a, stream);
}

cudaError_t launch_ternary_gemv(const GemmArgs &a, cudaStream_t stream) {
    if (a.M > kGemvMaxTokens) return cudaErrorInvalidValue;
    return a.act_bits == 4 ? launch_gemv_b<4>(a, stream) : launch_gemv_b<8>(a, stream);
}

}  // namespace bitnet
