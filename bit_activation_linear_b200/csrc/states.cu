// states.cu -- low-bit quantisation of the attention's Q / K / V states.
//
// BitNet v2 write-up, Tables 2 and 3 and the paragraph before them: the bit width of the QKV
// states is varied, and a 3-bit KV cache matches full precision.  The quantiser's formula is not
// printed; the reading taken is the activations' absmax rule applied per token, or per group of
// `group` consecutive features (one attention head): Q = 2^(bits-1) - 1, s = Q / max(max|x|, 1e-5)
// (IEEE fp32), c = clip(round_half_even(fl32(x * s)), -Q-1, Q), d = max(max|x|, 1e-5) / Q.
//
// Storage: each token row is a little-endian bit stream, code k in bits bits*k .. bits*k+bits-1
// (two's complement), C * bits / 8 bytes a row.  32 consecutive codes fill exactly `bits` 32-bit
// words, so a lane that owns 32 codes writes whole, aligned words.
//
// Kernel (HBM-bound: 2 bytes in, bits/8 bytes out per element): one warp per (token, group)
// segment.  Pass 1 takes max|x| with 16-byte loads; pass 2 (the segment is in L1 / L2 by then)
// gives each lane 32 consecutive values, which it turns into `bits` words of the stream.
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

template <int BITS>
__global__ void __launch_bounds__(256)
    quant_states_kernel(const uint4 *__restrict__ X, int64_t segments, int64_t C, int group,
                        uint32_t *__restrict__ codes, float *__restrict__ scales) {
    constexpr float Q = (float)((1 << (BITS - 1)) - 1);
    constexpr uint32_t MASK = (1u << BITS) - 1u;
    const int lane = threadIdx.x & 31;
    const int64_t seg = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (seg >= segments) return;  // the whole warp leaves together
    const int64_t per_row = C / group;
    const int64_t row = seg / per_row;
    const int64_t e0 = row * C + (seg - row * per_row) * group;  // first element of the segment
    const uint4 *xs = X + e0 / 8;
    const int chunks = group / 8;

    float mx = 0.f;
    for (int c = lane; c < chunks; c += 32) {
        const uint4 v = __ldg(xs + c);
        const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(h[i] << 16)),
                                 fabsf(__uint_as_float(h[i] & 0xFFFF0000u))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    const float g = fmaxf(mx, 1e-5f);
    const float s = __fdiv_rn(Q, g);
    if (lane == 0) scales[seg] = __fdiv_rn(g, Q);

    for (int b = lane; b < group / 32; b += 32) {  // 32 values -> BITS words
        uint32_t h[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldg(xs + 4 * b + q);
            h[4 * q] = v.x;
            h[4 * q + 1] = v.y;
            h[4 * q + 2] = v.z;
            h[4 * q + 3] = v.w;
        }
        uint32_t out[BITS];
        uint64_t acc = 0;
        int nb = 0, w = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float x = __uint_as_float((i & 1) ? (h[i / 2] & 0xFFFF0000u) : (h[i / 2] << 16));
            // __fmul_rn is never contracted with the rounding add: the code is round(fl(x * s))
            float t = fminf(fmaxf(__fmul_rn(x, s), -Q - 1.f), Q);
            const uint32_t code = __float_as_uint(__fadd_rn(t, 12582912.f)) & MASK;  // 1.5 * 2^23
            acc |= (uint64_t)code << nb;
            nb += BITS;
            if (nb >= 32) {
                out[w++] = (uint32_t)acc;
                acc >>= 32;
                nb -= 32;
            }
        }
        uint32_t *dst = codes + (e0 + 32 * b) / 32 * BITS;
#pragma unroll
        for (int i = 0; i < BITS; ++i) dst[i] = out[i];
    }
}

cudaError_t launch_quant_states(const void *X, int64_t M, int64_t C, int64_t group, int bits,
                                void *codes, float *scales, cudaStream_t stream) {
    const int64_t segments = M * (C / group);
    const unsigned blocks = (unsigned)((segments + 7) / 8);
    auto x = reinterpret_cast<const uint4 *>(X);
    auto c = reinterpret_cast<uint32_t *>(codes);
    switch (bits) {
#define BITNET_STATES_CASE(B) \
    case B: quant_states_kernel<B><<<blocks, 256, 0, stream>>>(x, segments, C, (int)group, c, scales); break
        BITNET_STATES_CASE(2);
        BITNET_STATES_CASE(3);
        BITNET_STATES_CASE(4);
        BITNET_STATES_CASE(5);
        BITNET_STATES_CASE(6);
        BITNET_STATES_CASE(7);
        BITNET_STATES_CASE(8);
#undef BITNET_STATES_CASE
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace bitnet
