// weights.cu -- step 1 of the forward: absmean ternarisation of the latent weights and their
// 2-bit packing.
//
// absmean ("The Era of 1-bit LLMs" summary page, sections 方法论 and 方法详解; BitNet b1.58 2B4T
// article, section 一.2): one scale per tensor, gamma = mean |W|; every weight becomes
// RoundClip(w / gamma, -1, 1).  The pages print no formula; the readings used here are
// gamma = fp32(max(mean, 1e-5)) with the mean in double, an IEEE fp32 division and
// round-half-to-even.
//
// Two launches, both HBM-bound streams over W (2 bytes per weight):
//   absmean_partials_kernel  fixed grid of P blocks (P depends only on the weight count), each
//                            sums |w| in fp64 over a fixed grid-stride subset and writes one
//                            partial; the reduction tree is fixed, so gamma is deterministic.
//   ternarize_pack_kernel    every block first sums the P partials (<= 9.5 KB, L2-resident) in a
//                            fixed tree, so no third launch or atomic is needed; then each thread
//                            turns 16 weights into one packed 32-bit word with integer compares
//                            against a bf16 threshold equivalent to the fp32 division.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace bitnet {

constexpr int kWeightThreads = 256;
constexpr int kMaxPartials = 1184;  // 8 blocks per SM on 148 SMs

int absmean_num_partials(int64_t n) {
    int64_t vec = n / 8;  // 16-byte vectors of 8 bf16
    int64_t p = (vec + kWeightThreads * 4 - 1) / (kWeightThreads * 4);
    if (p < 1) p = 1;
    if (p > kMaxPartials) p = kMaxPartials;
    return (int)p;
}

__device__ __forceinline__ double abs_bf16_pair_sum(uint32_t w) {
    // |bf16| is the bit pattern with the sign cleared; widening to fp32 is exact.
    float lo = __uint_as_float((w & 0x7FFFu) << 16);
    float hi = __uint_as_float(w & 0x7FFF0000u);
    return (double)lo + (double)hi;
}

__global__ void __launch_bounds__(kWeightThreads)
    absmean_partials_kernel(const uint4 *__restrict__ w, int64_t nvec,
                            double *__restrict__ partials) {
    double acc0 = 0.0, acc1 = 0.0;
    const int64_t stride = (int64_t)gridDim.x * kWeightThreads;
    int64_t i = (int64_t)blockIdx.x * kWeightThreads + threadIdx.x;
    // four independent 16-byte loads in flight per thread, then their sums
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = ldg_nc_v4(w + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc0 += abs_bf16_pair_sum(v[u].x);
            acc1 += abs_bf16_pair_sum(v[u].y);
            acc0 += abs_bf16_pair_sum(v[u].z);
            acc1 += abs_bf16_pair_sum(v[u].w);
        }
    }
    for (; i < nvec; i += stride) {
        uint4 v = ldg_nc_v4(w + i);
        acc0 += abs_bf16_pair_sum(v.x);
        acc1 += abs_bf16_pair_sum(v.y);
        acc0 += abs_bf16_pair_sum(v.z);
        acc1 += abs_bf16_pair_sum(v.w);
    }
    double s = acc0 + acc1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    __shared__ double warp_sums[kWeightThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int k = 0; k < kWeightThreads / 32; ++k) t += warp_sums[k];
        partials[blockIdx.x] = t;
    }
}

// Threshold for the ternary decision, as a 15-bit bf16 magnitude pattern.
// RoundClip(w / gamma, -1, 1) != 0  <=>  fl32(|w| / gamma) > 0.5 (ties to even send 0.5 to 0)
// <=>  |w| / gamma > 0.5 + 2^-25 (the midpoint between 0.5 and the next float rounds down to
// 0.5)  <=>  |w| > T with T = gamma * (0.5 + 2^-25), a product that is exact in double.  bf16
// magnitudes are ordered like their bit patterns, so the decision is |w|_bits >= the pattern of
// the smallest bf16 strictly above T.  This gives exactly the codes of the fp32 division.
__device__ __forceinline__ uint32_t ternary_threshold_bits(float gamma) {
    const double T = (double)gamma * (0.5 + 0x1p-25);
    const uint32_t f = __float_as_uint(__double2float_ru(T));  // smallest float >= T
    uint32_t h = (f + 0xFFFFu) >> 16;                          // smallest bf16 >= T
    if ((double)__uint_as_float(h << 16) == T) h += 1;         // strictly above T
    return h;
}

// gamma from the P partial sums; every block computes it the same way (a fixed assignment of
// partials to threads and a fixed reduction tree), so gamma does not depend on the launch.
// Block 0 writes gamma.  Contains __syncthreads.
__device__ __forceinline__ float block_gamma(const double *__restrict__ partials, int P,
                                             double n_weights, float *__restrict__ gamma_out) {
    __shared__ double warp_sums[kWeightThreads / 32];
    __shared__ float s_gamma;
    double s = 0.0;
    for (int j = threadIdx.x; j < P; j += kWeightThreads) s += partials[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int k = 0; k < kWeightThreads / 32; ++k) t += warp_sums[k];
        const float g = (float)fmax(t / n_weights, 1e-5);
        s_gamma = g;
        if (blockIdx.x == 0) *gamma_out = g;
    }
    __syncthreads();
    return s_gamma;
}

// gamma (block_gamma) and its decision threshold for bf16 weights.
__device__ __forceinline__ uint32_t block_threshold(const double *__restrict__ partials, int P,
                                                    double n_weights, float *__restrict__ gamma_out) {
    return ternary_threshold_bits(block_gamma(partials, P, n_weights, gamma_out));
}

// Offset code u = q + 1 of one bf16 weight against the threshold (see ternary_threshold_bits).
__device__ __forceinline__ uint32_t offset_code(uint32_t bits, uint32_t thr) {
    return (bits & 0x7FFFu) >= thr ? ((bits & 0x8000u) ? 0u : 2u) : 1u;
}

__global__ void __launch_bounds__(kWeightThreads)
    ternarize_pack_kernel(const uint4 *__restrict__ w, int64_t nwords, double n_weights,
                          const double *__restrict__ partials, int P, uint32_t *__restrict__ wp,
                          float *__restrict__ gamma_out) {
    // the first 16 weights of this thread do not depend on gamma: their loads are issued before
    // the reduction below, so the two memory latencies overlap
    int64_t i = (int64_t)blockIdx.x * kWeightThreads + threadIdx.x;
    uint4 a = make_uint4(0, 0, 0, 0), b = a;
    if (i < nwords) {
        a = ldg_nc_v4(w + 2 * i);
        b = ldg_nc_v4(w + 2 * i + 1);
    }
    const uint32_t thr = block_threshold(partials, P, n_weights, gamma_out);
    const int64_t stride = (int64_t)gridDim.x * kWeightThreads;
    for (bool first = true; i < nwords; i += stride, first = false) {
        // 16 consecutive weights k = 16i + e; weight e = 4p + j goes to bits 8j + 2p as u = q + 1.
        if (!first) {
            a = ldg_nc_v4(w + 2 * i);
            b = ldg_nc_v4(w + 2 * i + 1);
        }
        const uint32_t h[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const uint32_t bits = (e & 1) ? (h[e >> 1] >> 16) : (h[e >> 1] & 0xFFFFu);
            const uint32_t u = offset_code(bits, thr);
            word |= u << (8 * (e & 3) + 2 * (e >> 2));
        }
        wp[i] = word;
    }
}

// Base-3 storage for the decode product (2B4T article, section 一.1: five ternary weights in one
// byte): row n is ceil(K/20) 32-bit words; byte i of word w holds the offset codes of weights
// k = 20w + 5i .. +4 as the base-3 number u0*81 + u1*27 + u2*9 + u3*3 + u4 (first weight most
// significant); weights k >= K are stored as u = 1.  The decisions are those of
// ternarize_pack_kernel (same gamma, same threshold).  One thread per word.
__global__ void __launch_bounds__(kWeightThreads)
    ternarize_pack_base3_kernel(const uint16_t *__restrict__ w, int64_t N, int64_t K,
                                double n_weights, const double *__restrict__ partials, int P,
                                uint32_t *__restrict__ wp3, float *__restrict__ gamma_out) {
    const int64_t words = (K + 19) / 20;
    const int64_t total = N * words;
    const uint32_t thr = block_threshold(partials, P, n_weights, gamma_out);
    const int64_t stride = (int64_t)gridDim.x * kWeightThreads;
    for (int64_t i = (int64_t)blockIdx.x * kWeightThreads + threadIdx.x; i < total; i += stride) {
        const int64_t n = i / words, wd = i - n * words;
        const int64_t k0 = 20 * wd;
        const uint16_t *src = w + n * K + k0;
        uint32_t h[20];
        if (k0 + 20 <= K) {
            // 40 bytes at an 8-byte-aligned address (K % 128 == 0)
#pragma unroll
            for (int j = 0; j < 5; ++j) {
                const uint2 v = __ldg(reinterpret_cast<const uint2 *>(src) + j);
                h[4 * j] = v.x & 0xFFFFu;
                h[4 * j + 1] = v.x >> 16;
                h[4 * j + 2] = v.y & 0xFFFFu;
                h[4 * j + 3] = v.y >> 16;
            }
        } else {
#pragma unroll
            for (int e = 0; e < 20; ++e) h[e] = k0 + e < K ? (uint32_t)__ldg(src + e) : 0u;
        }
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            uint32_t v = 0;
#pragma unroll
            for (int t = 0; t < 5; ++t) {
                const int e = 5 * b + t;
                const uint32_t u = k0 + e < K ? offset_code(h[e], thr) : 1u;
                v = v * 3u + u;
            }
            word |= v << (8 * b);
        }
        wp3[i] = word;
    }
}

cudaError_t launch_ternarize_pack_base3(const void *W, int64_t N, int64_t K,
                                        const double *partials, int P, uint32_t *Wp3,
                                        float *gamma, cudaStream_t stream) {
    const int64_t total = N * ((K + 19) / 20);
    int64_t blocks = (total + kWeightThreads - 1) / kWeightThreads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    ternarize_pack_base3_kernel<<<(unsigned)blocks, kWeightThreads, 0, stream>>>(
        reinterpret_cast<const uint16_t *>(W), N, K, (double)N * (double)K, partials, P, Wp3,
        gamma);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// fp32 weights: the rows W' = W H / sqrt(K) of the weight + activation rotation (BitNet v2
// write-up: Hadamard rotation of the weights and the activations, or of the activations only).
// The same absmean ternarisation on fp32 values: partial sums of |w'| in fp64 (a fixed grid of P
// blocks, as for bf16), then q = RoundClip(w' / gamma, -1, 1) with one IEEE fp32 division.

__global__ void __launch_bounds__(kWeightThreads)
    absmean_partials_f32_kernel(const float4 *__restrict__ w, int64_t nvec,
                                double *__restrict__ partials) {
    double acc0 = 0.0, acc1 = 0.0;
    const int64_t stride = (int64_t)gridDim.x * kWeightThreads;
    int64_t i = (int64_t)blockIdx.x * kWeightThreads + threadIdx.x;
    for (; i + 3 * stride < nvec; i += 4 * stride) {  // four 16-byte loads in flight
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(w + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            acc0 += fabs((double)v[u].x) + fabs((double)v[u].y);
            acc1 += fabs((double)v[u].z) + fabs((double)v[u].w);
        }
    }
    for (; i < nvec; i += stride) {
        const float4 v = __ldg(w + i);
        acc0 += fabs((double)v.x) + fabs((double)v.y);
        acc1 += fabs((double)v.z) + fabs((double)v.w);
    }
    double s = acc0 + acc1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    __shared__ double warp_sums[kWeightThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_sums[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int k = 0; k < kWeightThreads / 32; ++k) t += warp_sums[k];
        partials[blockIdx.x] = t;
    }
}

__global__ void __launch_bounds__(kWeightThreads)
    ternarize_pack_f32_kernel(const float4 *__restrict__ w, int64_t nwords, double n_weights,
                              const double *__restrict__ partials, int P,
                              uint32_t *__restrict__ wp, float *__restrict__ gamma_out) {
    const float g = block_gamma(partials, P, n_weights, gamma_out);
    const int64_t stride = (int64_t)gridDim.x * kWeightThreads;
    for (int64_t i = (int64_t)blockIdx.x * kWeightThreads + threadIdx.x; i < nwords; i += stride) {
        float4 v[4];  // weights 16i .. 16i+15
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = __ldg(w + 4 * i + c);
        const float f[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                             v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            // rint(r) with ties to even is 0 for |r| <= 0.5 and +-1 (after the clip) above
            const float r = __fdiv_rn(f[e], g);
            const uint32_t u = fabsf(r) > 0.5f ? (r > 0.f ? 2u : 0u) : 1u;
            word |= u << (8 * (e & 3) + 2 * (e >> 2));
        }
        wp[i] = word;
    }
}

cudaError_t launch_ternarize_pack_f32(const float *W, int64_t n, double *partials, int P,
                                      uint32_t *Wp, float *gamma, cudaStream_t stream) {
    absmean_partials_f32_kernel<<<P, kWeightThreads, 0, stream>>>(
        reinterpret_cast<const float4 *>(W), n / 4, partials);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t nwords = n / 16;
    int64_t blocks = (nwords + kWeightThreads - 1) / kWeightThreads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    ternarize_pack_f32_kernel<<<(unsigned)blocks, kWeightThreads, 0, stream>>>(
        reinterpret_cast<const float4 *>(W), nwords, (double)n, partials, P, Wp, gamma);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Fixed device scratch for callers that cannot allocate device memory.
//
// The partial sums of |w| live in this file-scope array instead of caller workspace.  Every GPU
// that loads the library holds it (9472 bytes) until the process exits.  Host code must not pass
// the symbol itself to a kernel: the host-side name is only a stand-in, so its device address is
// looked up once per device with cudaGetSymbolAddress while that device is current.
// ------------------------------------------------------------------------------------------
static __device__ __align__(256) double g_noalloc_partials[kMaxPartials];

cudaError_t noalloc_partials_address(double **ptr, size_t *bytes) {
    static std::mutex mu;
    static double *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_partials);
        if (e != cudaSuccess) return e;
        addr[dev] = static_cast<double *>(p);
    }
    *ptr = addr[dev];
    *bytes = sizeof(g_noalloc_partials);
    return cudaSuccess;
}

cudaError_t launch_absmean_partials(const void *W, int64_t n, double *partials, int P,
                                    cudaStream_t stream) {
    absmean_partials_kernel<<<P, kWeightThreads, 0, stream>>>(
        reinterpret_cast<const uint4 *>(W), n / 8, partials);
    return cudaGetLastError();
}

cudaError_t launch_ternarize_pack(const void *W, int64_t n, const double *partials, int P,
                                  uint32_t *Wp, float *gamma, cudaStream_t stream) {
    int64_t nwords = n / 16;
    int64_t blocks = (nwords + kWeightThreads - 1) / kWeightThreads;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    ternarize_pack_kernel<<<(unsigned)blocks, kWeightThreads, 0, stream>>>(
        reinterpret_cast<const uint4 *>(W), nwords, (double)n, partials, P, Wp, gamma);
    return cudaGetLastError();
}

}  // namespace bitnet
