// hadamard_tc.cu -- steps 2 and 3 for K = 8192 and 16384 (the FFN down projections): the online
// Hadamard transform of each token row with its first seven butterfly levels on the tensor
// cores, fused with the per-token quantisation.
//
// BitNet v2 write-up, H-BitLinear paragraphs: z = H_K x / sqrt(K) (H_K Sylvester, entries +-1)
// before the activations of Wo and Wdown are quantised.  Write K = 128 n and a token row as the
// matrix X[a][b] = x[a n + b] (a: the top seven index bits, b: the low log2 n bits).  The
// Sylvester matrix factors as H_K = H_128 (x) H_n, so
//     z = (H_128 . X . H_n) / sqrt(K):
// the left factor is one tensor-core product per token, D[a', b] = sum_a H_128[a', a] X[a, b]
// (tcgen05.mma kind::f16: A = H_128 in bf16, exact +-1, built once per CTA in shared memory;
// B = X, bf16 as stored, in its natural row-major layout, i.e. the MN-major operand; fp32
// accumulation in tensor memory, one row a' per lane), and the right factor is log2 n butterfly
// levels over the n values that each lane holds, in registers, with no shuffles or shared-memory
// transposes.  Each product term is exact (bf16 times +-1); only the fp32 sums round, as the
// butterflies' additions do.
//
// The quantisation that follows is the one of fwht_quant_kernel: per token, absmax (INT8 and the
// absmax INT4 variant) or absmean (INT4) over the 128 lanes' values, the code decided as
// round_half_even(fl32(z * s)).  The same kernel writes z itself for the transform's parity entry,
// so the codes can be checked against the exact rows they were decided on.
//
// Persistent grid, one CTA per SM; a CTA takes tokens blockIdx.x, + gridDim.x, ...:
//   warp 0       TMA: the token's bf16 row as [128 rows x 64 values] boxes (128-byte swizzle) into
//                a ring of X slots;
//   warp 1       tensor-memory allocation; one thread issues the 8 MMAs (K = 16 each) of a token
//                into a tensor-memory slot of n columns;
//   warps 2 ..   two (K = 16384) or three (K = 8192) epilogue groups of four warps (one per lane
//                quadrant) taking tokens in turn: tcgen05.ld of the slot (thread = row a'), butterflies, scale, reduction
//                over the group (named barrier), codes, scale and code sum.
// Every mbarrier wait is bounded (~1 s, then BITNET_ERR_TIMEOUT and the kernel winds down without
// further waits); no TMA multicast is used.
#include "common.cuh"
#include "kernels.h"

#include <cudaTypedefs.h>

namespace bitnet {
namespace htc {

constexpr int ROWS = 128;                 // a: MMA M and K, tensor-memory lanes
constexpr int UMMA_K = 16;                // K per kind::f16 MMA
constexpr int MMAS = ROWS / UMMA_K;       // 8 per token
constexpr int BOX_N = 64;                 // b values per TMA box (128 B of bf16, one swizzle row)
constexpr int BOX_BYTES = ROWS * BOX_N * 2;  // 16 KB
constexpr int H_BYTES = ROWS * ROWS * 2;     // 32 KB: two K-major [128 x 64] sub-tiles
constexpr int TMEM_COLS = 512;

template <int LOGN>
struct Cfg {
    static constexpr int N = 1 << LOGN;                  // values per lane
    static constexpr int K = ROWS * N;
    // epilogue groups of four warps (tokens in flight per SM), as many as the registers allow
    static constexpr int GROUPS = LOGN == 7 ? 2 : 3;
    static constexpr int T_SLOTS = 2 * GROUPS;           // tensor-memory slots, two per group
    static constexpr int THREADS = (2 + 4 * GROUPS) * 32;
    static constexpr int X_BYTES = ROWS * N * 2;         // one token, bf16
    static constexpr int X_SLOTS = LOGN == 7 ? 4 : 6;
    static constexpr int OFF_H = 0;
    static constexpr int OFF_X = H_BYTES;
    static constexpr int OFF_RED = OFF_X + X_SLOTS * X_BYTES;   // per group: 4 doubles, 4 ints
    static constexpr int OFF_BAR = OFF_RED + GROUPS * 64;
    // + barriers, alignment slack, and a guard: every operand read of an MMA stays inside the
    // allocation whichever of its descriptor's two strides is taken along K
    static constexpr size_t SMEM = (size_t)OFF_BAR + 256 + 1024 + 2048;
    // stride between the two 64-value blocks of a token's X slot (one block when N = 64: then the
    // 8-row stride, so that the field never points past the slot)
    static constexpr uint32_t LBO = N == 128 ? BOX_BYTES : 1024;
    static_assert(N == 64 || N == 128, "one or two 64-value boxes per token");
    static_assert(T_SLOTS * N <= TMEM_COLS && T_SLOTS <= 8, "tensor-memory budget");
    static_assert(SMEM <= 227 * 1024, "shared-memory budget");
};

struct __align__(8) Bars {
    uint64_t x_full[8];
    uint64_t x_empty[8];
    uint64_t t_full[8];
    uint64_t t_empty[8];
    uint32_t tmem_base;
};

// sqrt(7) rounded to fp32 (the absmean INT4 code of the mean magnitude)
constexpr float kSqrt7 = 2.6457513110645906f;

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzled layout: 64-value (128 B)
// rows along MN, 8-row groups along K 1024 B apart (stride byte offset), consecutive 64-value MN
// blocks `lbo` bytes apart (leading byte offset).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t addr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// kind::f16 instruction descriptor: D f32, A and B bf16, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_kmaj_mnmaj(int M, int N) {
    return (1u << 4)                         // D format: f32
           | (1u << 7)                       // A format: bf16
           | (1u << 10)                      // B format: bf16
           | (1u << 16)                      // B is MN-major
           | ((uint32_t)(N >> 3) << 17)
           | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Barrier over the four warps of an epilogue group (named barrier 1 + group).
__device__ __forceinline__ void group_sync(int group) {
    asm volatile("bar.sync %0, 128;" ::"r"(1 + group) : "memory");
}

__device__ __forceinline__ float2 bfly_sub(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.f, -1.f), a);  // a - b, one rounding
}

// BITS 8 or 4; ABSMEAN: the INT4 absmean rule (else absmax with Q = 127 or 7); ZOUT: write z (fp32)
// instead of codes.
template <int LOGN, int BITS, bool ABSMEAN, bool ZOUT>
__global__ void __launch_bounds__(Cfg<LOGN>::THREADS, 1)
    hadamard_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, int M, float rsqrt_k,
                       uint8_t *__restrict__ codes, float *__restrict__ scales,
                       int32_t *__restrict__ rowsum, float *__restrict__ zout, int *status) {
    using C = Cfg<LOGN>;
    constexpr int N = C::N, GROUPS = C::GROUPS, T_SLOTS = C::T_SLOTS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sh = smem + C::OFF_H;
    uint8_t *sx = smem + C::OFF_X;
    Bars *bar = reinterpret_cast<Bars *>(smem + C::OFF_BAR);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int my_tokens = (int)blockIdx.x < M ? (M - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    // H_128 as the K-major A operand: values a = 64 j + 8 c .. +7 of row a' form 16-byte chunk c
    // of that row in sub-tile j, stored at chunk c ^ (a' % 8) (128-byte swizzle);
    // H[a', a] = (-1)^popcount(a' & a)
    for (int e = threadIdx.x; e < ROWS * ROWS / 8; e += C::THREADS) {
        const int j = e >> 10, ap = (e >> 3) & 127, c = e & 7;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int a = 64 * j + 8 * c + 2 * i;
            const uint32_t lo = (__popc(ap & a) & 1) ? 0xBF80u : 0x3F80u;  // bf16 -1 / +1
            const uint32_t hi = (__popc(ap & (a + 1)) & 1) ? 0xBF80u : 0x3F80u;
            w[i] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4 *>(sh + j * (ROWS * 128) + ap * 128 + ((c ^ (ap & 7)) << 4)) =
            make_uint4(w[0], w[1], w[2], w[3]);
    }
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::X_SLOTS; ++s) {
            mbar_init(&bar->x_full[s], 1);
            mbar_init(&bar->x_empty[s], 1);
        }
        for (int s = 0; s < T_SLOTS; ++s) {
            mbar_init(&bar->t_full[s], 1);
            mbar_init(&bar->t_empty[s], 4);
        }
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
    if (warp == 1) {
        tmem_alloc(&bar->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    // the product that reads these codes may start its own set-up now (it waits for this grid
    // to complete before it reads anything)
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            pdl_wait();
            uint32_t issued = 0, ph = 0;
            for (int i = 0; i < my_tokens; ++i) {
                const int s = i % C::X_SLOTS;
                const uint32_t p = (uint32_t)(i / C::X_SLOTS) & 1;
                if (!mbar_wait(&bar->x_empty[s], p ^ 1, status)) break;
                const int t = (int)blockIdx.x + i * (int)gridDim.x;
                mbar_arrive_expect_tx(&bar->x_full[s], C::X_BYTES);
#pragma unroll
                for (int j = 0; j < N / BOX_N; ++j)
                    tma_load_2d(sx + (size_t)s * C::X_BYTES + j * BOX_BYTES, &tmap_x, j * BOX_N,
                                t * ROWS, &bar->x_full[s]);
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
            }
            for (int s = 0; s < C::X_SLOTS; ++s)
                if (issued & (1u << s)) mbar_wait(&bar->x_full[s], (ph >> s) & 1, status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_kmaj_mnmaj(ROWS, N);
            const uint32_t h_addr = smem_addr(sh);
            const uint32_t x_addr = smem_addr(sx);
            for (int i = 0; i < my_tokens; ++i) {
                const int s = i % C::X_SLOTS, ts = i % T_SLOTS;
                if (!mbar_wait(&bar->x_full[s], (uint32_t)(i / C::X_SLOTS) & 1, status)) break;
                if (!mbar_wait(&bar->t_empty[ts], ((uint32_t)(i / T_SLOTS) & 1) ^ 1, status)) break;
                tc_fence_after();
                const uint32_t xs = x_addr + (uint32_t)(s * C::X_BYTES);
#pragma unroll
                for (int kk = 0; kk < MMAS; ++kk) {
                    // A: rows a' of H, K = a in [16 kk, 16 kk + 16): sub-tile kk / 4, 32 B steps
                    const uint64_t adesc =
                        smem_desc_kmajor_sw128(h_addr + (kk >> 2) * (ROWS * 128)) +
                        (uint64_t)((kk & 3) * 2);
                    // B: rows a = 16 kk .. +15 of X (two 8-row groups, 2 KB), all n values
                    const uint64_t bdesc = smem_desc_mn_sw128(xs + kk * 2048, C::LBO);
                    mma_bf16_ss(tmem + (uint32_t)(ts * N), adesc, bdesc, IDESC, kk != 0 ? 1u : 0u);
                }
                mma_commit(&bar->x_empty[s]);
                mma_commit(&bar->t_full[ts]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue groups
        const int grp = (warp - 2) >> 2;
        const int quad = warp & 3;                 // tensor-memory lanes 32 quad .. 32 quad + 31
        const int gw = (warp - 2) & 3;             // warp index within the group (reduction slot)
        const int ap = quad * 32 + lane;           // row a' of the transform
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        double *red_d = reinterpret_cast<double *>(smem + C::OFF_RED + grp * 64);
        float *red_f = reinterpret_cast<float *>(red_d);
        int *red_i = reinterpret_cast<int *>(smem + C::OFF_RED + grp * 64 + 32);
        bool ok = true;
        for (int i = grp; i < my_tokens; i += GROUPS) {
            const int ts = i % T_SLOTS;
            const int64_t t = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
            if (ok) {
                bool w_ok = true;
                if (lane == 0) w_ok = mbar_wait(&bar->t_full[ts], (uint32_t)(i / T_SLOTS) & 1, status);
                ok = __shfl_sync(0xFFFFFFFFu, w_ok ? 1 : 0, 0) != 0;
                __syncwarp();
            }
            tc_fence_after();
            // D[a', b] for this lane's row: N fp32 columns (all loads issued, then one wait)
            uint32_t r[N / 32][32];
#pragma unroll
            for (int q = 0; q < N / 32; ++q)
                tmem_ld_32x32b_x32(t_lane + (uint32_t)(ts * N + 32 * q), r[q]);
            tmem_wait_ld();
            float2 v[N / 2];
#pragma unroll
            for (int q = 0; q < N / 32; ++q)
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    v[16 * q + c] = make_float2(__uint_as_float(r[q][2 * c]),
                                                __uint_as_float(r[q][2 * c + 1]));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->t_empty[ts]);  // the slot may take the next token
            // ---- the right factor H_n over b: bit 0 inside each pair, bits 1 .. LOGN-1 ----
#pragma unroll
            for (int c = 0; c < N / 2; ++c) {
                const float x = v[c].x, y = v[c].y;
                v[c] = make_float2(x + y, x - y);
            }
#pragma unroll
            for (int m = 1; m < N / 2; m <<= 1) {
#pragma unroll
                for (int c = 0; c < N / 2; ++c) {
                    if (c & m) continue;
                    const float2 x = v[c], y = v[c | m];
                    v[c] = add2_rn(x, y);
                    v[c | m] = bfly_sub(x, y);
                }
            }
            // z = y / sqrt(K).  For even log2 K (K = 16384) 1 / sqrt(K) = 2^-7 exactly, so the
            // scaling commutes with every rounding below: it is folded into the token's scale (the
            // codes are the same bits) and applied to the row only when z itself is written.
            constexpr bool EXACT_SCALE = LOGN == 7;
            if (!EXACT_SCALE || ZOUT) {
                const float2 rk2 = make_float2(rsqrt_k, rsqrt_k);
#pragma unroll
                for (int c = 0; c < N / 2; ++c) v[c] = mul2_rn(v[c], rk2);
            }

            if constexpr (ZOUT) {
                float *zr = zout + t * C::K + (int64_t)ap * N;
#pragma unroll
                for (int c = 0; c < N / 4; ++c)
                    *reinterpret_cast<float4 *>(zr + 4 * c) =
                        make_float4(v[2 * c].x, v[2 * c].y, v[2 * c + 1].x, v[2 * c + 1].y);
                continue;
            } else {
                // ---- the token's scale: max |z| or mean |z| over the 128 rows of the group ----
                float g;
                if constexpr (ABSMEAN) {
                    // the sum of |z| to double accuracy (the oracle sums in double), two ways:
                    double sa = 0.0;
                    if constexpr (LOGN == 6) {
                        // Neumaier's compensation in fp32: t = s + a rounds, and its error
                        // (max(s, a) - t) + min(s, a) is exact (all terms are >= 0), so s + c
                        // carries the sum to about 2^-45 relative, without the f32 -> f64
                        // conversion per element, whose unit is the limit of this shape on B200.
                        // Four independent (s, c) pairs.
                        float s4[4] = {0.f, 0.f, 0.f, 0.f}, c4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int c = 0; c < N / 2; ++c) {
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int k = (2 * c + e) & 3;
                                const float x = fabsf(e == 0 ? v[c].x : v[c].y);
                                const float t = __fadd_rn(s4[k], x);
                                c4[k] = __fadd_rn(c4[k], __fadd_rn(__fsub_rn(fmaxf(s4[k], x), t),
                                                                   fminf(s4[k], x)));
                                s4[k] = t;
                            }
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) sa += (double)s4[k] + (double)c4[k];
                    } else {
                        // in double directly (two issued instructions per element; with 128
                        // values per thread the instruction issue, not the conversion unit, is
                        // the limit), eight independent sums
                        double p8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
                        for (int c = 0; c < N / 2; ++c)
                            p8[c & 7] += fabs((double)v[c].x) + fabs((double)v[c].y);
                        sa = ((p8[0] + p8[1]) + (p8[2] + p8[3])) + ((p8[4] + p8[5]) + (p8[6] + p8[7]));
                        if constexpr (EXACT_SCALE) sa *= (double)rsqrt_k;  // exact: 2^-7
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) sa += __shfl_xor_sync(0xFFFFFFFFu, sa, o);
                    if (lane == 0) red_d[gw] = sa;
                    group_sync(grp);
                    sa = (red_d[0] + red_d[1]) + (red_d[2] + red_d[3]);
                    g = (float)fmax(sa / (double)C::K, 1e-5);
                } else {
                    float m8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int c = 0; c < N / 2; ++c)
                        m8[c & 7] = fmaxf(m8[c & 7], fmaxf(fabsf(v[c].x), fabsf(v[c].y)));
                    float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                     fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
                    if (lane == 0) red_f[gw] = mx;
                    group_sync(grp);
                    mx = fmaxf(fmaxf(red_f[0], red_f[1]), fmaxf(red_f[2], red_f[3]));
                    if constexpr (EXACT_SCALE) mx *= rsqrt_k;  // exact: 2^-7
                    g = fmaxf(mx, 1e-5f);
                }
                constexpr float Q = ABSMEAN ? kSqrt7 : BITS == 4 ? 7.f : 127.f;
                const float s = __fdiv_rn(Q, g);
                const float dq = __fdiv_rn(g, Q);
                // the multiplier of the unscaled rows: fl(z * s) = fl(y * (s * 2^-7)) exactly
                const float s_y = EXACT_SCALE ? s * rsqrt_k : s;
                const float2 magic2 = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23
                int sums[4] = {0, 0, 0, 0};  // code sums, four independent chains
#pragma unroll
                for (int g16 = 0; g16 < N / 16; ++g16) {
                    int &sum = sums[g16 & 3];
                    // 16 consecutive values -> round(z * s): the low byte of t + 1.5 * 2^23
                    uint32_t f[16];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        // __fmul_rn is never contracted with the rounding add: the code is
                        // round(fl(z * s)), the two roundings the reference takes
                        float2 tt = make_float2(__fmul_rn(v[g16 * 8 + e].x, s_y),
                                                __fmul_rn(v[g16 * 8 + e].y, s_y));
                        if constexpr (ABSMEAN)  // clip before rounding: the same as after it
                            tt = make_float2(fminf(fmaxf(tt.x, -8.f), 7.f), fminf(fmaxf(tt.y, -8.f), 7.f));
                        const float2 u = __fadd2_rn(tt, magic2);
                        f[2 * e] = __float_as_uint(u.x);
                        f[2 * e + 1] = __float_as_uint(u.y);
                    }
                    const int64_t k0 = (int64_t)ap * N + 16 * g16;  // first element in the row
                    if constexpr (BITS == 8) {
                        uint4 w;
                        w.x = gather_low_bytes(f[0], f[1], f[2], f[3]);
                        w.y = gather_low_bytes(f[4], f[5], f[6], f[7]);
                        w.z = gather_low_bytes(f[8], f[9], f[10], f[11]);
                        w.w = gather_low_bytes(f[12], f[13], f[14], f[15]);
                        sum = __dp4a((int)w.x, 0x01010101, sum);
                        sum = __dp4a((int)w.y, 0x01010101, sum);
                        sum = __dp4a((int)w.z, 0x01010101, sum);
                        sum = __dp4a((int)w.w, 0x01010101, sum);
                        *reinterpret_cast<uint4 *>(codes + t * C::K + k0) = w;
                    } else {
                        // every 8 codes k0 .. k0+7 fill 4 bytes: byte j = code k0+j (low nibble)
                        // and k0+4+j (high nibble)
                        const uint32_t A0 = gather_low_bytes(f[0], f[1], f[2], f[3]);
                        const uint32_t B0 = gather_low_bytes(f[4], f[5], f[6], f[7]);
                        const uint32_t A1 = gather_low_bytes(f[8], f[9], f[10], f[11]);
                        const uint32_t B1 = gather_low_bytes(f[12], f[13], f[14], f[15]);
                        sum = __dp4a((int)A0, 0x01010101, sum);
                        sum = __dp4a((int)B0, 0x01010101, sum);
                        sum = __dp4a((int)A1, 0x01010101, sum);
                        sum = __dp4a((int)B1, 0x01010101, sum);
                        *reinterpret_cast<uint2 *>(codes + t * (C::K / 2) + k0 / 2) =
                            make_uint2((A0 & 0x0F0F0F0Fu) | ((B0 << 4) & 0xF0F0F0F0u),
                                       (A1 & 0x0F0F0F0Fu) | ((B1 << 4) & 0xF0F0F0F0u));
                    }
                }
                int sum = (sums[0] + sums[1]) + (sums[2] + sums[3]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
                if (lane == 0) red_i[gw] = sum;
                group_sync(grp);
                if (gw == 0 && lane == 0) {
                    scales[t] = dq;
                    rowsum[t] = red_i[0] + red_i[1] + red_i[2] + red_i[3];
                }
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int LOGN, int BITS, bool ABSMEAN, bool ZOUT>
static cudaError_t launch_t(const CUtensorMap &map, int64_t M, void *codes, float *scales,
                           int32_t *rowsum, float *zout, int *status, int num_sms,
                           cudaStream_t stream) {
    auto kern = hadamard_tc_kernel<LOGN, BITS, ABSMEAN, ZOUT>;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)Cfg<LOGN>::SMEM);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const int64_t blocks = M < num_sms ? M : num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, 1, 1);
    cfg.blockDim = dim3(Cfg<LOGN>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg<LOGN>::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const float rk = (float)(1.0 / sqrt((double)Cfg<LOGN>::K));
    return cudaLaunchKernelEx(&cfg, kern, map, (int)M, rk, reinterpret_cast<uint8_t *>(codes),
                              scales, rowsum, zout, status);
}

template <int LOGN>
static cudaError_t launch_n(const CUtensorMap &map, int64_t M, int act_bits, void *codes,
                            float *scales, int32_t *rowsum, float *zout, int *status, int num_sms,
                            cudaStream_t stream) {
    if (zout) return launch_t<LOGN, 8, false, true>(map, M, codes, scales, rowsum, zout, status, num_sms, stream);
    if (act_bits == 8) return launch_t<LOGN, 8, false, false>(map, M, codes, scales, rowsum, zout, status, num_sms, stream);
    if (act_bits == 4) return launch_t<LOGN, 4, true, false>(map, M, codes, scales, rowsum, zout, status, num_sms, stream);
    if (act_bits == kActInt4Absmax) return launch_t<LOGN, 4, false, false>(map, M, codes, scales, rowsum, zout, status, num_sms, stream);
    return cudaErrorInvalidValue;
}

}  // namespace htc

bool hadamard_tc_supported(int logk) { return logk == 13 || logk == 14; }

cudaError_t launch_hadamard_tc(const void *X, int64_t M, int logk, int act_bits, void *codes,
                               float *scales, int32_t *rowsum, float *zout, int *status,
                               void *encode_fn, int num_sms, cudaStream_t stream) {
    using namespace htc;
    if (!hadamard_tc_supported(logk) || M < 1 || M > (int64_t)INT32_MAX / ROWS)
        return cudaErrorInvalidValue;
    const int n = 1 << (logk - 7);
    // the rows as [M * 128, n] bf16: row t * 128 + a holds x[a n .. a n + n - 1] of token t
    CUtensorMap map;
    if (encode_tmap_2d(encode_fn, &map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)n,
                       (uint64_t)M * ROWS, (uint64_t)n * 2, BOX_N, ROWS,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    return logk == 14 ? launch_n<7>(map, M, act_bits, codes, scales, rowsum, zout, status, num_sms, stream)
                      : launch_n<6>(map, M, act_bits, codes, scales, rowsum, zout, status, num_sms, stream);
}

}  // namespace bitnet
