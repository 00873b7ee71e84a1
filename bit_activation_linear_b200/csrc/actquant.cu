// actquant.cu -- steps 2 and 3 of the forward: the online Hadamard transform of every token
// row (H-BitLinear) fused with per-token quantisation, absmax to INT8 or absmean to INT4.
//
// BitNet v2 write-up, paragraphs on H-BitLinear: before the activations of Wo and Wdown are
// quantised, each token row is multiplied by a Hadamard matrix (entries +-1, mutually
// orthogonal rows), which turns the sharp, outlier-heavy distribution into a near-Gaussian
// one.  BitNet b1.58 2B4T article, section 一.2: activations are quantised per token with
// absmax to 8 bits; the BitNet v2 write-up adds native 4-bit activations, each width with its
// own strategy: INT4 takes the absmean form (mean |z| -> code sqrt(7), clip [-8, 7]).  Readings:
// H_K in Sylvester order scaled by 1/sqrt(K); eps 1e-5; round half to even.
//
// Kernel design (HBM-bound: 2 bytes in, 1 or 0.5 byte out per element):
//   One "team" of TEAM = 2^t threads owns one token row of K = 2^k elements, V = 2^v values per
//   thread (v = k - t <= 7, so at most 128 fp32 registers of data).
//   Phase A  every thread loads bf16 pairs at j = c * 2*TEAM + 2*r + e (coalesced 4-byte loads)
//            and runs the butterflies of every index bit it holds in registers: bit 0 and the
//            top v-1 bits.  The Sylvester transform is a product of commuting per-bit
//            butterflies, so the bits may be processed in any order.
//   Phase B  the row goes through shared memory once (XOR-swizzled so both the 8-byte writes
//            and the 16-byte reads are conflict-free); each thread then holds whole contiguous
//            runs of L = 2^l elements and runs the butterflies of the remaining bits 1..t in
//            registers (for K = 2^15 and 2^14 the last one or two bits pair neighbouring
//            lanes through shuffles).
//   Quantise every thread holds contiguous runs, so codes are packed in registers (float
//            round-to-int by adding 1.5 * 2^23, byte gather with prmt) and written with 16-byte
//            stores; the team reduces max|z| and the code sum.
// Butterflies use the packed fp32x2 add/fma of sm_100.  The product that decides a code is a
// scalar __fmul_rn, which the compiler never fuses with the rounding add that follows (the
// packed forms give no such guarantee: a fused multiply-add rounds once and moves near-ties).
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

// Launch plan of the transform for K = 2^LOGK: team of 2^T_BITS threads per row, RING bf16 rows
// per team in shared memory, TEAMS teams per CTA.
template <int LOGK, int T_BITS_, int RING_, int TEAMS_>
struct FwhtPlan {
    static constexpr int K = 1 << LOGK;
    static constexpr int T_BITS = T_BITS_;
    static constexpr int TEAM = 1 << T_BITS;
    static constexpr int V_BITS = LOGK - T_BITS;
    static constexpr int V = 1 << V_BITS;  // values per thread
    static constexpr int L_BITS = V_BITS < T_BITS + 1 ? V_BITS : T_BITS + 1;
    static constexpr int L = 1 << L_BITS;  // run length held by one thread in phase B
    static constexpr int COLS = V / L;     // runs per thread
    static constexpr int SHFL_BITS = T_BITS + 1 - L_BITS;  // bits done by lane shuffles
    // bf16 rows per team in shared memory: the current one, and with RING = 2 the next
    static constexpr int RING = RING_;
    // per team: the fp32 transpose buffer (4K bytes) and RING bf16 rows (2K bytes each)
    static constexpr int TEAM_BYTES = K * 4 + RING * K * 2;
    static constexpr int TEAMS = TEAMS_;
    static constexpr int THREADS = TEAMS * TEAM;
    // resident CTAs per SM the register allocation is sized for: 16 warps per SM
    static constexpr int MIN_BLOCKS = THREADS >= 512 ? 1 : 512 / THREADS;
    static constexpr int WARPS_PER_TEAM = TEAM >= 32 ? TEAM / 32 : 1;
    static constexpr int RED = TEAMS * WARPS_PER_TEAM;  // reduction slots: max, code sum, |z| sum
    static constexpr int RED_BYTES = (2 * RED * 4 + RED * 8 + 15) / 16 * 16;
    static constexpr int CHUNKS = L / 4;                       // 16-byte chunks per run
    static constexpr int SWZ = (CHUNKS < 8 ? CHUNKS : 8) - 1;  // chunk XOR mask
    static constexpr size_t SMEM =
        (size_t)TEAMS * TEAM_BYTES + RED_BYTES + (size_t)TEAMS * RING * sizeof(uint64_t);
    static_assert(SHFL_BITS >= 0 && SHFL_BITS <= 5, "plan: shuffle partners inside a warp");
    static_assert(L >= 16, "runs must hold 16 codes");
    static_assert(V <= 128, "plan: register budget");
    static_assert(THREADS <= 1024 && THREADS % 32 == 0, "plan: CTA size");
    static_assert(TEAM <= 32 || TEAMS <= 15, "plan: one named barrier per team");
    static_assert(SMEM <= 227 * 1024, "plan: shared memory");
};

// The plan each K runs with.  Values per thread stay <= 64 from K = 2^11 up (<= 96 registers),
// with one bf16 row per team, so that 16 or more warps per SM keep rows in flight; the bits a
// thread does not hold in phase B go through lane shuffles.
template <int LOGK> struct FwhtConfig;
template <> struct FwhtConfig<7> { using P = FwhtPlan<7, 3, 2, 16>; };
template <> struct FwhtConfig<8> { using P = FwhtPlan<8, 3, 2, 16>; };
template <> struct FwhtConfig<9> { using P = FwhtPlan<9, 4, 2, 8>; };
template <> struct FwhtConfig<10> { using P = FwhtPlan<10, 4, 2, 8>; };
template <> struct FwhtConfig<11> { using P = FwhtPlan<11, 5, 1, 4>; };
template <> struct FwhtConfig<12> { using P = FwhtPlan<12, 6, 1, 2>; };
template <> struct FwhtConfig<13> { using P = FwhtPlan<13, 7, 1, 1>; };
template <> struct FwhtConfig<14> { using P = FwhtPlan<14, 8, 1, 1>; };
template <> struct FwhtConfig<15> { using P = FwhtPlan<15, 9, 1, 1>; };

__device__ __forceinline__ float2 bfly_add(float2 a, float2 b) { return add2_rn(a, b); }
__device__ __forceinline__ float2 bfly_sub(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.f, -1.f), a);  // a - b, one rounding
}

// Team-wide barrier: teams of <= 32 threads live inside one warp.
template <int TEAM>
__device__ __forceinline__ void team_sync(int team) {
    if constexpr (TEAM <= 32) {
        __syncwarp();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(team + 1), "n"(TEAM) : "memory");
    }
}

// sqrt(7) rounded to fp32: the code the mean |z| of a token maps to in the absmean INT4 quantiser
constexpr float kSqrt7 = 2.6457513110645906f;

// ABSMEAN: the INT4 quantiser (BITS == 4 only): the scale comes from the mean |z| of the token
// (summed in double) instead of max |z|, s = sqrt7 / max(mean, 1e-5), and codes are clipped to
// [-8, 7].  BITS == 4 without ABSMEAN is the variant absmax INT4 quantiser (Q = 7).
template <class P, int BITS, bool ZOUT, bool NORM, bool ABSMEAN = false>
__global__ void __launch_bounds__(P::THREADS, P::MIN_BLOCKS)
    fwht_quant_kernel(const uint8_t *__restrict__ X, int M, float rsqrt_k,
                      const uint32_t *__restrict__ gain2, float eps,
                      uint8_t *__restrict__ codes, float *__restrict__ scales,
                      int32_t *__restrict__ rowsum, float *__restrict__ zout, int *status) {
    constexpr int K = P::K, TEAM = P::TEAM, V = P::V, L = P::L;
    extern __shared__ float4 smem4[];
    float *smem = reinterpret_cast<float *>(smem4);
    const int team = threadIdx.x / TEAM;
    const int r = threadIdx.x % TEAM;
    const int lane = threadIdx.x & 31;
    float *tbuf = smem + team * K;
    float *red = smem + P::TEAMS * K;  // [RED] floats (max), then [RED] ints (code sums)
    uint8_t *rows = reinterpret_cast<uint8_t *>(red) + P::RED_BYTES;  // [TEAMS][RING][K] bf16
    uint64_t *bars = reinterpret_cast<uint64_t *>(rows + (size_t)P::TEAMS * P::RING * K * 2);
    uint8_t *ring = rows + (size_t)team * P::RING * K * 2;
    uint64_t *rbar = bars + team * P::RING;
    const int64_t stride = (int64_t)gridDim.x * P::TEAMS;
    constexpr uint32_t ROW_BYTES = K * 2;

    // the product that reads these codes may start its own set-up now (it waits for this grid
    // to complete before it reads anything)
    pdl_launch_dependents();
    // Persistent: the team walks rows base + team, base += stride.  The trip count is the same
    // for every team of the CTA (teams of <= 32 threads share a warp and its __syncwarp).  Rows
    // arrive by bulk asynchronous copies into a two-row ring, so the next row is in flight while
    // the current one is transformed.
    if (r == 0) {
        for (int i = 0; i < P::RING; ++i) mbar_init(&rbar[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // slots with a copy issued and not yet waited for, and the parity of that copy's phase
    uint32_t pending = 0, pend_ph = 0;
    int issued = 0;  // copies issued so far (sequence number of the next copy)
    auto issue = [&](int64_t rw, int slot) {
        if (rw < M) {
            if (r == 0) {
                mbar_arrive_expect_tx(&rbar[slot], ROW_BYTES);
                bulk_load(ring + (size_t)slot * ROW_BYTES, X + rw * ROW_BYTES, ROW_BYTES,
                          &rbar[slot]);
            }
            pending |= 1u << slot;
            pend_ph = (pend_ph & ~(1u << slot)) | ((uint32_t)(issued / P::RING & 1) << slot);
        }
        ++issued;
    };
    const int64_t first = (int64_t)blockIdx.x * P::TEAMS;
#pragma unroll
    for (int i = 0; i < P::RING; ++i) issue(first + i * stride + team, i);
    int iter = 0;
    bool ok = true;
    for (int64_t base = first; base < M; base += stride, ++iter) {
    const int64_t row = base + team;
    const bool valid = row < M;
    const int slot = iter % P::RING;
    if (valid && ok) {
        if (mbar_wait(&rbar[slot], (uint32_t)(iter / P::RING) & 1, status)) pending &= ~(1u << slot);
        else ok = false;
    }
    const uint32_t *xr = reinterpret_cast<const uint32_t *>(ring + (size_t)slot * ROW_BYTES);

    // ---- phase A: bf16 pairs -> fp32, butterflies over register bits ----
    float2 a[V / 2];
#pragma unroll
    for (int c = 0; c < V / 2; ++c) {
        const uint32_t w = (valid && ok) ? xr[c * TEAM + r] : 0u;
        a[c] = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
    if constexpr (NORM) {
        // RMS normalisation of the row before the transform: y = (x * rinv) * g with
        // rinv = 1 / sqrt(sum(x^2) / K + eps), every operation an IEEE fp32 one
        float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < V / 2; ++c) ss2 = __ffma2_rn(a[c], a[c], ss2);
        float ss = ss2.x + ss2.y;
        constexpr int W = TEAM < 32 ? TEAM : 32;
#pragma unroll
        for (int o = W / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        if constexpr (TEAM > 32) {
            // the previous row's reads of these slots ended before its later barriers
            constexpr int WPT = P::WARPS_PER_TEAM;
            if (lane == 0) red[team * WPT + (r >> 5)] = ss;
            team_sync<TEAM>(team);
            ss = red[team * WPT];
#pragma unroll
            for (int i = 1; i < WPT; ++i) ss += red[team * WPT + i];
        }
        const float rinv = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)K), eps)));
        const float2 r2 = make_float2(rinv, rinv);
#pragma unroll
        for (int c = 0; c < V / 2; ++c) {
            const uint32_t gw = gain2 ? __ldg(gain2 + c * TEAM + r) : 0x3F803F80u;  // 1.0, 1.0
            a[c] = mul2_rn(mul2_rn(a[c], r2),
                           make_float2(__uint_as_float(gw << 16), __uint_as_float(gw & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int c = 0; c < V / 2; ++c) {  // index bit 0 (inside the pair)
        float x = a[c].x, y = a[c].y;
        a[c] = make_float2(x + y, x - y);
    }
#pragma unroll
    for (int m = 1; m < V / 2; m <<= 1) {  // index bits t+1 .. k-1
#pragma unroll
        for (int c = 0; c < V / 2; ++c) {
            if (c & m) continue;
            float2 x = a[c], y = a[c | m];
            a[c] = bfly_add(x, y);
            a[c | m] = bfly_sub(x, y);
        }
    }
    // the refill is an async-proxy write into the slot this thread has just read: a proxy fence
    // orders the plain reads before it
    fence_proxy_async_smem();
    team_sync<TEAM>(team);  // this slot is read and the previous row's tbuf reads are done
    issue(row + P::RING * stride, slot);  // refill the slot with the row after next

    // ---- to shared memory: element j -> run R = j / L, offset o = j % L, chunk-swizzled ----
#pragma unroll
    for (int c = 0; c < V / 2; ++c) {
        const int j = c * 2 * TEAM + 2 * r;
        const int R = j >> P::L_BITS, o = j & (L - 1);
        const int phys = R * L + ((((o >> 2) ^ (R & P::SWZ))) << 2) + (o & 3);
        *reinterpret_cast<float2 *>(tbuf + phys) = a[c];
    }
    team_sync<TEAM>(team);

    // ---- phase B: whole runs per thread, butterflies over bits 1 .. l-1 ----
    float2 b[P::COLS][L / 2];
#pragma unroll
    for (int col = 0; col < P::COLS; ++col) {
        const int R = col * TEAM + r;
#pragma unroll
        for (int q = 0; q < P::CHUNKS; ++q) {
            float4 v = *reinterpret_cast<const float4 *>(tbuf + R * L + ((q ^ (R & P::SWZ)) << 2));
            b[col][2 * q] = make_float2(v.x, v.y);
            b[col][2 * q + 1] = make_float2(v.z, v.w);
        }
#pragma unroll
        for (int m = 1; m < L / 2; m <<= 1) {
#pragma unroll
            for (int p = 0; p < L / 2; ++p) {
                if (p & m) continue;
                float2 x = b[col][p], y = b[col][p | m];
                b[col][p] = bfly_add(x, y);
                b[col][p | m] = bfly_sub(x, y);
            }
        }
        // remaining bits l .. t: the partner run belongs to lane ^ (1 << sb)
#pragma unroll
        for (int sb = 0; sb < P::SHFL_BITS; ++sb) {
            const float sg = ((r >> sb) & 1) ? -1.f : 1.f;
            const float2 sg2 = make_float2(sg, sg);
#pragma unroll
            for (int p = 0; p < L / 2; ++p) {
                float2 mine = b[col][p];
                float2 other;
                other.x = __shfl_xor_sync(0xFFFFFFFFu, mine.x, 1 << sb);
                other.y = __shfl_xor_sync(0xFFFFFFFFu, mine.y, 1 << sb);
                b[col][p] = __ffma2_rn(mine, sg2, other);  // low: mine+other, high: other-mine
            }
        }
    }

    // ---- normalise and reduce max|z| (or, ABSMEAN, sum |z|) over the team ----
    const float2 rk2 = make_float2(rsqrt_k, rsqrt_k);
    float mx = 0.f;
    double sa = 0.0;
#pragma unroll
    for (int col = 0; col < P::COLS; ++col)
#pragma unroll
        for (int p = 0; p < L / 2; ++p) {
            b[col][p] = mul2_rn(b[col][p], rk2);
            if constexpr (ABSMEAN)
                sa += fabs((double)b[col][p].x) + fabs((double)b[col][p].y);
            else
                mx = fmaxf(mx, fmaxf(fabsf(b[col][p].x), fabsf(b[col][p].y)));
        }

    if constexpr (ZOUT) {
        if (valid) {
            float *zr = zout + row * K;
#pragma unroll
            for (int col = 0; col < P::COLS; ++col) {
                const int R = col * TEAM + r;
#pragma unroll
                for (int q = 0; q < L / 4; ++q)
                    *reinterpret_cast<float4 *>(zr + R * L + 4 * q) =
                        make_float4(b[col][2 * q].x, b[col][2 * q].y, b[col][2 * q + 1].x,
                                    b[col][2 * q + 1].y);
            }
        }
    } else {
        constexpr int W = TEAM < 32 ? TEAM : 32;
        static_assert(!ABSMEAN || BITS == 4, "the absmean rule is an INT4 quantiser");
        float g;
        if constexpr (ABSMEAN) {
#pragma unroll
            for (int o = W / 2; o > 0; o >>= 1) sa += __shfl_xor_sync(0xFFFFFFFFu, sa, o);
            if constexpr (TEAM > 32) {
                constexpr int WPT = P::WARPS_PER_TEAM;
                double *redd = reinterpret_cast<double *>(reinterpret_cast<uint8_t *>(red) +
                                                          2 * P::RED * 4);
                if (lane == 0) redd[team * WPT + (r >> 5)] = sa;
                team_sync<TEAM>(team);
                sa = redd[team * WPT];
#pragma unroll
                for (int i = 1; i < WPT; ++i) sa += redd[team * WPT + i];
            }
            g = (float)fmax(sa / (double)K, 1e-5);
        } else {
#pragma unroll
            for (int o = W / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
            if constexpr (TEAM > 32) {
                // all warps of this team finished their phase-B reads of tbuf before this barrier
                constexpr int WPT = P::WARPS_PER_TEAM;
                if (lane == 0) red[team * WPT + (r >> 5)] = mx;
                team_sync<TEAM>(team);
                mx = red[team * WPT];
#pragma unroll
                for (int i = 1; i < WPT; ++i) mx = fmaxf(mx, red[team * WPT + i]);
            }
            g = fmaxf(mx, 1e-5f);
        }
        constexpr float Q = ABSMEAN ? kSqrt7 : BITS == 4 ? 7.f : 127.f;
        const float s = __fdiv_rn(Q, g);
        const float dq = __fdiv_rn(g, Q);
        const float2 magic2 = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23

        int sum = 0;
#pragma unroll
        for (int col = 0; col < P::COLS; ++col) {
            const int R = col * TEAM + r;
#pragma unroll
            for (int g16 = 0; g16 < L / 16; ++g16) {
                // 16 consecutive values -> round(z * s); the integer is the low byte of the
                // float t + 1.5 * 2^23 (exact round-half-even for |t| < 2^22)
                uint32_t f[16];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    // __fmul_rn is never contracted with the following add: the code is
                    // round(fl(z * s)), the same two roundings the reference takes
                    float2 t = make_float2(__fmul_rn(b[col][g16 * 8 + i].x, s),
                                           __fmul_rn(b[col][g16 * 8 + i].y, s));
                    if constexpr (ABSMEAN)  // clip before rounding: the same as after it
                        t = make_float2(fminf(fmaxf(t.x, -8.f), 7.f), fminf(fmaxf(t.y, -8.f), 7.f));
                    float2 u = __fadd2_rn(t, magic2);
                    f[2 * i] = __float_as_uint(u.x);
                    f[2 * i + 1] = __float_as_uint(u.y);
                }
                const int64_t k0 = (int64_t)R * L + 16 * g16;
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
                    if (valid) *reinterpret_cast<uint4 *>(codes + row * K + k0) = w;
                } else {
                    uint32_t A0 = gather_low_bytes(f[0], f[1], f[2], f[3]);
                    uint32_t B0 = gather_low_bytes(f[4], f[5], f[6], f[7]);
                    uint32_t A1 = gather_low_bytes(f[8], f[9], f[10], f[11]);
                    uint32_t B1 = gather_low_bytes(f[12], f[13], f[14], f[15]);
                    sum = __dp4a((int)A0, 0x01010101, sum);
                    sum = __dp4a((int)B0, 0x01010101, sum);
                    sum = __dp4a((int)A1, 0x01010101, sum);
                    sum = __dp4a((int)B1, 0x01010101, sum);
                    uint2 w;
                    w.x = (A0 & 0x0F0F0F0Fu) | ((B0 << 4) & 0xF0F0F0F0u);
                    w.y = (A1 & 0x0F0F0F0Fu) | ((B1 << 4) & 0xF0F0F0F0u);
                    if (valid) *reinterpret_cast<uint2 *>(codes + row * (K / 2) + k0 / 2) = w;
                }
            }
        }
#pragma unroll
        for (int o = W / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        if constexpr (TEAM > 32) {
            constexpr int WPT = P::WARPS_PER_TEAM;
            int *redi = reinterpret_cast<int *>(red) + P::RED;
            if (lane == 0) redi[team * WPT + (r >> 5)] = sum;
            team_sync<TEAM>(team);
            sum = 0;
#pragma unroll
            for (int i = 0; i < WPT; ++i) sum += redi[team * WPT + i];
        }
        if (valid && r == 0) {
            scales[row] = dq;
            rowsum[row] = sum;
        }
    }
    }  // row loop
    // after a time-out, no copy may still be landing in shared memory when the CTA exits
    for (int i = 0; i < P::RING; ++i)
        if (pending & (1u << i)) mbar_wait(&rbar[i], (pend_ph >> i) & 1, status);
}

// ---- plain BitLinear: absmax quantisation without a transform (any K % 128 == 0) ----
// One warp per token row, two passes over the row (the second one hits L1/L2).
// With NORM each value is first RMS-normalised, y = (x * rinv) * g as in fwht_quant_kernel (an
// extra pass over the row for sum(x^2)); with ZOUT the kernel writes y in fp32 instead of codes.
template <int BITS, bool NORM, bool ZOUT, bool ABSMEAN = false>
__global__ void __launch_bounds__(256)
    act_quant_plain_kernel(const uint4 *__restrict__ X, int64_t M, int64_t K,
                           const uint4 *__restrict__ gain8, float eps,
                           uint8_t *__restrict__ codes, float *__restrict__ scales,
                           int32_t *__restrict__ rowsum, float *__restrict__ zout) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    pdl_launch_dependents();  // as in fwht_quant_kernel
    if (row >= M) return;  // whole warp leaves together
    const uint4 *xr = X + row * (K / 8);
    const int64_t nchunk = K / 8;
    float rinv = 1.f;
    if constexpr (NORM) {
        float ss = 0.f;
        for (int64_t c = lane; c < nchunk; c += 32) {
            const uint4 v = __ldg(xr + c);
            const uint32_t h[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float x0 = __uint_as_float(h[i] << 16), x1 = __uint_as_float(h[i] & 0xFFFF0000u);
                ss = __fmaf_rn(x0, x0, ss);
                ss = __fmaf_rn(x1, x1, ss);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        rinv = __fdiv_rn(1.f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)K), eps)));
    }
    // the eight values of chunk c as four float pairs (normalised with NORM)
    auto load8 = [&](int64_t c, float2 (&y)[4]) {
        const uint4 v = __ldg(xr + c);
        const uint32_t h[4] = {v.x, v.y, v.z, v.w};
        uint32_t gh[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};  // unit gain
        if (NORM && gain8) {
            const uint4 gv = __ldg(gain8 + c);
            gh[0] = gv.x; gh[1] = gv.y; gh[2] = gv.z; gh[3] = gv.w;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            y[i] = make_float2(__uint_as_float(h[i] << 16), __uint_as_float(h[i] & 0xFFFF0000u));
            if constexpr (NORM)
                y[i] = mul2_rn(mul2_rn(y[i], make_float2(rinv, rinv)),
                               make_float2(__uint_as_float(gh[i] << 16),
                                           __uint_as_float(gh[i] & 0xFFFF0000u)));
        }
    };
    if constexpr (ZOUT) {
        for (int64_t c = lane; c < nchunk; c += 32) {
            float2 y[4];
            load8(c, y);
            float4 *zr = reinterpret_cast<float4 *>(zout + row * K + 8 * c);
            zr[0] = make_float4(y[0].x, y[0].y, y[1].x, y[1].y);
            zr[1] = make_float4(y[2].x, y[2].y, y[3].x, y[3].y);
        }
        return;
    }
    static_assert(!ABSMEAN || BITS == 4, "the absmean rule is an INT4 quantiser");
    float mx = 0.f;
    double sa = 0.0;  // ABSMEAN: sum |y| in double (see fwht_quant_kernel)
    for (int64_t c = lane; c < nchunk; c += 32) {
        float2 y[4];
        load8(c, y);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (ABSMEAN)
                sa += fabs((double)y[i].x) + fabs((double)y[i].y);
            else
                mx = fmaxf(mx, fmaxf(fabsf(y[i].x), fabsf(y[i].y)));
        }
    }
    float g;
    if constexpr (ABSMEAN) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sa += __shfl_xor_sync(0xFFFFFFFFu, sa, o);
        g = (float)fmax(sa / (double)K, 1e-5);
    } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        g = fmaxf(mx, 1e-5f);
    }
    constexpr float Q = ABSMEAN ? kSqrt7 : BITS == 4 ? 7.f : 127.f;
    const float s = __fdiv_rn(Q, g);
    const float dq = __fdiv_rn(g, Q);
    const float2 magic2 = make_float2(12582912.f, 12582912.f);
    int sum = 0;
    for (int64_t c = lane; c < nchunk; c += 32) {
        float2 y[4];
        load8(c, y);
        uint32_t f[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // __fmul_rn is never contracted with the following add (see fwht_quant_kernel)
            float2 t = make_float2(__fmul_rn(y[i].x, s), __fmul_rn(y[i].y, s));
            if constexpr (ABSMEAN)
                t = make_float2(fminf(fmaxf(t.x, -8.f), 7.f), fminf(fmaxf(t.y, -8.f), 7.f));
            float2 u = __fadd2_rn(t, magic2);
            f[2 * i] = __float_as_uint(u.x);
            f[2 * i + 1] = __float_as_uint(u.y);
        }
        uint32_t A = gather_low_bytes(f[0], f[1], f[2], f[3]);
        uint32_t B = gather_low_bytes(f[4], f[5], f[6], f[7]);
        sum = __dp4a((int)A, 0x01010101, sum);
        sum = __dp4a((int)B, 0x01010101, sum);
        if constexpr (BITS == 8) {
            *reinterpret_cast<uint2 *>(codes + row * K + 8 * c) = make_uint2(A, B);
        } else {
            *reinterpret_cast<uint32_t *>(codes + row * (K / 2) + 4 * c) =
                (A & 0x0F0F0F0Fu) | ((B << 4) & 0xF0F0F0F0u);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane == 0) {
        scales[row] = dq;
        rowsum[row] = sum;
    }
}

template <class P, int BITS, bool ZOUT, bool NORM, bool ABSMEAN = false>
static cudaError_t launch_fwht_t(const void *X, int64_t M, const NormArgs &nrm, void *codes,
                                 float *scales, int32_t *rowsum, float *zout, int *status,
                                 cudaStream_t stream) {
    auto kern = fwht_quant_kernel<P, BITS, ZOUT, NORM, ABSMEAN>;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)P::SMEM);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    static int per_sm[64] = {};
    static int num_sms[64] = {};
    if (dev >= 0 && dev < 64 && per_sm[dev] == 0) {
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[dev], kern, P::THREADS, P::SMEM);
        cudaDeviceGetAttribute(&num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (per_sm[dev] < 1) per_sm[dev] = 1;
    }
    const int64_t want = (M + P::TEAMS - 1) / P::TEAMS;
    const int64_t cap = (int64_t)(dev >= 0 && dev < 64 ? per_sm[dev] * num_sms[dev] : 148);
    const int64_t blocks = want < cap ? want : cap;
    const float rk = (float)(1.0 / sqrt((double)P::K));
    kern<<<(unsigned)blocks, P::THREADS, P::SMEM, stream>>>(
        reinterpret_cast<const uint8_t *>(X), (int)M, rk,
        reinterpret_cast<const uint32_t *>(nrm.gain), nrm.eps,
        reinterpret_cast<uint8_t *>(codes), scales, rowsum, zout, status);
    return cudaGetLastError();
}

template <int LOGK, bool NORM>
static cudaError_t launch_fwht_n(const void *X, int64_t M, int act_bits, const NormArgs &nrm,
                                 void *codes, float *scales, int32_t *rowsum, float *zout,
                                 int *status, cudaStream_t stream) {
    using P = typename FwhtConfig<LOGK>::P;
    if (act_bits == kActInt4Absmax) {
        if constexpr (NORM) return cudaErrorInvalidValue;  // not offered with the norm
        else
            return launch_fwht_t<P, 4, false, false, false>(X, M, nrm, codes, scales, rowsum,
                                                             nullptr, status, stream);
    }
    if (zout)
        return launch_fwht_t<P, 8, true, NORM>(X, M, nrm, codes, scales, rowsum, zout, status,
                                               stream);
    if (act_bits == 4)
        return launch_fwht_t<P, 4, false, NORM, true>(X, M, nrm, codes, scales, rowsum, zout,
                                                      status, stream);
    return launch_fwht_t<P, 8, false, NORM>(X, M, nrm, codes, scales, rowsum, zout, status,
                                            stream);
}

template <int LOGK>
static cudaError_t launch_fwht_k(const void *X, int64_t M, int act_bits, const NormArgs &nrm,
                                 void *codes, float *scales, int32_t *rowsum, float *zout,
                                 int *status, cudaStream_t stream) {
    return nrm.on ? launch_fwht_n<LOGK, true>(X, M, act_bits, nrm, codes, scales, rowsum, zout,
                                              status, stream)
                  : launch_fwht_n<LOGK, false>(X, M, act_bits, nrm, codes, scales, rowsum, zout,
                                               status, stream);
}

cudaError_t launch_fwht_quant(const void *X, int64_t M, int logk, int act_bits,
                              const NormArgs &nrm, void *codes, float *scales, int32_t *rowsum,
                              float *zout, int *status, cudaStream_t stream) {
#define BITNET_FWHT_CASE(L) \
    case L: return launch_fwht_k<L>(X, M, act_bits, nrm, codes, scales, rowsum, zout, status, stream)
    switch (logk) {
        BITNET_FWHT_CASE(7);
        BITNET_FWHT_CASE(8);
        BITNET_FWHT_CASE(9);
        BITNET_FWHT_CASE(10);
        BITNET_FWHT_CASE(11);
        BITNET_FWHT_CASE(12);
        BITNET_FWHT_CASE(13);
        BITNET_FWHT_CASE(14);
        BITNET_FWHT_CASE(15);
        default: return cudaErrorInvalidValue;
    }
#undef BITNET_FWHT_CASE
}

template <int BITS, bool NORM, bool ZOUT, bool ABSMEAN = false>
static cudaError_t launch_plain_t(const void *X, int64_t M, int64_t K, const NormArgs &nrm,
                                  void *codes, float *scales, int32_t *rowsum, float *zout,
                                  cudaStream_t stream) {
    const int64_t blocks = (M + 7) / 8;
    act_quant_plain_kernel<BITS, NORM, ZOUT, ABSMEAN><<<(unsigned)blocks, 256, 0, stream>>>(
        reinterpret_cast<const uint4 *>(X), M, K, reinterpret_cast<const uint4 *>(nrm.gain),
        nrm.eps, reinterpret_cast<uint8_t *>(codes), scales, rowsum, zout);
    return cudaGetLastError();
}

cudaError_t launch_act_quant_plain(const void *X, int64_t M, int64_t K, int act_bits,
                                   const NormArgs &nrm, void *codes, float *scales,
                                   int32_t *rowsum, float *zout, cudaStream_t stream) {
    if (act_bits == kActInt4Absmax) {
        if (nrm.on || zout) return cudaErrorInvalidValue;
        return launch_plain_t<4, false, false>(X, M, K, nrm, codes, scales, rowsum, zout, stream);
    }
    if (zout)  // the normalised rows themselves (the parity entry); only with a norm
        return launch_plain_t<8, true, true>(X, M, K, nrm, codes, scales, rowsum, zout, stream);
    if (nrm.on)
        return act_bits == 4
                   ? launch_plain_t<4, true, false, true>(X, M, K, nrm, codes, scales, rowsum,
                                                          zout, stream)
                   : launch_plain_t<8, true, false>(X, M, K, nrm, codes, scales, rowsum, zout, stream);
    return act_bits == 4
               ? launch_plain_t<4, false, false, true>(X, M, K, nrm, codes, scales, rowsum, zout,
                                                       stream)
               : launch_plain_t<8, false, false>(X, M, K, nrm, codes, scales, rowsum, zout, stream);
}

}  // namespace bitnet
