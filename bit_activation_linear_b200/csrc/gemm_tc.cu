// gemm_tc.cu -- step 4 for many tokens (prefill): the ternary x integer product on the
// 5th-generation tensor cores (tcgen05, kind::i8), accumulating in int32 in tensor memory,
// with the rescale to bf16 fused into the epilogue.
//
// 2B4T article, section 一.2 (W1.58A8 BitLinear; the product needs only additions and
// subtractions) and section 三.3 (GPU kernel: pack-store-load-unpack-compute).  On sm_100a the
// cheapest exact "add/subtract" is the int8 tensor-core MMA: the 2-bit weights are unpacked
// on chip, never in HBM.
//
// Tile: 128 output features (MMA M, operand A) x 256 tokens (MMA N, operand B), both operands
// in shared memory, K in stages of 128 (four 128x256x32 MMAs, 512 tensor cycles).  Measured on
// B200: a tcgen05.mma issues in ~45 cycles, a commit costs ~50, and an mbarrier test issued after
// MMAs returns ~180 cycles later, so the MMA thread tests the next stage before issuing the
// current one and every instruction it issues covers 128 tensor cycles; the tensor core reads
// its shared-memory operands at full rate while other warps write shared memory.  The two
// 256-column int32 accumulators fill the 512 TMEM columns, so one tile's epilogue overlaps the
// next tile's main loop.  A persistent CTA per SM walks its tiles; warp roles:
//   warp 0       code-tile TMA (INT8): [256 tokens x 128 B] with the 128-byte swizzle (the UMMA
//                K-major layout), four tiles in flight: under full load a load lands ~1800
//                cycles after it is issued.
//   warp 2       weight-tile TMA: packed weights [128 rows x 64 B] (two K stages).
//   warp 1       MMA issuer (and TMEM owner): tcgen05.mma.kind::i8, A = unsigned bytes
//                u = q + 1, B = signed codes c, D += u * c; tcgen05.commit frees stages and
//                publishes finished accumulators; it also frees a weight tile once the A stages
//                made from it are complete.
//   warps 4-7/11 A producers (two groups taking alternate stages for INT8, one for INT4):
//                thread i expands the 32 packed bytes of output feature n0 + i for the stage
//                (one shift-and-mask per four weights) and stores the 128 int8 bytes in the
//                swizzled K-major layout.  The 2-bit weights never exist unpacked in HBM.
//   warps 8-11   (INT4 only) B producers: coalesced 16-byte loads of nibble codes, sign-extended
//                to int8 in registers and stored in the swizzled K-major layout.
//   warps 12-19  two epilogue warpgroups, each taking half of the tile's tokens: tcgen05.ld of
//                the int32 accumulator, subtract the token's code sum (sum_k q*c =
//                sum_k u*c - sum_k c), scale by d_m * gamma, round to bf16 and store: lane pairs
//                swap one value so each half-warp writes a contiguous 64-byte row segment.
// Every wait is bounded: after ~1 s a role records BITNET_ERR_TIMEOUT and stops; in-flight TMA
// loads and MMAs are drained before TMEM is released.  No cluster multicast is used.
#include "common.cuh"
#include "kernels.h"

#include <cudaTypedefs.h>

namespace bitnet {
namespace tc {

constexpr int BW = 128;    // output features per tile (MMA M)
constexpr int BT = 256;    // tokens per tile (MMA N)
constexpr int BK = 128;    // K per stage: one 128-byte swizzled row of int8
constexpr int UMMA_K = 32;
constexpr int MMAS = BK / UMMA_K;  // 4 per stage
constexpr int B_STAGES = 4;        // code tiles in flight (a TMA load takes ~1800 cycles to land)
constexpr int A_STAGES = 4;        // unpacked A tiles
constexpr int W_STAGES = 3;        // packed-weight tiles in flight
constexpr int SPW = 2;             // K stages per packed-weight tile [128 rows x 64 B]
constexpr int ACC_BUFS = 2;
constexpr int TMEM_COLS = 512;
constexpr int A_STAGE_BYTES = BW * BK;  // 16 KB
constexpr int B_STAGE_BYTES = BT * BK;  // 32 KB
constexpr int W_STAGE_BYTES = BW * SPW * BK / 4;
constexpr int EPI_WARPS = 8;
constexpr uint32_t IDESC = idesc_i8_u8s8(BW, BT);
static_assert(ACC_BUFS * BT <= TMEM_COLS, "TMEM budget");

constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_WTMA = 2, WARP_A0 = 4, WARP_B4 = 8, WARP_EPI = 12;
constexpr int NUM_THREADS = 20 * 32;

struct __align__(8) Barriers {
    uint64_t full_b[B_STAGES];   // code tile landed
    uint64_t empty_b[B_STAGES];  // the MMAs that read it have completed
    uint64_t full_a[A_STAGES];   // unpacked A tile written
    uint64_t empty_a[A_STAGES];
    uint64_t full_w[W_STAGES];
    uint64_t empty_w[W_STAGES];
    uint64_t acc_full[ACC_BUFS];
    uint64_t acc_empty[ACC_BUFS];
    uint64_t done;
    uint32_t tmem_base;
};

constexpr size_t OFF_A = 0;
constexpr size_t OFF_B = OFF_A + (size_t)A_STAGES * A_STAGE_BYTES;
constexpr size_t OFF_W = OFF_B + (size_t)B_STAGES * B_STAGE_BYTES;
constexpr size_t OFF_SCALE = OFF_W + (size_t)W_STAGES * W_STAGE_BYTES;  // [8 warps][BT/2] floats
constexpr size_t OFF_RSUM = OFF_SCALE + EPI_WARPS * (BT / 2) * sizeof(float);
constexpr size_t OFF_BAR = OFF_RSUM + EPI_WARPS * (BT / 2) * sizeof(int32_t);
constexpr size_t SMEM_BYTES = OFF_BAR + sizeof(Barriers) + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast, __syncwarp orders the
// other lanes after the acquire (needed before warp-collective .sync.aligned tcgen05 ops).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, status);
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

template <int BITS, bool OUT_I32>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ternary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                           const __grid_constant__ CUtensorMap tmap_w,
                           void *__restrict__ Yout, const uint8_t *__restrict__ codes4,
                           const float *__restrict__ scales,
                           const int32_t *__restrict__ rowsum, const float *__restrict__ gamma_ptr,
                           int M, int N, int K, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sa = smem + OFF_A;
    uint8_t *sb = smem + OFF_B;
    uint8_t *sw = smem + OFF_W;
    float *s_scale = reinterpret_cast<float *>(smem + OFF_SCALE);
    int32_t *s_rsum = reinterpret_cast<int32_t *>(smem + OFF_RSUM);
    Barriers *bar = reinterpret_cast<Barriers *>(smem + OFF_BAR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_wtiles = (N + BW - 1) / BW;
    const int n_ttiles = (M + BT - 1) / BT;
    const int num_tiles = n_wtiles * n_ttiles;
    const int KS = K / BK;                 // stages per tile
    const int WPT = (KS + SPW - 1) / SPW;  // weight tiles per output tile
    constexpr int A_GROUPS = BITS == 8 ? 2 : 1;
    const int my_tiles =
        (int)blockIdx.x < num_tiles ? (num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_tiles * KS;  // (tile, stage) iterations of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < B_STAGES; ++s) {
            // the TMA arrival (INT8) or the four INT4 producer warps
            mbar_init(&bar->full_b[s], BITS == 8 ? 1 : 4);
            mbar_init(&bar->empty_b[s], 1);
        }
        for (int s = 0; s < A_STAGES; ++s) {
            mbar_init(&bar->full_a[s], 4);
            mbar_init(&bar->empty_a[s], 1);
        }
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&bar->full_w[s], 1);
            mbar_init(&bar->empty_w[s], 1);
        }
        for (int s = 0; s < ACC_BUFS; ++s) {
            mbar_init(&bar->acc_full[s], 1);
            mbar_init(&bar->acc_empty[s], EPI_WARPS);
        }
        mbar_init(&bar->done, 1);
        fence_mbar_init();
    }
    if (warp == WARP_TMA && lane == 0) {
        if (BITS == 8) prefetch_tensormap(&tmap_codes);
        prefetch_tensormap(&tmap_w);
    }
    if (warp == WARP_MMA) {
        tmem_alloc(&bar->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == WARP_TMA) {
        // ------------------------------------------------------------------ code-tile TMA
        if (BITS == 8 && lane == 0) {
            uint32_t issued = 0, ph = 0;  // for the final drain
            int t = 0, ks = 0;
            for (int it = 0; it < total; ++it) {
                const int tile = blockIdx.x + t * gridDim.x;
                const int s = it % B_STAGES;
                const uint32_t p = (uint32_t)(it / B_STAGES) & 1;
                if (!mbar_wait(&bar->empty_b[s], p ^ 1, status)) break;
                mbar_arrive_expect_tx(&bar->full_b[s], B_STAGE_BYTES);
                tma_load_2d(sb + (size_t)s * B_STAGE_BYTES, &tmap_codes, ks * BK,
                            (tile / n_wtiles) * BT, &bar->full_b[s]);
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
                if (++ks == KS) { ks = 0; ++t; }
            }
            // no copy may still be writing shared memory when the CTA exits
            for (int i = 0; i < B_STAGES; ++i)
                if (issued & (1u << i)) mbar_wait(&bar->full_b[i], (ph >> i) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_WTMA) {
        // ------------------------------------------------------------------ weight-tile TMA
        if (lane == 0) {
            uint32_t issued = 0, ph = 0;
            const int w_total = my_tiles * WPT;
            for (int w = 0; w < w_total; ++w) {
                const int s_w = w % W_STAGES;
                const uint32_t p_w = (uint32_t)(w / W_STAGES) & 1;
                if (!mbar_wait(&bar->empty_w[s_w], p_w ^ 1, status)) break;
                const int tile_w = blockIdx.x + (w / WPT) * gridDim.x;
                mbar_arrive_expect_tx(&bar->full_w[s_w], W_STAGE_BYTES);
                tma_load_2d(sw + (size_t)s_w * W_STAGE_BYTES, &tmap_w, (w % WPT) * SPW * (BK / 4),
                            (tile_w % n_wtiles) * BW, &bar->full_w[s_w]);
                issued |= 1u << s_w;
                ph = (ph & ~(1u << s_w)) | (p_w << s_w);
            }
            for (int i = 0; i < W_STAGES; ++i)
                if (issued & (1u << i)) mbar_wait(&bar->full_w[i], (ph >> i) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sa_addr = smem_addr(sa);
            const uint32_t sb_addr = smem_addr(sb);
            bool ok = true;
            bool next_a = total > 0 && mbar_test_wait(&bar->full_a[0], 0);
            bool next_b = total > 0 && mbar_test_wait(&bar->full_b[0], 0);
            int t = 0, ks = 0;
            for (int it = 0; it < total; ++it) {
                const int ab = t & 1;
                const int sa_i = it % A_STAGES, sb_i = it % B_STAGES;
                if (ks == 0 &&
                    !mbar_wait(&bar->acc_empty[ab], ((uint32_t)(t >> 1) & 1) ^ 1, status)) {
                    ok = false;
                    break;
                }
                if ((!next_a && !mbar_wait(&bar->full_a[sa_i], (uint32_t)(it / A_STAGES) & 1, status)) ||
                    (!next_b && !mbar_wait(&bar->full_b[sb_i], (uint32_t)(it / B_STAGES) & 1, status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // ask now whether the next stage is ready: the answers are needed only after this
                // stage's MMAs have been issued, so their latency is hidden behind them
                if (it + 1 < total) {
                    next_a = mbar_test_wait(&bar->full_a[(it + 1) % A_STAGES],
                                            (uint32_t)((it + 1) / A_STAGES) & 1);
                    next_b = mbar_test_wait(&bar->full_b[(it + 1) % B_STAGES],
                                            (uint32_t)((it + 1) / B_STAGES) & 1);
                }
                const uint32_t d_tmem = tmem + ab * BT;
                const uint64_t adesc = smem_desc_kmajor_sw128(sa_addr + (uint32_t)sa_i * A_STAGE_BYTES);
                const uint64_t bdesc = smem_desc_kmajor_sw128(sb_addr + (uint32_t)sb_i * B_STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < MMAS; ++kk)
                    mma_i8_ss(d_tmem, adesc + (uint64_t)(kk * UMMA_K / 16),
                              bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                              (ks | kk) != 0 ? 1u : 0u);
                mma_commit(&bar->empty_b[sb_i]);
                mma_commit(&bar->empty_a[sa_i]);
                // the A tiles made from this weight tile are complete (full_a observed): refill it
                if (ks % SPW == SPW - 1 || ks == KS - 1)
                    mbar_arrive(&bar->empty_w[(t * WPT + ks / SPW) % W_STAGES]);
                if (ks == KS - 1) mma_commit(&bar->acc_full[ab]);
                if (++ks == KS) { ks = 0; ++t; }
            }
            (void)ok;
            // every MMA issued above has finished before TMEM is released
            mma_commit(&bar->done);
            mbar_wait(&bar->done, 0, status);
        }
        __syncwarp();
    } else if (warp >= WARP_A0 && warp < WARP_A0 + 4 * A_GROUPS) {
        // ------------------------------------------------------------------ A producers
        const int grp = (warp - WARP_A0) >> 2;  // takes iterations it = grp (mod A_GROUPS)
        const int rr = (warp & 3) * 32 + lane;  // row of the A tile = output feature n0 + rr
        for (int it = grp; it < total; it += A_GROUPS) {
            const int t = it / KS, ks = it - t * KS;
            const int wseq = t * WPT + ks / SPW;
            const int s_w = wseq % W_STAGES, s = it % A_STAGES;
            if (!warp_wait(&bar->full_w[s_w], (uint32_t)(wseq / W_STAGES) & 1, status, lane)) break;
            // row rr of the weight tile: SPW stages x 32 B
            const uint4 *wsrc = reinterpret_cast<const uint4 *>(
                sw + (size_t)s_w * W_STAGE_BYTES + rr * (SPW * BK / 4) + (ks % SPW) * (BK / 4));
            const uint4 p0 = wsrc[0], p1 = wsrc[1];
            const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            if (!warp_wait(&bar->empty_a[s], ((uint32_t)(it / A_STAGES) & 1) ^ 1, status, lane)) break;
            // packed word g holds k = 16g .. 16g+15; (w >> 2p) & 0x03030303 is k = 16g+4p .. +3,
            // so word g becomes the 16-byte chunk g of the row, stored at chunk g ^ (rr & 7)
            uint8_t *arow = sa + (size_t)s * A_STAGE_BYTES + rr * 128;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                uint4 o;
                o.x = w[g] & 0x03030303u;
                o.y = (w[g] >> 2) & 0x03030303u;
                o.z = (w[g] >> 4) & 0x03030303u;
                o.w = (w[g] >> 6) & 0x03030303u;
                *reinterpret_cast<uint4 *>(arow + ((g ^ (rr & 7)) << 4)) = o;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->full_a[s]);
        }
    } else if (warp >= WARP_EPI && warp < WARP_EPI + EPI_WARPS) {
        // ------------------------------------------------------------------ epilogue
        const int wq = warp & 3;                  // TMEM lanes 32*wq .. 32*wq+31
        const int half = (warp - WARP_EPI) >> 2;  // tokens 128*half .. 128*half+127 of the tile
        const int ew = warp - WARP_EPI;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        float *w_scale = s_scale + ew * (BT / 2);  // this warp's copy: no cross-warp barrier
        int32_t *w_rsum = s_rsum + ew * (BT / 2);
        const float gamma = *gamma_ptr;
        const bool odd = lane & 1;
        for (int t = 0; t < my_tiles; ++t) {
            const int tile = blockIdx.x + t * gridDim.x;
            const int nw = tile % n_wtiles;
            const int mt = tile / n_wtiles;
            const int ab = t & 1;
            __syncwarp();  // the previous tile's scales are no longer read
#pragma unroll
            for (int i = 0; i < BT / 64; ++i) {
                const int ml = i * 32 + lane;
                const int64_t m = (int64_t)mt * BT + half * (BT / 2) + ml;
                w_scale[ml] = m < M ? scales[m] * gamma : 0.f;
                w_rsum[ml] = m < M ? rowsum[m] : 0;
            }
            if (!warp_wait(&bar->acc_full[ab], (uint32_t)(t >> 1) & 1, status, lane)) break;
            tc_fence_after();
            const int n = nw * BW + wq * 32 + lane;  // this lane's output feature
#pragma unroll 1
            for (int ch = 0; ch < BT / 64; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_lane + ab * BT + half * (BT / 2) + ch * 32, v);
                tmem_wait_ld();
                const int64_t m_base = (int64_t)mt * BT + half * (BT / 2) + ch * 32;
                if constexpr (OUT_I32) {
                    int32_t *out = reinterpret_cast<int32_t *>(Yout);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int64_t m = m_base + i;
                        if (m < M && n < N) out[m * N + n] = (int)v[i] - w_rsum[ch * 32 + i];
                    }
                } else {
                    // this lane holds column n of rows i; lane pairs swap one value so the even
                    // lane stores row i (n, n+1) and the odd lane row i+1 (n-1, n): each half-warp
                    // writes one contiguous 64-byte row segment
                    __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(Yout);
                    const int n_pair = nw * BW + wq * 32 + (lane & ~1);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const int m0 = ch * 32 + i;
                        const float2 sc = *reinterpret_cast<const float2 *>(w_scale + m0);
                        const int2 rs = *reinterpret_cast<const int2 *>(w_rsum + m0);
                        const float y0 = (float)((int)v[i] - rs.x) * sc.x;
                        const float y1 = (float)((int)v[i + 1] - rs.y) * sc.y;
                        const float other = __shfl_xor_sync(0xFFFFFFFFu, odd ? y0 : y1, 1);
                        const __nv_bfloat162 pr =
                            odd ? __floats2bfloat162_rn(other, y1) : __floats2bfloat162_rn(y0, other);
                        const int64_t m = m_base + i + (odd ? 1 : 0);
                        if (m < M && n_pair < N)
                            *reinterpret_cast<__nv_bfloat162 *>(out + m * N + n_pair) = pr;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->acc_empty[ab]);
        }
    } else if (BITS == 4 && warp >= WARP_B4 && warp < WARP_B4 + 4) {
        // ------------------------------------------------------------------ INT4 B producer
        // warp w covers tokens 64w .. 64w+63 of the tile; in sub-step i, lane l loads the
        // 16-byte quarter (l % 4) of token 64w + 8i + l / 4: 8 tokens x 64 B per instruction,
        // fully used sectors.  The next stage's bytes are loaded before this one is stored.
        const int wq = warp - WARP_B4;
        const int q = lane & 3;
        uint4 nxt[8];
        auto fetch = [&](int it2) {
            const int t2 = it2 / KS, ks2 = it2 - t2 * KS;
            const int tile2 = blockIdx.x + t2 * gridDim.x;
            const int64_t mbase = (int64_t)(tile2 / n_wtiles) * BT + wq * 64 + (lane >> 2);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t m = mbase + 8 * i;
                nxt[i] = (it2 < total && m < M)
                             ? ldg_nc_v4(codes4 + m * (K / 2) + ks2 * (BK / 2) + q * 16)
                             : make_uint4(0, 0, 0, 0);
            }
        };
        fetch(0);
        for (int it = 0; it < total; ++it) {
            const int s = it % B_STAGES;
            uint4 raw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) raw[i] = nxt[i];
            fetch(it + 1);
            if (!warp_wait(&bar->empty_b[s], ((uint32_t)(it / B_STAGES) & 1) ^ 1, status, lane))
                break;
            uint8_t *dst = sb + (size_t)s * B_STAGE_BYTES;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = wq * 64 + 8 * i + (lane >> 2);
                // 32 codes k = 32q .. 32q+31 -> chunks 2q (words x, y) and 2q+1 (words z, w)
                const uint32_t wd[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w0 = wd[2 * h], w1 = wd[2 * h + 1];
                    uint4 o;
                    o.x = sext_nibbles(w0 & 0x0F0F0F0Fu);
                    o.y = sext_nibbles((w0 >> 4) & 0x0F0F0F0Fu);
                    o.z = sext_nibbles(w1 & 0x0F0F0F0Fu);
                    o.w = sext_nibbles((w1 >> 4) & 0x0F0F0F0Fu);
                    const int c = 2 * q + h;
                    *reinterpret_cast<uint4 *>(dst + row * 128 + ((c ^ (row & 7)) << 4)) = o;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->full_b[s]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int BITS, bool OUT_I32>
static cudaError_t launch_tc_t(const GemmArgs &a, const CUtensorMap &mc, const CUtensorMap &mw,
                               void *out, int grid, cudaStream_t stream) {
    auto kern = ternary_gemm_tc_kernel<BITS, OUT_I32>;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    kern<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(
        mc, mw, out, reinterpret_cast<const uint8_t *>(a.codes), a.scales, a.rowsum, a.gamma,
        (int)a.M, (int)a.N, (int)a.K, a.status);
    return cudaGetLastError();
}

}  // namespace tc

static CUresult encode_2d(void *encode_fn, CUtensorMap *map, CUtensorMapDataType dt,
                          const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                          uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
    auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(encode_fn);
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

cudaError_t launch_ternary_gemm_tc(const GemmArgs &a, void *encode_fn, int num_sms,
                                   cudaStream_t stream) {
    using namespace tc;
    const int64_t tiles = ((a.N + BW - 1) / BW) * ((a.M + BT - 1) / BT);
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    CUtensorMap mc, mw;
    memset(&mc, 0, sizeof mc);
    memset(&mw, 0, sizeof mw);
    if (a.act_bits == 8 &&
        encode_2d(encode_fn, &mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, (uint64_t)a.K,
                  (uint64_t)a.M, (uint64_t)a.K, BK, BT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // packed weights: [N rows][K/4 bytes], one [128 x 64 B] box (two K stages) per tile
    if (encode_2d(encode_fn, &mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, (uint64_t)a.K / 4,
                  (uint64_t)a.N, (uint64_t)a.K / 4, SPW * BK / 4, BW,
                  CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (a.Y) {
        e = a.act_bits == 8 ? launch_tc_t<8, false>(a, mc, mw, a.Y, grid, stream)
                            : launch_tc_t<4, false>(a, mc, mw, a.Y, grid, stream);
        if (e != cudaSuccess) return e;
    }
    if (a.acc) {
        e = a.act_bits == 8 ? launch_tc_t<8, true>(a, mc, mw, a.acc, grid, stream)
                            : launch_tc_t<4, true>(a, mc, mw, a.acc, grid, stream);
    }
    return e;
}

}  // namespace bitnet
