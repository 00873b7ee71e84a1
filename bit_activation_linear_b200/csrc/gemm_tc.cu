// gemm_tc.cu -- step 4 for many tokens (prefill): the ternary x integer product on the
// 5th-generation tensor cores (tcgen05, kind::i8), accumulating in int32 in tensor memory,
// with the rescale to bf16 fused into the epilogue.
//
// 2B4T article, section 一.2 (W1.58A8 BitLinear; the product needs only additions and
// subtractions) and section 三.3 (GPU kernel: pack-store-load-unpack-compute).  On sm_100a the
// cheapest exact "add/subtract" is the int8 tensor-core MMA: the 2-bit weights are unpacked
// on chip, never in HBM.
//
// Tile: 128 output features (MMA M, operand A) x 128 tokens (MMA N, operand B).  K advances in
// stages of 256 (eight 128x128x32 MMAs).  Measured on B200: one tcgen05.mma issues in ~45 cycles
// and runs 64 cycles at this shape, a commit costs ~50 issue cycles, and an mbarrier test issued
// after MMAs returns ~180 cycles later; so a stage must hold enough MMAs to pay for its one wait
// and one commit, and the MMA thread tests the next stage before it issues the current one.
// A persistent CTA per SM walks its tiles; warp roles:
//   warp 0       TMA producer: packed weight tiles [128 rows x 128 B] (two K stages) and (INT8)
//                code tiles [128 tokens x 128 B] x 2 per stage, all with the 128-byte swizzle;
//                the code tiles land straight in the UMMA K-major layout.
//   warp 1       MMA issuer (and TMEM owner): tcgen05.mma.kind::i8 with A from TMEM (unsigned
//                bytes u = q + 1) and B from shared memory (signed codes c), D += u * c;
//                tcgen05.commit frees stages and publishes finished accumulators; it also frees a
//                weight tile once the A stages made from it are in TMEM.
//   warps 2-3    (INT4 only) B producer: coalesced 16-byte loads of nibble codes, sign-extended
//                to int8 in registers and stored in the swizzled K-major layout.
//   warps 4-11   two A-producer warpgroups taking alternate stages.  Thread i of a group owns
//                TMEM lane i (output feature n0 + i): it reads its 64 packed bytes from shared
//                memory, expands each 2-bit code to a byte with one shift-and-mask per four
//                weights and writes 64 words into TMEM (tcgen05.st).
//   warps 12-19  two epilogue warpgroups, each taking half of the tile's tokens: tcgen05.ld of
//                the int32 accumulator, subtract the token's code sum (sum_k q*c =
//                sum_k u*c - sum_k c), scale by d_m * gamma, round to bf16 (lane pairs swap
//                values so each lane stores one bf16x2 word: conflict-free), stage in shared
//                memory and TMA-store.  Two TMEM accumulators let one tile's epilogue overlap
//                the next tile's main loop.
// Every wait is bounded: after ~1 s a role records BITNET_ERR_TIMEOUT and stops; in-flight TMA
// loads and MMAs are drained before TMEM is released.  No cluster multicast is used.
#include "common.cuh"
#include "kernels.h"

#include <cudaTypedefs.h>

namespace bitnet {
namespace tc {

constexpr int BW = 128;    // output features per tile (MMA M)
constexpr int BT = 128;    // tokens per tile (MMA N)
constexpr int BKS = 256;   // K per stage
constexpr int BKH = 128;   // K per swizzled half-stage (one 128-byte row of int8 codes)
constexpr int UMMA_K = 32;
constexpr int MMAS = BKS / UMMA_K;  // 8 per stage
constexpr int STAGES = 4;           // stages in flight: code tile in smem + A slot in TMEM each
constexpr int W_STAGES = 3;         // packed-weight tiles in flight
constexpr int SPW = 2;              // K stages per packed-weight tile [128 rows x 128 B]
constexpr int ACC_BUFS = 2;
constexpr int TMEM_COLS = 512;
constexpr int A_COLS = BKS / 4;        // 64 TMEM columns per A stage
constexpr int A_COL0 = ACC_BUFS * BT;  // A stages live after the accumulators
constexpr int HALF_BYTES = BT * BKH;   // 16 KB
constexpr int B_STAGE_BYTES = 2 * HALF_BYTES;
constexpr int W_STAGE_BYTES = BW * 128;
constexpr int EPI_WARPS = 8;
constexpr int EPI_BUF_BYTES = 32 * 32 * 2;  // one bf16 32 x 32 box (int32 boxes use two)
constexpr uint32_t IDESC = idesc_i8_u8s8(BW, BT);
static_assert(A_COL0 + STAGES * A_COLS <= TMEM_COLS, "TMEM budget");
static_assert(STAGES % 2 == 0, "two producer groups take alternate stages");

constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_B4 = 2, WARP_A0 = 4, WARP_EPI = 12;
constexpr int NUM_THREADS = 20 * 32;

struct __align__(8) Barriers {
    uint64_t full[STAGES];   // stage s holds its code tile and its A slot
    uint64_t empty[STAGES];  // the MMAs of stage s have completed
    uint64_t full_w[W_STAGES];
    uint64_t empty_w[W_STAGES];
    uint64_t acc_full[ACC_BUFS];
    uint64_t acc_empty[ACC_BUFS];
    uint64_t done;
    uint32_t tmem_base;
};

constexpr size_t OFF_B = 0;
constexpr size_t OFF_W = OFF_B + (size_t)STAGES * B_STAGE_BYTES;
constexpr size_t OFF_EPI = OFF_W + (size_t)W_STAGES * W_STAGE_BYTES;
constexpr size_t OFF_SCALE = OFF_EPI + EPI_WARPS * 2 * EPI_BUF_BYTES;  // [8 warps][BT/2] floats
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
                           const __grid_constant__ CUtensorMap tmap_out,
                           const uint8_t *__restrict__ codes4, const float *__restrict__ scales,
                           const int32_t *__restrict__ rowsum, const float *__restrict__ gamma_ptr,
                           int M, int N, int K, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sb = smem + OFF_B;
    uint8_t *sw = smem + OFF_W;
    uint8_t *sepi = smem + OFF_EPI;
    float *s_scale = reinterpret_cast<float *>(smem + OFF_SCALE);
    int32_t *s_rsum = reinterpret_cast<int32_t *>(smem + OFF_RSUM);
    Barriers *bar = reinterpret_cast<Barriers *>(smem + OFF_BAR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_wtiles = (N + BW - 1) / BW;
    const int n_ttiles = (M + BT - 1) / BT;
    const int num_tiles = n_wtiles * n_ttiles;
    const int KS = (K + BKS - 1) / BKS;    // stages per tile (a last half stage reads zeros)
    const int WPT = (KS + SPW - 1) / SPW;  // weight tiles per output tile
    const int my_tiles =
        (int)blockIdx.x < num_tiles ? (num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_tiles * KS;  // (tile, stage) iterations of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // codes: the TMA arrival (INT8) or the two INT4 producer warps; A: four warps
            mbar_init(&bar->full[s], (BITS == 8 ? 1 : 2) + 4);
            mbar_init(&bar->empty[s], 1);
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
        prefetch_tensormap(&tmap_out);
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
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t issued_b = 0, ph_b = 0, issued_w = 0, ph_w = 0;  // for the final drain
            int t = 0, ks = 0;
            for (int it = 0; it < total; ++it) {
                const int tile = blockIdx.x + t * gridDim.x;
                if (ks % SPW == 0) {
                    const int wseq = t * WPT + ks / SPW;
                    const int s_w = wseq % W_STAGES;
                    const uint32_t p_w = (uint32_t)(wseq / W_STAGES) & 1;
                    if (!mbar_wait(&bar->empty_w[s_w], p_w ^ 1, status)) break;
                    mbar_arrive_expect_tx(&bar->full_w[s_w], W_STAGE_BYTES);
                    tma_load_2d(sw + (size_t)s_w * W_STAGE_BYTES, &tmap_w, ks * (BKS / 4),
                                (tile % n_wtiles) * BW, &bar->full_w[s_w]);
                    issued_w |= 1u << s_w;
                    ph_w = (ph_w & ~(1u << s_w)) | (p_w << s_w);
                }
                if constexpr (BITS == 8) {
                    const int s = it % STAGES;
                    const uint32_t p = (uint32_t)(it / STAGES) & 1;
                    if (!mbar_wait(&bar->empty[s], p ^ 1, status)) break;
                    mbar_arrive_expect_tx(&bar->full[s], B_STAGE_BYTES);
                    uint8_t *dst = sb + (size_t)s * B_STAGE_BYTES;
                    const int y = (tile / n_wtiles) * BT;
                    tma_load_2d(dst, &tmap_codes, ks * BKS, y, &bar->full[s]);
                    tma_load_2d(dst + HALF_BYTES, &tmap_codes, ks * BKS + BKH, y, &bar->full[s]);
                    issued_b |= 1u << s;
                    ph_b = (ph_b & ~(1u << s)) | (p << s);
                }
                if (++ks == KS) { ks = 0; ++t; }
            }
            // no copy may still be writing shared memory when the CTA exits
            for (int i = 0; i < W_STAGES; ++i)
                if (issued_w & (1u << i)) mbar_wait(&bar->full_w[i], (ph_w >> i) & 1, status);
            for (int i = 0; i < STAGES; ++i)
                if (issued_b & (1u << i)) mbar_wait(&bar->full[i], (ph_b >> i) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sb_addr = smem_addr(sb);
            bool ok = true;
            bool next_full = total > 0 && mbar_test_wait(&bar->full[0], 0);
            int t = 0, ks = 0;
            for (int it = 0; it < total; ++it) {
                const int ab = t & 1;
                const int s = it % STAGES;
                if (ks == 0 &&
                    !mbar_wait(&bar->acc_empty[ab], ((uint32_t)(t >> 1) & 1) ^ 1, status)) {
                    ok = false;
                    break;
                }
                if (!next_full && !mbar_wait(&bar->full[s], (uint32_t)(it / STAGES) & 1, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // ask now whether the next stage is ready: the answer is needed only after this
                // stage's MMAs have been issued, so its latency is hidden behind them
                if (it + 1 < total)
                    next_full = mbar_test_wait(&bar->full[(it + 1) % STAGES],
                                               (uint32_t)((it + 1) / STAGES) & 1);
                const uint32_t d_tmem = tmem + ab * BT;
                const uint32_t a_tmem = tmem + A_COL0 + s * A_COLS;
                const uint64_t bdesc0 = smem_desc_kmajor_sw128(sb_addr + (uint32_t)s * B_STAGE_BYTES);
                const uint64_t bdesc1 = bdesc0 + (uint64_t)(HALF_BYTES >> 4);
#pragma unroll
                for (int kk = 0; kk < MMAS; ++kk) {
                    const uint64_t bd = (kk < 4 ? bdesc0 : bdesc1) + (uint64_t)((kk & 3) * UMMA_K / 16);
                    mma_i8_ts(d_tmem, a_tmem + kk * (UMMA_K / 4), bd, IDESC,
                              (ks | kk) != 0 ? 1u : 0u);
                }
                mma_commit(&bar->empty[s]);
                // the A stages of this weight tile are in TMEM (full[s] observed): refill it
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
    } else if (warp >= WARP_A0 && warp < WARP_A0 + 8) {
        // ------------------------------------------------------------------ A producers
        const int grp = (warp - WARP_A0) >> 2;  // takes iterations it = grp, grp + 2, ...
        const int wq = warp & 3;                // TMEM lanes 32*wq .. 32*wq+31
        const int rr = wq * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        for (int it = grp; it < total; it += 2) {
            const int t = it / KS, ks = it - t * KS;
            const int wseq = t * WPT + ks / SPW;
            const int s_w = wseq % W_STAGES, s = it % STAGES;
            if (!warp_wait(&bar->full_w[s_w], (uint32_t)(wseq / W_STAGES) & 1, status, lane)) break;
            // row rr of the weight tile: 2 stages x 64 B; 16-byte chunk c sits at c ^ (rr & 7)
            const uint8_t *wrow = sw + (size_t)s_w * W_STAGE_BYTES + rr * 128;
            const int c0 = 4 * (ks % SPW);
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = *reinterpret_cast<const uint4 *>(wrow + (((c0 + c) ^ (rr & 7)) << 4));
                w[4 * c] = v.x;
                w[4 * c + 1] = v.y;
                w[4 * c + 2] = v.z;
                w[4 * c + 3] = v.w;
            }
            if (!warp_wait(&bar->empty[s], ((uint32_t)(it / STAGES) & 1) ^ 1, status, lane)) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t out[32];
#pragma unroll
                for (int g = 0; g < 8; ++g)
#pragma unroll
                    for (int p = 0; p < 4; ++p)
                        out[4 * g + p] = (w[8 * h + g] >> (2 * p)) & 0x03030303u;
                tmem_st_32x32b_x32(t_lane + A_COL0 + s * A_COLS + h * 32, out);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->full[s]);
        }
    } else if (warp >= WARP_EPI && warp < WARP_EPI + EPI_WARPS) {
        // ------------------------------------------------------------------ epilogue
        const int wq = warp & 3;                  // TMEM lanes 32*wq .. 32*wq+31
        const int half = (warp - WARP_EPI) >> 2;  // tokens 64*half .. 64*half+63 of the tile
        const int ew = warp - WARP_EPI;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        float *w_scale = s_scale + ew * (BT / 2);  // this warp's copy: no cross-warp barrier
        int32_t *w_rsum = s_rsum + ew * (BT / 2);
        uint8_t *w_stage = sepi + (size_t)ew * 2 * EPI_BUF_BYTES;  // 2 bf16 boxes / 1 int32 box
        const float gamma = *gamma_ptr;
        const bool odd = lane & 1;
        int buf = 0;
        for (int t = 0; t < my_tiles; ++t) {
            const int tile = blockIdx.x + t * gridDim.x;
            const int nw = tile % n_wtiles;
            const int mt = tile / n_wtiles;
            const int ab = t & 1;
            __syncwarp();  // the previous tile's scales are no longer read
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int ml = i * 32 + lane;
                const int64_t m = (int64_t)mt * BT + half * 64 + ml;
                w_scale[ml] = m < M ? scales[m] * gamma : 0.f;
                w_rsum[ml] = m < M ? rowsum[m] : 0;
            }
            if (!warp_wait(&bar->acc_full[ab], (uint32_t)(t >> 1) & 1, status, lane)) break;
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_lane + ab * BT + half * 64 + ch * 32, v);
                tmem_wait_ld();
                uint8_t *stage = w_stage + (OUT_I32 ? 0 : buf * EPI_BUF_BYTES);
                if (lane == 0) {
                    if (OUT_I32) bulk_wait_group_read<0>();  // the single buffer is free
                    else bulk_wait_group_read<1>();          // this buffer's previous store is done
                }
                __syncwarp();
                if constexpr (OUT_I32) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        reinterpret_cast<int32_t *>(stage)[i * 32 + lane] =
                            (int)v[i] - w_rsum[ch * 32 + i];
                } else {
                    // this lane holds column n = lane of rows i; lane pairs swap one value so
                    // the even lane stores row i (n, n+1) and the odd lane row i+1 (n-1, n)
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
                        *reinterpret_cast<__nv_bfloat162 *>(stage + (i + (odd ? 1 : 0)) * 64 +
                                                            (lane & ~1) * 2) = pr;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                // boxes that lie wholly outside Y (ragged last tiles) are not stored; partial
                // boxes are clipped by the tensor map
                const int x0 = nw * BW + wq * 32, y0 = mt * BT + half * 64 + ch * 32;
                if (lane == 0 && x0 < N && y0 < M) {
                    tma_store_2d(&tmap_out, stage, x0, y0);
                    bulk_commit_group();
                }
                buf ^= 1;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->acc_empty[ab]);
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    } else if (BITS == 4 && warp >= WARP_B4 && warp < WARP_B4 + 2) {
        // ------------------------------------------------------------------ INT4 B producer
        // warp w covers tokens 64w .. 64w+63 of the tile; for each half-stage and sub-step i,
        // lane l loads the 16-byte quarter (l % 4) of token 64w + 8i + l / 4: 8 tokens x 64 B
        // per instruction, fully used sectors.
        const int wq = warp - WARP_B4;
        const int q = lane & 3;
        int t = 0, ks = 0;
        for (int it = 0; it < total; ++it) {
            const int tile = blockIdx.x + t * gridDim.x;
            const int s = it % STAGES;
            if (!warp_wait(&bar->empty[s], ((uint32_t)(it / STAGES) & 1) ^ 1, status, lane))
                break;
            const int64_t mbase = (int64_t)(tile / n_wtiles) * BT + wq * 64 + (lane >> 2);
#pragma unroll 1
            for (int hs = 0; hs < 2; ++hs) {
                const int kbyte = (ks * BKS + hs * BKH) / 2 + q * 16;  // byte offset in the row
                const bool kin = kbyte < K / 2;
                uint4 raw[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int64_t m = mbase + 8 * i;
                    raw[i] = (m < M && kin) ? ldg_nc_v4(codes4 + m * (K / 2) + kbyte)
                                            : make_uint4(0, 0, 0, 0);
                }
                uint8_t *dst = sb + (size_t)s * B_STAGE_BYTES + hs * HALF_BYTES;
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
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->full[s]);
            if (++ks == KS) { ks = 0; ++t; }
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
                               const CUtensorMap &mo, int grid, cudaStream_t stream) {
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
        mc, mw, mo, reinterpret_cast<const uint8_t *>(a.codes), a.scales, a.rowsum, a.gamma,
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
    CUtensorMap mc, mw, mo;
    memset(&mc, 0, sizeof mc);
    memset(&mw, 0, sizeof mw);
    memset(&mo, 0, sizeof mo);
    if (a.act_bits == 8 &&
        encode_2d(encode_fn, &mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, (uint64_t)a.K,
                  (uint64_t)a.M, (uint64_t)a.K, BKH, BT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // packed weights: [N rows][K/4 bytes], one [128 x 128 B] box (two K stages) per tile
    if (encode_2d(encode_fn, &mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, (uint64_t)a.K / 4,
                  (uint64_t)a.N, (uint64_t)a.K / 4, 128, BW,
                  CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (a.Y) {
        if (encode_2d(encode_fn, &mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Y, (uint64_t)a.N,
                      (uint64_t)a.M, (uint64_t)a.N * 2, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        e = a.act_bits == 8 ? launch_tc_t<8, false>(a, mc, mw, mo, grid, stream)
                            : launch_tc_t<4, false>(a, mc, mw, mo, grid, stream);
        if (e != cudaSuccess) return e;
    }
    if (a.acc) {
        if (encode_2d(encode_fn, &mo, CU_TENSOR_MAP_DATA_TYPE_INT32, a.acc, (uint64_t)a.N,
                      (uint64_t)a.M, (uint64_t)a.N * 4, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        e = a.act_bits == 8 ? launch_tc_t<8, true>(a, mc, mw, mo, grid, stream)
                            : launch_tc_t<4, true>(a, mc, mw, mo, grid, stream);
    }
    return e;
}

}  // namespace bitnet
