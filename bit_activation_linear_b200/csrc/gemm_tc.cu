// gemm_tc.cu -- step 4 for many tokens (prefill): the ternary x integer product on the
// 5th-generation tensor cores (tcgen05, kind::i8), accumulating in int32 in tensor memory,
// with the rescale to bf16 fused into the epilogue.
//
// 2B4T article, section 一.2 (W1.58A8 BitLinear; the product needs only additions and
// subtractions) and section 三.3 (GPU kernel: pack-store-load-unpack-compute).  On sm_100a the
// cheapest exact "add/subtract" is the int8 tensor-core MMA: the 2-bit weights are unpacked
// on chip, never in HBM.
//
// A CTA pair (a cluster of two CTAs on neighbouring SMs) computes a tile of 256 tokens x 256
// output features with tcgen05.mma.cta_group::2: D[256 x 256] += A[256 x 32] * B[256 x 32]^T,
// A = activation codes (signed), B = weight offset codes u = q + 1 in {0, 1, 2} (unsigned).
// CTA r of the pair holds tokens 128r .. 128r+127 of A, features 128r .. 128r+127 of B and
// accumulator rows (tokens) 128r .. 128r+127 for all 256 features.  Against one CTA computing a
// 128 x 256 tile alone, each SM moves half the activation bytes from L2 and through shared
// memory per multiply-add: measured on B200, a lone CTA spent ~1050 cycles per 128-deep K stage
// on 512 cycles of tensor work, its operand traffic (TMA and unpack writes plus tensor-core reads)
// saturating shared memory and the L2->SM path.
//
// K runs in stages of 128 (four K=32 MMAs, 512 tensor cycles).  The two 256-column int32
// accumulators fill the 512 TMEM columns, so a tile's epilogue overlaps the next tile's MMAs.
// Warp roles, in both CTAs unless noted:
//   warp 0       code-tile TMA (INT8): [128 tokens x 128 B] with the 128-byte swizzle (the UMMA
//                K-major layout); the pair form of the copy completes on the even CTA's barrier,
//                which expects both halves.
//   warp 2       packed-weight TMA: [128 features x 64 B] (two K stages) into a local ring.
//   warp 1       even CTA: MMA issuer (one thread).  Both CTAs: tensor-memory allocation.
//   warps 4-11   weight unpack (two groups taking alternate stages; one group for INT4): thread i
//                expands the 32 packed bytes of feature i for the stage (one shift-and-mask per
//                four weights) into 128 bytes of the swizzled layout, then signals the even CTA.
//   warps 8-11   (INT4 only) code producers: 16-byte loads of nibble codes, sign-extended to
//                int8 in registers, stored in the swizzled layout.
//   warps 12-19  epilogue: thread = token row; tcgen05.ld of 32 features, subtract the token's
//                code sum (sum_k c*q = sum_k c*u - sum_k c), scale by d_m * gamma, round to bf16,
//                64 contiguous bytes per thread and chunk.
// Commits multicast to both CTAs; every wait is bounded: after ~1 s a role records
// BITNET_ERR_TIMEOUT and stops; in-flight copies and MMAs are drained and both CTAs meet at a
// cluster barrier before tensor memory is released.  No TMA multicast is used.
#include "common.cuh"
#include "kernels.h"

#include <cudaTypedefs.h>

namespace bitnet {
namespace tc {

constexpr int BM = 256;            // tokens per pair tile (MMA M)
constexpr int BN = 256;            // output features per pair tile (MMA N)
constexpr int HM = BM / 2;         // tokens held by one CTA
constexpr int HN = BN / 2;         // features held by one CTA
constexpr int BK = 128;            // K per stage: one 128-byte swizzled row of int8
constexpr int UMMA_K = 32;
constexpr int MMAS = BK / UMMA_K;  // 4 per stage
constexpr int A_STAGES = 6;        // code tiles in flight
constexpr int B_STAGES = 4;        // unpacked weight tiles
constexpr int W_STAGES = 4;        // packed-weight tiles in flight
constexpr int SPW = 2;             // K stages per packed-weight tile [128 features x 64 B]
constexpr int ACC_BUFS = 2;
constexpr int TMEM_COLS = 512;
constexpr int A_STAGE_BYTES = HM * BK;               // 16 KB
constexpr int B_STAGE_BYTES = HN * BK;               // 16 KB
constexpr int W_STAGE_BYTES = HN * SPW * BK / 4;     // 8 KB
constexpr int EPI_WARPS = 8;
constexpr uint32_t IDESC = idesc_i8_s8u8(BM, BN);
static_assert(ACC_BUFS * BN <= TMEM_COLS, "TMEM budget");

constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_WTMA = 2, WARP_B0 = 4, WARP_A4 = 8, WARP_EPI = 12;
constexpr int NUM_THREADS = 20 * 32;

struct __align__(8) Barriers {
    uint64_t full_a[A_STAGES];     // even CTA: both halves of the code tile are in place
    uint64_t empty_a[A_STAGES];    // both: the MMAs that read the stage have completed
    uint64_t full_b[B_STAGES];     // even CTA: the unpack warps of both CTAs wrote the stage
    uint64_t empty_b[B_STAGES];    // both
    uint64_t full_w[W_STAGES];     // local packed-weight ring
    uint64_t empty_w[W_STAGES];    // local; arrived by the MMA thread of the even CTA
    uint64_t acc_full[ACC_BUFS];   // both
    uint64_t acc_empty[ACC_BUFS];  // even CTA: the epilogue warps of both CTAs
    uint64_t done;                 // both: every MMA has completed
    uint32_t tmem_base;
};

// identical offsets in both CTAs: the pair MMA addresses the peer's operands by the even CTA's
// shared-memory offsets
constexpr size_t OFF_A = 0;
constexpr size_t OFF_B = OFF_A + (size_t)A_STAGES * A_STAGE_BYTES;
constexpr size_t OFF_W = OFF_B + (size_t)B_STAGES * B_STAGE_BYTES;
constexpr size_t OFF_BAR = OFF_W + (size_t)W_STAGES * W_STAGE_BYTES;
constexpr size_t SMEM_BYTES = OFF_BAR + sizeof(Barriers) + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast,
// __syncwarp orders the other lanes after the acquire (needed before warp-collective tcgen05 ops).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, status);
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

template <int BITS, bool OUT_I32>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
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
    Barriers *bar = reinterpret_cast<Barriers *>(smem + OFF_BAR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int n_ftiles = (N + BN - 1) / BN;
    const int n_ttiles = (M + BM - 1) / BM;
    const int num_tiles = n_ftiles * n_ttiles;
    const int KS = K / BK;                 // stages per tile
    const int WPT = (KS + SPW - 1) / SPW;  // packed-weight tiles per output tile
    constexpr int B_GROUPS = BITS == 8 ? 2 : 1;
    const int my_tiles = pair < num_tiles ? (num_tiles - 1 - pair) / npairs + 1 : 0;
    const int total = my_tiles * KS;  // (tile, stage) iterations of this pair

    if (threadIdx.x == 0) {
        for (int s = 0; s < A_STAGES; ++s) {
            // INT8: the even CTA's expect-tx arrival; INT4: the code warps of both CTAs
            mbar_init(&bar->full_a[s], BITS == 8 ? 1 : 8);
            mbar_init(&bar->empty_a[s], 1);
        }
        for (int s = 0; s < B_STAGES; ++s) {
            mbar_init(&bar->full_b[s], 8);
            mbar_init(&bar->empty_b[s], 1);
        }
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&bar->full_w[s], 1);
            mbar_init(&bar->empty_w[s], 1);
        }
        for (int s = 0; s < ACC_BUFS; ++s) {
            mbar_init(&bar->acc_full[s], 1);
            mbar_init(&bar->acc_empty[s], 2 * EPI_WARPS);
        }
        mbar_init(&bar->done, 1);
        fence_mbar_init();
    }
    if (warp == WARP_TMA && lane == 0) {
        if (BITS == 8) prefetch_tensormap(&tmap_codes);
        prefetch_tensormap(&tmap_w);
    }
    if (warp == WARP_MMA) {
        tmem_alloc_pair(&bar->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised and the tensor memory is allocated
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == WARP_TMA) {
        // ------------------------------------------------------------------ code-tile TMA
        if (BITS == 8 && lane == 0) {
            uint32_t issued = 0, ph = 0;  // for the final drain
            int t = 0, ks = 0;
            for (int it = 0; it < total; ++it) {
                const int tile = pair + t * npairs;
                const int s = it % A_STAGES;
                const uint32_t p = (uint32_t)(it / A_STAGES) & 1;
                if (!mbar_wait(&bar->empty_a[s], p ^ 1, status)) break;
                if (leader) mbar_arrive_expect_tx(&bar->full_a[s], 2 * A_STAGE_BYTES);
                tma_load_2d_pair(sa + (size_t)s * A_STAGE_BYTES, &tmap_codes, ks * BK,
                                 (tile / n_ftiles) * BM + (int)rank * HM,
                                 mapa_shared(smem_addr(&bar->full_a[s]), 0));
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
                if (++ks == KS) { ks = 0; ++t; }
            }
            // no copy may still be writing shared memory when the CTA exits: the even CTA sees
            // its barrier complete, the odd CTA sees the stage consumed (or gives up)
            for (int i = 0; i < A_STAGES; ++i)
                if (issued & (1u << i))
                    mbar_wait(leader ? &bar->full_a[i] : &bar->empty_a[i], (ph >> i) & 1,
                                 status);
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
                const int tile_w = pair + (w / WPT) * npairs;
                mbar_arrive_expect_tx(&bar->full_w[s_w], W_STAGE_BYTES);
                tma_load_2d(sw + (size_t)s_w * W_STAGE_BYTES, &tmap_w, (w % WPT) * SPW * (BK / 4),
                            (tile_w % n_ftiles) * BN + (int)rank * HN, &bar->full_w[s_w]);
                issued |= 1u << s_w;
                ph = (ph & ~(1u << s_w)) | (p_w << s_w);
            }
            for (int i = 0; i < W_STAGES; ++i)
                if (issued & (1u << i)) mbar_wait(&bar->full_w[i], (ph >> i) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        if (leader && lane == 0) {
            const uint32_t sa_addr = smem_addr(sa);
            const uint32_t sb_addr = smem_addr(sb);
            bool next_a = total > 0 && mbar_test_wait(&bar->full_a[0], 0);
            bool next_b = total > 0 && mbar_test_wait(&bar->full_b[0], 0);
            int t = 0, ks = 0;
            for (int it = 0; it < total; ++it) {
                const int ab = t & 1;
                const int sa_i = it % A_STAGES, sb_i = it % B_STAGES;
                if (ks == 0 &&
                    !mbar_wait(&bar->acc_empty[ab], ((uint32_t)(t >> 1) & 1) ^ 1, status))
                    break;
                if ((!next_a &&
                     !mbar_wait(&bar->full_a[sa_i], (uint32_t)(it / A_STAGES) & 1, status)) ||
                    (!next_b &&
                     !mbar_wait(&bar->full_b[sb_i], (uint32_t)(it / B_STAGES) & 1, status)))
                    break;
                tc_fence_after();
                // ask now whether the next stage is ready: the answers are needed only after this
                // stage's MMAs have been issued, so their latency is hidden behind them
                if (it + 1 < total) {
                    next_a = mbar_test_wait(&bar->full_a[(it + 1) % A_STAGES],
                                               (uint32_t)((it + 1) / A_STAGES) & 1);
                    next_b = mbar_test_wait(&bar->full_b[(it + 1) % B_STAGES],
                                               (uint32_t)((it + 1) / B_STAGES) & 1);
                }
                const uint32_t d_tmem = tmem + ab * BN;
                const uint64_t adesc =
                    smem_desc_kmajor_sw128(sa_addr + (uint32_t)sa_i * A_STAGE_BYTES);
                const uint64_t bdesc =
                    smem_desc_kmajor_sw128(sb_addr + (uint32_t)sb_i * B_STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < MMAS; ++kk)
                    mma_i8_ss_pair(d_tmem, adesc + (uint64_t)(kk * UMMA_K / 16),
                                   bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                                   (ks | kk) != 0 ? 1u : 0u);
                mma_commit_pair(&bar->empty_a[sa_i], 3);
                mma_commit_pair(&bar->empty_b[sb_i], 3);
                // the unpack warps of both CTAs are done with this packed-weight tile (full_b
                // observed for its last stage): both may refill it
                if (ks % SPW == SPW - 1 || ks == KS - 1) {
                    uint64_t *ew = &bar->empty_w[(t * WPT + ks / SPW) % W_STAGES];
                    mbar_arrive(ew);
                    mbar_arrive_cluster(mapa_shared(smem_addr(ew), 1));
                }
                if (ks == KS - 1) mma_commit_pair(&bar->acc_full[ab], 3);
                if (++ks == KS) { ks = 0; ++t; }
            }
            // every MMA issued above has finished before either CTA releases tensor memory
            mma_commit_pair(&bar->done, 3);
        }
        if (lane == 0) mbar_wait(&bar->done, 0, status);
        __syncwarp();
    } else if (warp >= WARP_B0 && warp < WARP_B0 + 4 * B_GROUPS) {
        // ------------------------------------------------------------------ weight unpack
        const int grp = (warp - WARP_B0) >> 2;  // takes iterations it = grp (mod B_GROUPS)
        const int rr = (warp & 3) * 32 + lane;  // row of this CTA's B half = feature
        for (int it = grp; it < total; it += B_GROUPS) {
            const int t = it / KS, ks = it - t * KS;
            const int wseq = t * WPT + ks / SPW;
            const int s_w = wseq % W_STAGES, s = it % B_STAGES;
            if (!warp_wait(&bar->full_w[s_w], (uint32_t)(wseq / W_STAGES) & 1, status, lane)) break;
            // row rr of the weight tile: SPW stages x 32 B
            const uint4 *wsrc = reinterpret_cast<const uint4 *>(
                sw + (size_t)s_w * W_STAGE_BYTES + rr * (SPW * BK / 4) + (ks % SPW) * (BK / 4));
            const uint4 p0 = wsrc[0], p1 = wsrc[1];
            const uint32_t w[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
            if (!warp_wait(&bar->empty_b[s], ((uint32_t)(it / B_STAGES) & 1) ^ 1, status, lane))
                break;
            // packed word g holds k = 16g .. 16g+15; (w >> 2p) & 0x03030303 is k = 16g+4p .. +3,
            // so word g becomes the 16-byte chunk g of the row, stored at chunk g ^ (rr & 7)
            uint8_t *brow = sb + (size_t)s * B_STAGE_BYTES + rr * 128;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                uint4 o;
                o.x = w[g] & 0x03030303u;
                o.y = (w[g] >> 2) & 0x03030303u;
                o.z = (w[g] >> 4) & 0x03030303u;
                o.w = (w[g] >> 6) & 0x03030303u;
                *reinterpret_cast<uint4 *>(brow + ((g ^ (rr & 7)) << 4)) = o;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->full_b[s]), 0));
        }
    } else if (warp >= WARP_EPI && warp < WARP_EPI + EPI_WARPS) {
        // ------------------------------------------------------------------ epilogue
        const int wq = warp & 3;                   // TMEM lanes 32*wq .. 32*wq+31 = tokens
        const int half = (warp - WARP_EPI) >> 2;   // features 128*half .. 128*half+127
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        const float gamma = *gamma_ptr;
        for (int t = 0; t < my_tiles; ++t) {
            const int tile = pair + t * npairs;
            const int nf = tile % n_ftiles;
            const int mt = tile / n_ftiles;
            const int ab = t & 1;
            const int64_t m = (int64_t)mt * BM + (int)rank * HM + wq * 32 + lane;
            const bool m_ok = m < M;
            const float sc = m_ok ? scales[m] * gamma : 0.f;
            const int rs = m_ok ? rowsum[m] : 0;
            if (!warp_wait(&bar->acc_full[ab], (uint32_t)(t >> 1) & 1, status, lane)) break;
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < HN / 32; ++ch) {
                const int col = half * HN + ch * 32;
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_lane + ab * BN + col, v);
                tmem_wait_ld();
                const int n0 = nf * BN + col;
                if constexpr (OUT_I32) {
                    int32_t *row = reinterpret_cast<int32_t *>(Yout) + m * N;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int n = n0 + 4 * j;
                        if (m_ok && n < N)
                            *reinterpret_cast<int4 *>(row + n) =
                                make_int4((int)v[4 * j] - rs, (int)v[4 * j + 1] - rs,
                                          (int)v[4 * j + 2] - rs, (int)v[4 * j + 3] - rs);
                    }
                } else {
                    __nv_bfloat16 *row = reinterpret_cast<__nv_bfloat16 *>(Yout) + m * N;
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float y0 = (float)((int)v[2 * i] - rs) * sc;
                        const float y1 = (float)((int)v[2 * i + 1] - rs) * sc;
                        const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
                        pk[i] = *reinterpret_cast<const uint32_t *>(&h);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int n = n0 + 8 * j;
                        if (m_ok && n < N)
                            *reinterpret_cast<uint4 *>(row + n) =
                                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->acc_empty[ab]), 0));
        }
    } else if (BITS == 4 && warp >= WARP_A4 && warp < WARP_A4 + 4) {
        // ------------------------------------------------------------------ INT4 code producer
        // warp w covers tokens 32w .. 32w+31 of this CTA's half; in sub-step i, lane l loads the
        // 16-byte quarter (l % 4) of token 32w + 8i + l / 4: 8 tokens x 64 B per instruction,
        // fully used sectors.  The next stage's bytes are loaded before this one is stored.
        const int wq = warp - WARP_A4;
        const int q = lane & 3;
        uint4 nxt[4];
        auto fetch = [&](int it2) {
            const int t2 = it2 / KS, ks2 = it2 - t2 * KS;
            const int tile2 = pair + t2 * npairs;
            const int64_t mbase =
                (int64_t)(tile2 / n_ftiles) * BM + (int)rank * HM + wq * 32 + (lane >> 2);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t m = mbase + 8 * i;
                nxt[i] = (it2 < total && m < M)
                             ? ldg_nc_v4(codes4 + m * (K / 2) + ks2 * (BK / 2) + q * 16)
                             : make_uint4(0, 0, 0, 0);
            }
        };
        fetch(0);
        for (int it = 0; it < total; ++it) {
            const int s = it % A_STAGES;
            uint4 raw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) raw[i] = nxt[i];
            fetch(it + 1);
            if (!warp_wait(&bar->empty_a[s], ((uint32_t)(it / A_STAGES) & 1) ^ 1, status, lane))
                break;
            uint8_t *dst = sa + (size_t)s * A_STAGE_BYTES;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = wq * 32 + 8 * i + (lane >> 2);
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
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->full_a[s]), 0));
        }
    }

    // neither CTA leaves while the other may still signal its barriers or read its operands
    __syncwarp();
    tc_fence_before();
    cluster_sync();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

// Co-resident pairs per device (a persistent grid of one pair per two SMs where the GPU's
// layout allows it), looked up once per device and kernel instance.
template <int BITS, bool OUT_I32>
static int max_pairs(int num_sms) {
    static int cache[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_sms & ~1), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, ternary_gemm_tc_kernel<BITS, OUT_I32>, &cfg) !=
            cudaSuccess ||
        clusters < 1) {
        (void)cudaGetLastError();
        clusters = num_sms / 2;
    }
    if (dev >= 0 && dev < 64) cache[dev] = clusters;
    return clusters;
}

template <int BITS, bool OUT_I32>
static cudaError_t launch_tc_t(const GemmArgs &a, const CUtensorMap &mc, const CUtensorMap &mw,
                               void *out, int64_t tiles, int num_sms, cudaStream_t stream) {
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
    const int pairs_max = max_pairs<BITS, OUT_I32>(num_sms);
    const int pairs = (int)(tiles < pairs_max ? tiles : pairs_max);
    kern<<<2 * pairs, NUM_THREADS, SMEM_BYTES, stream>>>(
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
    const int64_t tiles = ((a.N + BN - 1) / BN) * ((a.M + BM - 1) / BM);
    CUtensorMap mc, mw;
    memset(&mc, 0, sizeof mc);
    memset(&mw, 0, sizeof mw);
    // codes: [M rows][K bytes], one [128 tokens x 128 B] swizzled box per CTA and stage
    if (a.act_bits == 8 &&
        encode_2d(encode_fn, &mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, (uint64_t)a.K,
                  (uint64_t)a.M, (uint64_t)a.K, BK, HM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // packed weights: [N rows][K/4 bytes], one [128 features x 64 B] box (two K stages)
    if (encode_2d(encode_fn, &mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, (uint64_t)a.K / 4,
                  (uint64_t)a.N, (uint64_t)a.K / 4, SPW * BK / 4, HN,
                  CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (a.Y) {
        e = a.act_bits == 8 ? launch_tc_t<8, false>(a, mc, mw, a.Y, tiles, num_sms, stream)
                            : launch_tc_t<4, false>(a, mc, mw, a.Y, tiles, num_sms, stream);
        if (e != cudaSuccess) return e;
    }
    if (a.acc) {
        e = a.act_bits == 8 ? launch_tc_t<8, true>(a, mc, mw, a.acc, tiles, num_sms, stream)
                            : launch_tc_t<4, true>(a, mc, mw, a.acc, tiles, num_sms, stream);
    }
    return e;
}

}  // namespace bitnet
