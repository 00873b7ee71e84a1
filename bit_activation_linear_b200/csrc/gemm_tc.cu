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
// accumulator rows (tokens) 128r .. 128r+127 for all 256 features, so each SM moves half the
// activation bytes per multiply-add that a lone CTA with a 128 x 256 tile would.
//
// K runs in stages of 256: eight K=32 MMAs (1024 tensor cycles) per readiness test and commit.
// Measured on B200, issuing one MMA costs ~45-65 cycles and a readiness test ~100, so with
// 128-deep stages the issuing thread itself used ~900 of every 512 tensor cycles.  A stage
// holds each operand as two 128-deep sub-tiles [128 rows x 128 B] in the 128-byte-swizzled
// K-major layout.  The two 256-column int32 accumulators fill the 512 TMEM columns, so a tile's
// epilogue overlaps the next tile's MMAs.
// Warp roles, in both CTAs unless noted (warps 5, 9, 13 stay idle so that the scheduler
// partition of the MMA warp hosts only it and two epilogue warps):
//   warp 0       code TMA.  INT8: two [128 tokens x 128 B] boxes per stage; the pair form of the
//                copy completes on the even CTA's stage barrier, which expects all four boxes.
//                INT4: one [128 tokens x 128 B] box of packed nibbles into the second sub-tile.
//   warp 2       packed-weight TMA: [128 features x 64 B] (one stage), 64-byte swizzle, into a
//                local ring.
//   warp 1       even CTA: MMA issuer (one thread).  Both CTAs: tensor-memory allocation.
//   unpack warps (two groups of four taking alternate stages; one group for INT4): thread i
//                expands the 64 packed bytes of feature i for the stage (one shift-and-mask per
//                four weights) into 256 bytes of the swizzled layout, then signals the even CTA
//                and releases the packed-weight slot.
//   code warps   (INT4 only) thread = token row sign-extends its 256 packed codes in place to
//                int8 in both sub-tiles.
//   warps 16-23  epilogue: thread = token row; tcgen05.ld of 32 features, subtract the token's
//                code sum (sum_k c*q = sum_k c*u - sum_k c), scale by d_m * gamma, round to bf16;
//                each warp stages [32 tokens x 16 features] boxes in shared memory and writes
//                them with bulk tensor stores.  (Direct stores of one row per thread touch 32
//                lines per instruction; on B200 they held up the unpack warps' shared-memory
//                stores for ~6000 cycles per tile.)
// Work: a persistent grid of pairs walks the output tiles, each in one pass over K.  (Products of
// a few tokens, where the tiles would be mostly empty, take gemm_skinny.cu instead.)
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
constexpr int BK = 256;            // K per stage
constexpr int SUBK = 128;          // K per sub-tile: one 128-byte swizzled row of int8
constexpr int UMMA_K = 32;
constexpr int MMAS = BK / UMMA_K;  // 8 per stage
constexpr int STAGES = 3;          // operand stages in flight
constexpr int W_STAGES = 3;        // packed-weight tiles in flight (one per stage)
constexpr int ACC_BUFS = 2;
constexpr int TMEM_COLS = 512;
constexpr int SUB_BYTES = 128 * SUBK;                // 16 KB: [128 rows x 128 B]
constexpr int A_STAGE_BYTES = 2 * SUB_BYTES;         // 32 KB of codes per CTA
constexpr int B_STAGE_BYTES = 2 * SUB_BYTES;         // 32 KB of unpacked weights per CTA
constexpr int W_STAGE_BYTES = HN * BK / 4;           // 8 KB of packed weights per CTA
constexpr int EPI_WARPS = 8;
constexpr int Y_BOX_N = 16;                          // features per output box (32 B of bf16)
constexpr int Y_BOX_BYTES = 32 * Y_BOX_N * 2;        // [32 tokens x 16 features] = 1 KB
constexpr uint32_t IDESC = idesc_i8_s8u8(BM, BN);
static_assert(ACC_BUFS * BN <= TMEM_COLS, "TMEM budget");

constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_WTMA = 2, WARP_EPI = 16;

// What the epilogue writes: the int32 accumulators (parity entry), the rescaled bf16 output, or
// the rescaled output through an activation (squared ReLU; SwiGLU over interleaved gate/up
// features, half as many columns).
enum OutMode { OUT_ACC = 0, OUT_BF16 = 1, OUT_RELU2 = 2, OUT_SWIGLU = 3 };
constexpr int NUM_THREADS = 24 * 32;

// Unpack / code warps: eight warps outside the MMA warp's scheduler partition (warp % 4 == 1).
// Returns 0..7, or -1 for every other warp.
__device__ __forceinline__ int worker_index(int w) {
    switch (w) {
        case 4: return 0;
        case 6: return 1;
        case 7: return 2;
        case 8: return 3;
        case 10: return 4;
        case 11: return 5;
        case 12: return 6;
        case 14: return 7;
        default: return -1;
    }
}

struct __align__(8) Barriers {
    // even CTA: the stage's code tiles of both CTAs are in place (INT8: the TMA bytes and one
    // expect-tx arrival; INT4: the code warps of both CTAs) and the unpack warps of both CTAs
    // have written their weight halves
    uint64_t full[STAGES];
    uint64_t empty[STAGES];        // both: the MMAs that read the stage have completed
    uint64_t packed[STAGES];       // local, INT4: the packed codes of the stage have landed
    uint64_t full_w[W_STAGES];     // local packed-weight ring
    uint64_t empty_w[W_STAGES];    // local; arrived by this CTA's unpack warps
    uint64_t acc_full[ACC_BUFS];   // both
    uint64_t acc_empty[ACC_BUFS];  // even CTA: the epilogue warps of both CTAs
    uint64_t done;                 // both: every MMA has completed
    uint32_t tmem_base;
};

// identical offsets in both CTAs: the pair MMA addresses the peer's operands by the even CTA's
// shared-memory offsets
constexpr size_t OFF_A = 0;
constexpr size_t OFF_B = OFF_A + (size_t)STAGES * A_STAGE_BYTES;
constexpr size_t OFF_W = OFF_B + (size_t)STAGES * B_STAGE_BYTES;
constexpr size_t OFF_Y = OFF_W + (size_t)W_STAGES * W_STAGE_BYTES;  // per epilogue warp
constexpr size_t OFF_BAR = OFF_Y + (size_t)EPI_WARPS * Y_BOX_BYTES;
constexpr size_t SMEM_BYTES = OFF_BAR + sizeof(Barriers) + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast, __syncwarp orders the other
// lanes after the acquire (needed before warp-collective tcgen05 ops).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, status);
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

template <int BITS, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    ternary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                           const __grid_constant__ CUtensorMap tmap_w,
                           const __grid_constant__ CUtensorMap tmap_y,
                           void *__restrict__ Yout, const float *__restrict__ scales,
                           const int32_t *__restrict__ rowsum, const float *__restrict__ gamma_ptr,
                           int M, int N, int K, int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sa = smem + OFF_A;
    uint8_t *sb = smem + OFF_B;
    uint8_t *sw = smem + OFF_W;
    uint8_t *sy = smem + OFF_Y;
    Barriers *bar = reinterpret_cast<Barriers *>(smem + OFF_BAR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int wi = worker_index(warp);
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int n_ftiles = (N + BN - 1) / BN;
    const int n_ttiles = (M + BM - 1) / BM;
    const int num_tiles = n_ftiles * n_ttiles;
    const int KS = (K + BK - 1) / BK;  // stages per tile (the last one may be half: K % 256 = 128)
    constexpr int B_GROUPS = BITS == 8 ? 2 : 1;
    // Pair p takes tiles p, p + npairs, ...; a unit is one tile and all KS stages of its K axis.
    const int num_units = num_tiles;
    const int my_units = pair < num_units ? (num_units - 1 - pair) / npairs + 1 : 0;
    auto unit = [&](int t, int &tile, int &kb, int &ke) {
        tile = pair + t * npairs;
        kb = 0;
        ke = KS;
    };
    int total = 0;  // (unit, stage) iterations of this pair
    for (int t = 0; t < my_units; ++t) {
        int tile, kb, ke;
        unit(t, tile, kb, ke);
        total += ke - kb;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // 8 unpack-warp arrivals (4 per CTA), plus the even CTA's expect-tx arrival (INT8)
            // or 8 code-warp arrivals (INT4)
            mbar_init(&bar->full[s], BITS == 8 ? 9 : 16);
            mbar_init(&bar->empty[s], 1);
            mbar_init(&bar->packed[s], 1);
        }
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&bar->full_w[s], 1);
            mbar_init(&bar->empty_w[s], 4);  // the four unpack warps of the stage's group
        }
        for (int s = 0; s < ACC_BUFS; ++s) {
            mbar_init(&bar->acc_full[s], 1);
            mbar_init(&bar->acc_empty[s], 2 * EPI_WARPS);
        }
        mbar_init(&bar->done, 1);
        fence_mbar_init();
    }
    if (warp == WARP_TMA && lane == 0) {
        prefetch_tensormap(&tmap_codes);
        prefetch_tensormap(&tmap_w);
        if (MODE != OUT_ACC) prefetch_tensormap(&tmap_y);
    }
    if (warp == WARP_MMA) {
        tmem_alloc_pair(&bar->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers are initialised and the tensor memory is allocated
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    // everything above overlaps the tail of the kernel that produced the codes (programmatic
    // dependent launch); nothing is read from global memory before this point
    pdl_wait();

    if (warp == WARP_TMA) {
        // ------------------------------------------------------------------ code TMA
        if (lane == 0) {
            uint32_t issued = 0, ph = 0;  // for the final drain
            int t = 0, s = 0, tile = 0, kb = 0, ke = 0;
            if (my_units > 0) unit(0, tile, kb, ke);
            int ks = kb;
            uint32_t p = 0;
            for (int it = 0; it < total; ++it) {
                const int m0 = (tile / n_ftiles) * BM + (int)rank * HM;
                if (!mbar_wait(&bar->empty[s], p ^ 1, status)) break;
                uint8_t *dst = sa + (size_t)s * A_STAGE_BYTES;
                if constexpr (BITS == 8) {
                    if (leader) mbar_arrive_expect_tx(&bar->full[s], 4 * SUB_BYTES);
                    const uint32_t fb = mapa_shared(smem_addr(&bar->full[s]), 0);
                    tma_load_2d_pair(dst, &tmap_codes, ks * BK, m0, fb);
                    tma_load_2d_pair(dst + SUB_BYTES, &tmap_codes, ks * BK + SUBK, m0, fb);
                } else {
                    // packed nibbles of the stage (128 B per token) into the second sub-tile,
                    // widened in place by the code warps
                    mbar_arrive_expect_tx(&bar->packed[s], SUB_BYTES);
                    tma_load_2d(dst + SUB_BYTES, &tmap_codes, ks * (BK / 2), m0, &bar->packed[s]);
                }
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
                if (++ks == ke && ++t < my_units) {
                    unit(t, tile, kb, ke);
                    ks = kb;
                }
                if (++s == STAGES) { s = 0; p ^= 1; }
            }
            // no copy may still be writing shared memory when the CTA exits: each CTA waits
            // until the stages it loaded have been consumed (or gives up after the time limit)
            for (int i = 0; i < STAGES; ++i)
                if (issued & (1u << i)) mbar_wait(&bar->empty[i], (ph >> i) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_WTMA) {
        // ------------------------------------------------------------------ weight-tile TMA
        if (lane == 0) {
            uint32_t issued = 0, ph = 0;
            int t = 0, s_w = 0, tile = 0, kb = 0, ke = 0;
            if (my_units > 0) unit(0, tile, kb, ke);
            int ks = kb;
            uint32_t p_w = 0;
            for (int it = 0; it < total; ++it) {
                if (!mbar_wait(&bar->empty_w[s_w], p_w ^ 1, status)) break;
                mbar_arrive_expect_tx(&bar->full_w[s_w], W_STAGE_BYTES);
                tma_load_2d(sw + (size_t)s_w * W_STAGE_BYTES, &tmap_w, ks * (BK / 4),
                            (tile % n_ftiles) * BN + (int)rank * HN, &bar->full_w[s_w]);
                issued |= 1u << s_w;
                ph = (ph & ~(1u << s_w)) | (p_w << s_w);
                if (++ks == ke && ++t < my_units) {
                    unit(t, tile, kb, ke);
                    ks = kb;
                }
                if (++s_w == W_STAGES) { s_w = 0; p_w ^= 1; }
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
            bool next = total > 0 && mbar_test_wait(&bar->full[0], 0);
            int t = 0, s = 0, tile = 0, kb = 0, ke = 0;
            if (my_units > 0) unit(0, tile, kb, ke);
            int ks = kb;
            uint32_t p = 0;
            for (int it = 0; it < total; ++it) {
                const int ab = t & 1;
                if (ks == kb &&
                    !mbar_wait(&bar->acc_empty[ab], ((uint32_t)(t >> 1) & 1) ^ 1, status))
                    break;
                if (!next && !mbar_wait(&bar->full[s], p, status)) break;
                tc_fence_after();
                // ask now whether the next stage is ready: the answer is needed only after this
                // stage's MMAs have been issued
                const int s1 = s + 1 == STAGES ? 0 : s + 1;
                next = mbar_test_wait(&bar->full[s1], s1 == 0 ? p ^ 1 : p);
                const uint32_t d_tmem = tmem + ab * BN;
                const uint32_t a_st = sa_addr + (uint32_t)s * A_STAGE_BYTES;
                const uint32_t b_st = sb_addr + (uint32_t)s * B_STAGE_BYTES;
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    const uint64_t adesc = smem_desc_kmajor_sw128(a_st + sub * SUB_BYTES);
                    const uint64_t bdesc = smem_desc_kmajor_sw128(b_st + sub * SUB_BYTES);
#pragma unroll
                    for (int kk = 0; kk < SUBK / UMMA_K; ++kk)
                        mma_i8_ss_pair(d_tmem, adesc + (uint64_t)(kk * UMMA_K / 16),
                                       bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                                       (ks != kb || sub != 0 || kk != 0) ? 1u : 0u);
                }
                mma_commit_pair(&bar->empty[s], 3);
                if (ks == ke - 1) mma_commit_pair(&bar->acc_full[ab], 3);
                if (++ks == ke && ++t < my_units) {
                    unit(t, tile, kb, ke);
                    ks = kb;
                }
                s = s1;
                if (s == 0) p ^= 1;
            }
            // every MMA issued above has finished before either CTA releases tensor memory
            mma_commit_pair(&bar->done, 3);
        }
        if (lane == 0) mbar_wait(&bar->done, 0, status);
        __syncwarp();
    } else if (wi >= 0 && wi < 4 * B_GROUPS) {
        // ------------------------------------------------------------------ weight unpack
        const int grp = wi >> 2;             // takes iterations it = grp (mod B_GROUPS)
        const int rr = (wi & 3) * 32 + lane;  // row of this CTA's B half = feature
        const int sx = (rr >> 1) & 3;
        for (int it = grp; it < total; it += B_GROUPS) {
            const int s = it % STAGES, s_w = it % W_STAGES;
            if (!warp_wait(&bar->full_w[s_w], (uint32_t)(it / W_STAGES) & 1, status, lane)) break;
            // row rr of the weight tile: 64 B, 16-byte chunk c stored at chunk c ^ ((rr >> 1) & 3)
            // (64-byte swizzle: conflict-free reads down the rows)
            const uint8_t *wrow = sw + (size_t)s_w * W_STAGE_BYTES + rr * (BK / 4);
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 v = *reinterpret_cast<const uint4 *>(wrow + ((c ^ sx) << 4));
                w[4 * c] = v.x;
                w[4 * c + 1] = v.y;
                w[4 * c + 2] = v.z;
                w[4 * c + 3] = v.w;
            }
            if (!warp_wait(&bar->empty[s], ((uint32_t)(it / STAGES) & 1) ^ 1, status, lane))
                break;
            // packed word g holds k = 16g .. 16g+15; (w >> 2p) & 0x03030303 is k = 16g+4p .. +3,
            // so word g becomes 16-byte chunk g of the row: sub-tile g / 8, stored at chunk
            // (g % 8) ^ (rr & 7)
            uint8_t *brow = sb + (size_t)s * B_STAGE_BYTES + rr * SUBK;
#pragma unroll
            for (int g = 0; g < 16; ++g) {
                uint4 o;
                o.x = w[g] & 0x03030303u;
                o.y = (w[g] >> 2) & 0x03030303u;
                o.z = (w[g] >> 4) & 0x03030303u;
                o.w = (w[g] >> 6) & 0x03030303u;
                *reinterpret_cast<uint4 *>(brow + (g >> 3) * SUB_BYTES + (((g & 7) ^ (rr & 7)) << 4)) =
                    o;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive_cluster(mapa_shared(smem_addr(&bar->full[s]), 0));
                mbar_arrive(&bar->empty_w[s_w]);  // the packed tile was consumed above
            }
        }
    } else if (warp >= WARP_EPI && warp < WARP_EPI + EPI_WARPS) {
        // ------------------------------------------------------------------ epilogue
        const int wq = warp & 3;                   // TMEM lanes 32*wq .. 32*wq+31 = tokens
        const int half = (warp - WARP_EPI) >> 2;   // features 128*half .. 128*half+127
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        uint8_t *ybox = sy + (size_t)(warp - WARP_EPI) * Y_BOX_BYTES;
        const float gamma = *gamma_ptr;
        for (int t = 0; t < my_units; ++t) {
            int tile, kb, ke;
            unit(t, tile, kb, ke);
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
                if constexpr (MODE == OUT_ACC) {
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
                    // bf16 pairs of this token's 32 features, then out through the warp's
                    // staging box by bulk tensor stores: 16 features x 32 tokens per store, the
                    // box rows in the 32-byte-swizzled layout (chunk c of row r at c ^ (r >> 2 & 1))
                    // (SwiGLU: pair i of the chunk is (gate, up) = features 2i, 2i+1; its 16
                    // outputs fill one box at output column n0 / 2)
                    constexpr int BOXES = MODE == OUT_SWIGLU ? 1 : 2;
                    uint32_t pk[16];
                    if constexpr (MODE == OUT_SWIGLU) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            float o[2];
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float g = (float)((int)v[4 * i + 2 * e] - rs) * sc;
                                const float u = (float)((int)v[4 * i + 2 * e + 1] - rs) * sc;
                                o[e] = __fdiv_rn(g, 1.f + expf(-g)) * u;
                            }
                            const __nv_bfloat162 h = __floats2bfloat162_rn(o[0], o[1]);
                            pk[i] = *reinterpret_cast<const uint32_t *>(&h);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float y0 = (float)((int)v[2 * i] - rs) * sc;
                            float y1 = (float)((int)v[2 * i + 1] - rs) * sc;
                            if constexpr (MODE == OUT_RELU2) {
                                y0 = y0 > 0.f ? y0 * y0 : 0.f;
                                y1 = y1 > 0.f ? y1 * y1 : 0.f;
                            }
                            const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
                            pk[i] = *reinterpret_cast<const uint32_t *>(&h);
                        }
                    }
                    const int m_w = mt * BM + (int)rank * HM + wq * 32;  // the warp's first token
                    const int sx = (lane >> 2) & 1;
                    const int nx0 = MODE == OUT_SWIGLU ? n0 / 2 : n0;  // first output column
                    const int n_out = MODE == OUT_SWIGLU ? N / 2 : N;
#pragma unroll
                    for (int hb = 0; hb < BOXES; ++hb) {
                        if (lane == 0) bulk_wait_group_read<0>();  // the previous box was read
                        __syncwarp();
#pragma unroll
                        for (int c = 0; c < 2; ++c)
                            *reinterpret_cast<uint4 *>(ybox + lane * (Y_BOX_N * 2) + ((c ^ sx) << 4)) =
                                make_uint4(pk[8 * hb + 4 * c], pk[8 * hb + 4 * c + 1],
                                           pk[8 * hb + 4 * c + 2], pk[8 * hb + 4 * c + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        // rows >= M and features >= N of a box are not written; a box wholly
                        // outside Y is not issued
                        if (lane == 0 && m_w < M && nx0 + hb * Y_BOX_N < n_out) {
                            tma_store_2d(&tmap_y, ybox, nx0 + hb * Y_BOX_N, m_w);
                            bulk_commit_group();
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->acc_empty[ab]), 0));
        }
        // the staging box stays in use until its last store has completed
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    } else if (BITS == 4 && wi >= 4) {
        // ------------------------------------------------------------------ INT4 code widening
        // thread = token row of this CTA's half: its 128 packed bytes (256 codes) sit in the
        // second sub-tile; it reads them all, then writes 256 int8 codes over both sub-tiles
        // (the row's own 128-byte slots, so no other thread's input is overwritten)
        const int row = (wi - 4) * 32 + lane;
        const int sx = row & 7;
        for (int it = 0; it < total; ++it) {
            const int s = it % STAGES;
            if (!warp_wait(&bar->packed[s], (uint32_t)(it / STAGES) & 1, status, lane)) break;
            uint8_t *arow = sa + (size_t)s * A_STAGE_BYTES + row * SUBK;
            uint4 raw[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                raw[c] = *reinterpret_cast<const uint4 *>(arow + SUB_BYTES + ((c ^ sx) << 4));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                // 32 codes k = 32c .. 32c+31 -> 16-byte chunks 2c (words x, y) and 2c+1 (z, w)
                const uint32_t wd[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w0 = wd[2 * h], w1 = wd[2 * h + 1];
                    uint4 o;
                    o.x = sext_nibbles(w0 & 0x0F0F0F0Fu);
                    o.y = sext_nibbles((w0 >> 4) & 0x0F0F0F0Fu);
                    o.z = sext_nibbles(w1 & 0x0F0F0F0Fu);
                    o.w = sext_nibbles((w1 >> 4) & 0x0F0F0F0Fu);
                    const int oc = 2 * c + h;  // chunk of the 256-byte row: sub-tile oc / 8
                    *reinterpret_cast<uint4 *>(arow + (oc >> 3) * SUB_BYTES + (((oc & 7) ^ sx) << 4)) =
                        o;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->full[s]), 0));
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
template <int BITS, int MODE>
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
    if (cudaOccupancyMaxActiveClusters(&clusters, ternary_gemm_tc_kernel<BITS, MODE>, &cfg) !=
            cudaSuccess ||
        clusters < 1) {
        (void)cudaGetLastError();
        clusters = num_sms / 2;
    }
    if (dev >= 0 && dev < 64) cache[dev] = clusters;
    return clusters;
}

template <int BITS, int MODE>
static cudaError_t launch_tc_t(const GemmArgs &a, const CUtensorMap &mc, const CUtensorMap &mw,
                               const CUtensorMap &my, void *out, int64_t tiles, int num_sms,
                               cudaStream_t stream) {
    auto kern = ternary_gemm_tc_kernel<BITS, MODE>;
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const int pairs_max = max_pairs<BITS, MODE>(num_sms);
    const int pairs = (int)(tiles < pairs_max ? tiles : pairs_max);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mc, mw, my, out, a.scales, a.rowsum, a.gamma, (int)a.M,
                              (int)a.N, (int)a.K, a.status);
}

}  // namespace tc

CUresult encode_tmap_2d(void *encode_fn, CUtensorMap *map, CUtensorMapDataType dt,
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
                                   cudaStream_t stream, int *launches) {
    using namespace tc;
    const int64_t tiles = ((a.N + BN - 1) / BN) * ((a.M + BM - 1) / BM);
    CUtensorMap mc, mw, my;
    memset(&mc, 0, sizeof mc);
    memset(&mw, 0, sizeof mw);
    memset(&my, 0, sizeof my);
    // codes: INT8 [M rows][K bytes], two [128 tokens x 128 B] boxes per CTA and stage;
    // INT4 [M rows][K/2 bytes], one [128 tokens x 128 B] box of packed nibbles per CTA and stage;
    // both with the 128-byte swizzle
    const uint64_t cb = a.act_bits == 8 ? (uint64_t)a.K : (uint64_t)a.K / 2;
    if (encode_tmap_2d(encode_fn, &mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, cb, (uint64_t)a.M, cb,
                  SUBK, HM, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // packed weights: [N rows][K/4 bytes], one [128 features x 64 B] box per stage, 64-byte
    // swizzle
    if (encode_tmap_2d(encode_fn, &mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, (uint64_t)a.K / 4,
                  (uint64_t)a.N, (uint64_t)a.K / 4, BK / 4, HN,
                  CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (launches) *launches = (a.Y ? 1 : 0) + (a.acc ? 1 : 0);
    if (a.Y) {
        // bf16 output [M rows][N] (N/2 with SwiGLU), one [32 tokens x 16 features] box per
        // store, 32-byte swizzle
        const uint64_t n_out = a.activation == 2 ? (uint64_t)a.N / 2 : (uint64_t)a.N;
        if (encode_tmap_2d(encode_fn, &my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Y, n_out, (uint64_t)a.M,
                      n_out * 2, Y_BOX_N, 32, CU_TENSOR_MAP_SWIZZLE_32B) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        switch (a.activation * 2 + (a.act_bits == 8 ? 1 : 0)) {
            case 0: e = launch_tc_t<4, OUT_BF16>(a, mc, mw, my, a.Y, tiles, num_sms, stream); break;
            case 1: e = launch_tc_t<8, OUT_BF16>(a, mc, mw, my, a.Y, tiles, num_sms, stream); break;
            case 2: e = launch_tc_t<4, OUT_RELU2>(a, mc, mw, my, a.Y, tiles, num_sms, stream); break;
            case 3: e = launch_tc_t<8, OUT_RELU2>(a, mc, mw, my, a.Y, tiles, num_sms, stream); break;
            case 4: e = launch_tc_t<4, OUT_SWIGLU>(a, mc, mw, my, a.Y, tiles, num_sms, stream); break;
            case 5: e = launch_tc_t<8, OUT_SWIGLU>(a, mc, mw, my, a.Y, tiles, num_sms, stream); break;
            default: return cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
    }
    if (a.acc) {
        e = a.act_bits == 8 ? launch_tc_t<8, OUT_ACC>(a, mc, mw, my, a.acc, tiles, num_sms, stream)
                            : launch_tc_t<4, OUT_ACC>(a, mc, mw, my, a.acc, tiles, num_sms, stream);
    }
    return e;
}

}  // namespace bitnet
