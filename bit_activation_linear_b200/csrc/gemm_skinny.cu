// gemm_skinny.cu -- step 4 for a few tokens (9 .. 64, decode and small batches): the ternary x
// integer product on the tensor cores with the weights on the MMA's M side ("swap AB"), streamed
// from HBM once.
//
// 2B4T article, section 一.2 (W1.58A8: the product is additions and subtractions) and section
// 三.3 (GPU kernel: pack-store-load-unpack-compute).  With few tokens the product is bound by the
// stream of packed weights, NK/4 bytes, and by how fast they can be turned into tensor-core
// operands.  A tile of 256 tokens x 256 features would leave most of its rows empty, so here the
// roles are swapped: each CTA owns 128 output features (MMA M = 128, one per tensor-memory lane)
// and all tokens (MMA N = MT = 16, 32 or 64; missing tokens are zero rows of the TMA box):
//   D[feature, token] = sum_k u[feature, k] * c[token, k]   (u = q + 1 unsigned, c signed)
// in int32 in tensor memory, and the per-token code sum removes the offset as in the other
// product kernels.
//
// The packed weights never go through shared memory twice: TMA brings a stage of 128 features x
// 512 weights (16 KB, 128-byte swizzle); each of four unpack warps turns its 32 rows into int8
// lanes with one shift-and-mask per four weights (word g of a row holds k = 16g .. 16g+15; the
// shift by 2p gives k = 16g+4p .. +3, which is exactly tensor-memory column 4g + p of that row) and
// writes them straight into tensor memory with tcgen05.st, where the MMA reads its A operand
// (tcgen05.mma ... [d], [a_tmem], b_desc).  Shared memory only holds the packed weights (read
// once) and the tokens' codes (B operand, K-major, 128-byte swizzle).
//
// K split over a cluster: a feature block has KS = K / 512 stages; the S CTAs of a cluster (S <= 8,
// chosen so that the grid fills the GPU) take consecutive chunks of them.  Each CTA copies its
// int32 partial sums from tensor memory to its own shared memory; after a cluster barrier every
// CTA sums a share of the outputs over the S CTAs' shared memory (distributed shared memory
// loads) and applies the epilogue (offset, d_m * gamma, bf16 and the optional activation) with
// the same fp32 operations as the other product kernels, so every path gives the same bits.
// No global scratch is used: calls on different streams may run concurrently.
//
// Warp roles (256 threads): warps 0-3 unpack (warp w owns tensor-memory lanes 32w .. 32w+31, i.e.
// features 32w ..), then run the epilogue; warp 4 issues the TMA loads; warp 5 allocates tensor
// memory and (one thread) issues the MMAs; warps 6-7 widen INT4 codes to int8 in place (thread =
// token row).  Every mbarrier wait is bounded: after ~1 s a role records BITNET_ERR_TIMEOUT and
// stops, and every thread still meets the cluster barriers, so the kernel always returns.  No TMA
// multicast is used.
#include "common.cuh"
#include "kernels.h"

#include <cudaTypedefs.h>

namespace bitnet {
namespace sk {

constexpr int FEAT = 128;                 // output features per CTA (MMA M, tensor-memory lanes)
constexpr int KST = 512;                  // K per stage
constexpr int UMMA_K = 32;                // K per kind::i8 MMA
constexpr int WBYTES = FEAT * KST / 4;    // 16 KB of packed weights per stage
constexpr int SUB = 128;                  // bytes of K per code sub-tile row (one swizzle row)
constexpr int SUBS = KST / SUB;           // 4 code sub-tiles per stage
constexpr int A_STAGES = 2;               // unpacked weight stages in tensor memory
constexpr int A_COLS = KST / 4;           // 128 columns of 4 int8 each per A stage
constexpr int ACC_COL = A_STAGES * A_COLS;
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 256;
constexpr int WARP_TMA = 4, WARP_MMA = 5, WARP_CODE = 6, CODE_WARPS = 2;
constexpr int MAX_STAGES = 8;

template <int MT>
struct Cfg {
    static constexpr int CBYTES = MT * KST;                    // int8 codes per stage
    static constexpr int STAGE_BYTES = WBYTES + CBYTES;
    static constexpr int STAGES_FIT = (200 * 1024) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT < MAX_STAGES ? STAGES_FIT : MAX_STAGES;
    static constexpr int RED_BYTES = MT * FEAT * 4;            // int32 partials [MT][FEAT]
    static_assert(STAGES >= 2, "stages");
    static_assert(RED_BYTES <= STAGES * STAGE_BYTES, "the partials reuse the stage memory");
    static_assert(STAGE_BYTES % 1024 == 0 && (MT * SUB) % 1024 == 0, "swizzle-atom alignment");
    static_assert(ACC_COL + MT <= TMEM_COLS, "tensor-memory budget");
};

struct __align__(8) Bars {
    uint64_t full[MAX_STAGES];   // TMA bytes of the stage (weights and codes) have landed
    uint64_t cfull[MAX_STAGES];  // INT4: the code warps have widened the stage's codes
    uint64_t empty[MAX_STAGES];  // the stage's MMAs have completed (commit)
    uint64_t a_full[A_STAGES];   // the four unpack warps have written the A stage
    uint64_t a_empty[A_STAGES];  // the MMAs reading the A stage have completed (commit)
    uint64_t acc_full;           // every MMA of this CTA has completed (commit)
    uint32_t tmem_base;
};

// Warp-uniform bounded wait (lane 0 polls; __syncwarp orders the other lanes after it).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, status);
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// MODE: OUT_PLAIN writes the int32 sums (acc) and/or the rescaled bf16 output (Y), whichever
// pointer is given; OUT_RELU2 / OUT_SWIGLU write the activation of the rescaled output (SwiGLU:
// interleaved gate / up features, N/2 output columns).
enum Mode { OUT_PLAIN = 0, OUT_RELU2 = 1, OUT_SWIGLU = 2 };

template <int BITS, int MT, int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ternary_gemm_skinny_kernel(const __grid_constant__ CUtensorMap tmap_w,
                               const __grid_constant__ CUtensorMap tmap_c,
                               int32_t *__restrict__ acc_out, __nv_bfloat16 *__restrict__ Y,
                               const float *__restrict__ scales,
                               const int32_t *__restrict__ rowsum,
                               const float *__restrict__ gamma_ptr, int M, int N, int K,
                               int early_weights, int *status) {
    using C = Cfg<MT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars *bar = reinterpret_cast<Bars *>(smem + (size_t)C::STAGES * C::STAGE_BYTES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = (int)cluster_nctarank();     // CTAs sharing this feature block's K axis
    const int rank = (int)cluster_ctarank();   // this CTA's K chunk
    const int n0 = (int)(blockIdx.x / S) * FEAT;
    const int KS = (K + KST - 1) / KST;
    const int kb = rank * KS / S;
    const int nst = (rank + 1) * KS / S - kb;  // >= 1: the launcher keeps S <= KS
    constexpr uint32_t CB = BITS == 8 ? MT * KST : MT * KST / 2;  // code bytes a stage loads

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&bar->full[s], 1);
            mbar_init(&bar->cfull[s], CODE_WARPS);
            mbar_init(&bar->empty[s], 1);
        }
        for (int a = 0; a < A_STAGES; ++a) {
            mbar_init(&bar->a_full[a], 4);
            mbar_init(&bar->a_empty[a], 1);
        }
        mbar_init(&bar->acc_full, 1);
        fence_mbar_init();
    }
    if (warp == WARP_TMA && lane == 0) {
        prefetch_tensormap(&tmap_w);
        prefetch_tensormap(&tmap_c);
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
            // The packed weights of the first stages may be requested before the preceding kernel
            // (the quantiser) has finished, when the caller guarantees they were complete before
            // it started; every other global read waits for it (programmatic dependent launch).
            const int pre = early_weights ? (nst < C::STAGES ? nst : C::STAGES) : 0;
            for (int it = 0; it < pre; ++it) {
                mbar_arrive_expect_tx(&bar->full[it], WBYTES + CB);
                tma_load_2d(smem + (size_t)it * C::STAGE_BYTES, &tmap_w, (kb + it) * (KST / 4), n0,
                            &bar->full[it]);
            }
            pdl_wait();
            uint32_t issued = 0, ph = 0;  // slots with a load issued, and that load's phase
            for (int it = 0; it < nst; ++it) {
                const int s = it % C::STAGES;
                const uint32_t p = (uint32_t)(it / C::STAGES) & 1;
                uint8_t *st = smem + (size_t)s * C::STAGE_BYTES;
                if (it >= pre) {
                    if (!mbar_wait(&bar->empty[s], p ^ 1, status)) break;
                    mbar_arrive_expect_tx(&bar->full[s], WBYTES + CB);
                    tma_load_2d(st, &tmap_w, (kb + it) * (KST / 4), n0, &bar->full[s]);
                }
                const int kx = (kb + it) * KST;  // first weight of the stage
                if constexpr (BITS == 8) {
#pragma unroll
                    for (int j = 0; j < SUBS; ++j)
                        tma_load_2d(st + WBYTES + j * MT * SUB, &tmap_c, kx + j * SUB, 0,
                                    &bar->full[s]);
                } else {
                    // packed nibbles (256 B per token) into the last two sub-tiles; the code warps
                    // widen them in place
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        tma_load_2d(st + WBYTES + (2 + j) * MT * SUB, &tmap_c, kx / 2 + j * SUB, 0,
                                    &bar->full[s]);
                }
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
            }
            // no copy may still be landing in shared memory when the CTA moves on
            for (int s = 0; s < C::STAGES; ++s)
                if (issued & (1u << s)) mbar_wait(&bar->full[s], (ph >> s) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_i8_u8s8(FEAT, MT);
            const uint32_t base = smem_addr(smem);
            for (int it = 0; it < nst; ++it) {
                const int s = it % C::STAGES, as = it % A_STAGES;
                if (!mbar_wait(&bar->a_full[as], (uint32_t)(it / A_STAGES) & 1, status)) break;
                if (!mbar_wait(BITS == 8 ? &bar->full[s] : &bar->cfull[s],
                               (uint32_t)(it / C::STAGES) & 1, status))
                    break;
                tc_fence_after();
                const uint32_t cst = base + (uint32_t)(s * C::STAGE_BYTES + WBYTES);
#pragma unroll
                for (int j = 0; j < SUBS; ++j) {
                    const uint64_t bdesc = smem_desc_kmajor_sw128(cst + j * MT * SUB);
#pragma unroll
                    for (int kk = 0; kk < SUB / UMMA_K; ++kk)
                        mma_i8_ts(tmem + ACC_COL,
                                  tmem + (uint32_t)(as * A_COLS + (j * (SUB / UMMA_K) + kk) * 8),
                                  bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                                  (it | j | kk) != 0 ? 1u : 0u);
                }
                mma_commit(&bar->empty[s]);
                mma_commit(&bar->a_empty[as]);
            }
            // arrives once every MMA issued above has completed (also after a time-out)
            mma_commit(&bar->acc_full);
        }
        __syncwarp();
    } else if (warp >= WARP_CODE) {
        // ------------------------------------------------------------------ INT4 code widening
        if constexpr (BITS == 4) {
            // thread = token row: its 256 packed bytes (512 codes) sit in sub-tiles 2 and 3; it
            // reads them all, then writes 512 int8 codes over the four sub-tiles of its row
            const int row = (warp - WARP_CODE) * 32 + lane;
            const int sx = row & 7;
            for (int it = 0; it < nst; ++it) {
                const int s = it % C::STAGES;
                if (!warp_wait(&bar->full[s], (uint32_t)(it / C::STAGES) & 1, status, lane)) break;
                if (row < MT) {
                    uint8_t *crow = smem + (size_t)s * C::STAGE_BYTES + WBYTES + row * SUB;
                    uint4 raw[16];
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        raw[c] = *reinterpret_cast<const uint4 *>(
                            crow + (2 + c / 8) * MT * SUB + (((c & 7) ^ sx) << 4));
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        // 32 codes k = 32c .. 32c+31 -> output chunks 2c (words x, y), 2c+1 (z, w)
                        const uint32_t wd[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t w0 = wd[2 * h], w1 = wd[2 * h + 1];
                            uint4 o;
                            o.x = sext_nibbles(w0 & 0x0F0F0F0Fu);
                            o.y = sext_nibbles((w0 >> 4) & 0x0F0F0F0Fu);
                            o.z = sext_nibbles(w1 & 0x0F0F0F0Fu);
                            o.w = sext_nibbles((w1 >> 4) & 0x0F0F0F0Fu);
                            const int oc = 2 * c + h;
                            *reinterpret_cast<uint4 *>(crow + (oc / 8) * MT * SUB +
                                                       (((oc & 7) ^ sx) << 4)) = o;
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->cfull[s]);
            }
        }
    } else {
        // ------------------------------------------------------------------ weight unpack
        const int r = warp * 32 + lane;  // feature row of the block = tensor-memory lane
        const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
        for (int it = 0; it < nst; ++it) {
            const int s = it % C::STAGES, as = it % A_STAGES;
            if (!warp_wait(&bar->full[s], (uint32_t)(it / C::STAGES) & 1, status, lane)) break;
            // row r of the weight tile: 128 B, 16-byte chunk c stored at chunk c ^ (r & 7)
            const uint8_t *wrow = smem + (size_t)s * C::STAGE_BYTES + r * (KST / 4);
            uint4 v[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                v[c] = *reinterpret_cast<const uint4 *>(wrow + ((c ^ (r & 7)) << 4));
            if (!warp_wait(&bar->a_empty[as], ((uint32_t)(it / A_STAGES) & 1) ^ 1, status, lane))
                break;
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // words 8q .. 8q+7 -> columns 32q .. 32q+31
                uint32_t o[32];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint4 vv = v[2 * q + g / 4];
                    const uint32_t w = (g & 3) == 0 ? vv.x : (g & 3) == 1 ? vv.y : (g & 3) == 2 ? vv.z : vv.w;
                    o[4 * g] = w & 0x03030303u;
                    o[4 * g + 1] = (w >> 2) & 0x03030303u;
                    o[4 * g + 2] = (w >> 4) & 0x03030303u;
                    o[4 * g + 3] = (w >> 6) & 0x03030303u;
                }
                tmem_st_32x32b_x32(t_lane + (uint32_t)(as * A_COLS + 32 * q), o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->a_full[as]);
        }
        // ---- this CTA's partial sums: tensor memory -> shared memory [MT tokens][FEAT] ----
        warp_wait(&bar->acc_full, 0, status, lane);
        tc_fence_after();
        int32_t *red = reinterpret_cast<int32_t *>(smem);  // every stage has been consumed
#pragma unroll
        for (int q = 0; q < MT / 16; ++q) {
            uint32_t v16[16];
            tmem_ld_32x32b_x16(t_lane + (uint32_t)(ACC_COL + 16 * q), v16);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) red[(16 * q + j) * FEAT + r] = (int32_t)v16[j];
        }
        tc_fence_before();
    }

    // every CTA of the cluster has its partial sums in shared memory
    __syncwarp();
    cluster_sync();

    if (warp < 4) {
        // ------------------------------------------------------------------ epilogue
        // unit = (token m, 8 consecutive features); CTA `rank` takes every S-th group of 128
        pdl_wait();  // scales, code sums and Y belong to the stream order (returns at once here)
        const float gamma = *gamma_ptr;
        const uint32_t red_addr = smem_addr(smem);
        const int units = M * (FEAT / 8);
        for (int u = rank * 128 + (int)threadIdx.x; u < units; u += S * 128) {
            const int m = u / (FEAT / 8);
            const int g = u % (FEAT / 8);
            const int n = n0 + 8 * g;
            if (n >= N) continue;  // N % 8 == 0: a group is whole or absent
            int a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            const uint32_t off = (uint32_t)((m * FEAT + 8 * g) * 4);
            for (int p = 0; p < S; ++p) {
                const uint32_t ra = mapa_shared(red_addr + off, (uint32_t)p);
                const uint4 x0 = ld_shared_cluster_v4(ra), x1 = ld_shared_cluster_v4(ra + 16);
                a[0] += (int)x0.x; a[1] += (int)x0.y; a[2] += (int)x0.z; a[3] += (int)x0.w;
                a[4] += (int)x1.x; a[5] += (int)x1.y; a[6] += (int)x1.z; a[7] += (int)x1.w;
            }
            const int rs = rowsum[m];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] -= rs;
            if constexpr (MODE == OUT_SWIGLU) {
                const float sc = scales[m] * gamma;
                uint32_t pk[2];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float o[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float gt = (float)a[4 * i + 2 * e] * sc;
                        const float up = (float)a[4 * i + 2 * e + 1] * sc;
                        o[e] = __fdiv_rn(gt, 1.f + expf(-gt)) * up;
                    }
                    const __nv_bfloat162 h = __floats2bfloat162_rn(o[0], o[1]);
                    pk[i] = *reinterpret_cast<const uint32_t *>(&h);
                }
                *reinterpret_cast<uint2 *>(Y + (int64_t)m * (N / 2) + n / 2) = make_uint2(pk[0], pk[1]);
            } else {
                if (acc_out) {
                    int4 *dst = reinterpret_cast<int4 *>(acc_out + (int64_t)m * N + n);
                    dst[0] = make_int4(a[0], a[1], a[2], a[3]);
                    dst[1] = make_int4(a[4], a[5], a[6], a[7]);
                }
                if (Y) {
                    const float sc = scales[m] * gamma;
                    uint32_t pk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float y0 = (float)a[2 * i] * sc, y1 = (float)a[2 * i + 1] * sc;
                        if constexpr (MODE == OUT_RELU2) {
                            y0 = y0 > 0.f ? y0 * y0 : 0.f;
                            y1 = y1 > 0.f ? y1 * y1 : 0.f;
                        }
                        const __nv_bfloat162 h = __floats2bfloat162_rn(y0, y1);
                        pk[i] = *reinterpret_cast<const uint32_t *>(&h);
                    }
                    *reinterpret_cast<uint4 *>(Y + (int64_t)m * N + n) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
    }

    // no CTA leaves while a peer may still read its shared memory
    __syncwarp();
    tc_fence_before();
    cluster_sync();
    if (warp == WARP_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------

template <int BITS, int MT, int MODE>
static cudaError_t configure(int dev) {
    static bool done[64] = {};
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev]) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(ternary_gemm_skinny_kernel<BITS, MT, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(Cfg<MT>::STAGES * Cfg<MT>::STAGE_BYTES +
                                               sizeof(Bars) + 1024));
    if (e == cudaSuccess) done[dev] = true;
    return e;
}

// Clusters of S CTAs that can be resident at once on this device, for the largest instance
// (MT = 64, which needs the most shared memory); looked up once per device and S.
static int max_clusters(int S) {
    static int cache[64][9] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || S < 1 || S > 8) return 0;
    if (cache[dev][S] > 0) return cache[dev][S];
    auto kern = ternary_gemm_skinny_kernel<8, 64, OUT_PLAIN>;
    if (configure<8, 64, OUT_PLAIN>(dev) != cudaSuccess) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(S * 16), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg<64>::STAGES * Cfg<64>::STAGE_BYTES + sizeof(Bars) + 1024;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
        (void)cudaGetLastError();
        n = 0;
    }
    cache[dev][S] = n;
    return n;
}

}  // namespace sk

int ternary_gemm_skinny_split(int64_t N, int64_t K) {
    using namespace sk;
    const int64_t blocks = (N + FEAT - 1) / FEAT;
    const int64_t KS = (K + KST - 1) / KST;
    // the largest cluster (<= 8 CTAs, <= KS chunks) whose grid is resident in one wave
    for (int S = (int)(KS < 8 ? KS : 8); S > 1; --S)
        if (blocks <= max_clusters(S)) return S;
    return 1;
}

template <int BITS, int MT, int MODE>
static cudaError_t launch_skinny_t(const GemmArgs &a, const CUtensorMap &mw, const CUtensorMap &mc,
                                   int S, cudaStream_t stream) {
    using namespace sk;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaError_t e = configure<BITS, MT, MODE>(dev);
    if (e != cudaSuccess) return e;
    const int64_t blocks = (a.N + FEAT - 1) / FEAT;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(blocks * S), 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg<MT>::STAGES * Cfg<MT>::STAGE_BYTES + sizeof(Bars) + 1024;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, ternary_gemm_skinny_kernel<BITS, MT, MODE>, mw, mc, a.acc,
                              reinterpret_cast<__nv_bfloat16 *>(a.Y), a.scales, a.rowsum, a.gamma,
                              (int)a.M, (int)a.N, (int)a.K, a.early_weights ? 1 : 0, a.status);
}

template <int BITS, int MT>
static cudaError_t launch_skinny_mode(const GemmArgs &a, const CUtensorMap &mw,
                                      const CUtensorMap &mc, int S, cudaStream_t stream) {
    using namespace sk;
    switch (a.Y ? a.activation : 0) {
        case 1: return launch_skinny_t<BITS, MT, OUT_RELU2>(a, mw, mc, S, stream);
        case 2: return launch_skinny_t<BITS, MT, OUT_SWIGLU>(a, mw, mc, S, stream);
        default: return launch_skinny_t<BITS, MT, OUT_PLAIN>(a, mw, mc, S, stream);
    }
}

template <int BITS>
static cudaError_t launch_skinny_bits(const GemmArgs &a, const CUtensorMap &mw,
                                      const CUtensorMap &mc, int MT, int S, cudaStream_t stream) {
    switch (MT) {
        case 16: return launch_skinny_mode<BITS, 16>(a, mw, mc, S, stream);
        case 32: return launch_skinny_mode<BITS, 32>(a, mw, mc, S, stream);
        default: return launch_skinny_mode<BITS, 64>(a, mw, mc, S, stream);
    }
}

cudaError_t launch_ternary_gemm_skinny(const GemmArgs &a, void *encode_fn, cudaStream_t stream) {
    using namespace sk;
    if (a.M < 1 || a.M > kSkinnyMaxTokens) return cudaErrorInvalidValue;
    const int MT = a.M <= 16 ? 16 : a.M <= 32 ? 32 : 64;
    CUtensorMap mw, mc;
    // packed weights [N rows][K/4 bytes]: one [128 features x 128 B] box per stage
    if (encode_tmap_2d(encode_fn, &mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, (uint64_t)a.K / 4,
                       (uint64_t)a.N, (uint64_t)a.K / 4, KST / 4, FEAT,
                       CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // codes [M rows][K or K/2 bytes]: [MT tokens x 128 B] boxes; rows past M read as zeros
    const uint64_t cb = a.act_bits == 8 ? (uint64_t)a.K : (uint64_t)a.K / 2;
    if (encode_tmap_2d(encode_fn, &mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, cb, (uint64_t)a.M,
                       cb, SUB, (uint32_t)MT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int S = ternary_gemm_skinny_split(a.N, a.K);
    return a.act_bits == 8 ? launch_skinny_bits<8>(a, mw, mc, MT, S, stream)
                           : launch_skinny_bits<4>(a, mw, mc, MT, S, stream);
}

}  // namespace bitnet
