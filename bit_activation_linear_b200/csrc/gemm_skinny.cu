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
// 512 weights (16 KB, 128-byte swizzle); eight unpack warps (two per tensor-memory lane quadrant,
// each taking half of the stage's K) turn their rows into int8 lanes with one shift-and-mask per
// four weights (word g of a row holds k = 16g .. 16g+15; the shift by 2p gives k = 16g+4p .. +3,
// which is exactly tensor-memory column 4g + p of that row) and write them straight into tensor
// memory with tcgen05.st, where the MMA reads its A operand (tcgen05.mma ... [d], [a_tmem],
// b_desc).  Shared memory only holds the packed weights (read once) and the tokens' codes (B
// operand, K-major, 128-byte swizzle).
//
// With so few tokens each MMA holds little work (128 x MT x 32), and one thread issues an MMA only
// every ~53 cycles on B200 whatever its size; with the operand A in tensor memory two issuing
// threads double the rate (measured: 128 x 64 x 32 then runs at the tensor pipe's 32 cycles).  So
// two MMA warps issue alternate halves of every stage into accumulators of their own, and the
// epilogue adds the two.
//
// K split over a cluster: a feature block has KS = K / 512 stages; the S CTAs of a cluster (S <= 8,
// chosen so that the grid fills the GPU) take consecutive chunks of them.  Each CTA copies its
// int32 partial sums from tensor memory to its own shared memory; after a cluster barrier every
// CTA sums a share of the outputs over the S CTAs' shared memory (distributed shared memory
// loads) and applies the epilogue (offset, d_m * gamma, bf16 and the optional activation) with
// the same fp32 operations as the other product kernels, so every path gives the same bits.
// No global scratch is used: calls on different streams may run concurrently.
//
// Warp roles (416 threads): warps 0-7 unpack (warp w owns tensor-memory lanes 32(w%4) .. +31, i.e.
// features 32(w%4) .., and half w/4 of each stage's K); warps 0-3 then run the epilogue; warp 8
// issues the TMA loads; warps 9 and 10 each issue half of the MMAs (one thread each), warp 9 also
// allocates tensor memory; warps 11-12 widen INT4 codes to int8 in place (thread = token row).  Every mbarrier wait is bounded: after ~1 s a role records BITNET_ERR_TIMEOUT and
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
constexpr int A_STAGES = 3;               // unpacked weight stages in tensor memory
constexpr int A_COLS = KST / 4;           // 128 columns of 4 int8 each per A stage
constexpr int ACC_COL = A_STAGES * A_COLS;
constexpr int TMEM_COLS = 512;
constexpr int UNPACK_WARPS = 8;           // two per lane quadrant, one per half of a stage's K
constexpr int ISSUERS = 2;                // MMA-issuing warps, one per half, one accumulator each
constexpr int W_STAGES = 8;               // packed-weight ring (HBM latency: ~2300 cycles)
constexpr int WARP_WTMA = 8, WARP_MMA = 9, WARP_CTMA = 11, WARP_CODE = 12, CODE_WARPS = 2;
constexpr int NUM_THREADS = (WARP_CODE + CODE_WARPS) * 32;

template <int MT>
struct Cfg {
    static constexpr int CBYTES = MT * KST;                    // int8 codes of a stage
    static constexpr int C_STAGES = MT >= 64 ? 3 : 4;          // code ring (L2 hits)
    static constexpr int W_OFF = 0;
    static constexpr int C_OFF = W_STAGES * WBYTES;
    static constexpr int BAR_OFF = C_OFF + C_STAGES * CBYTES;
    static constexpr int RED_BYTES = MT * FEAT * 4;            // int32 partials [MT][FEAT]
    static constexpr size_t SMEM = (size_t)BAR_OFF + 512 + 1024;  // + barriers + alignment
    static_assert(RED_BYTES <= W_STAGES * WBYTES, "the partials reuse the weight ring");
    static_assert(CBYTES % 1024 == 0 && (MT * SUB) % 1024 == 0, "swizzle-atom alignment");
    static_assert(ACC_COL + ISSUERS * MT <= TMEM_COLS, "tensor-memory budget");
    static_assert(SMEM <= 227 * 1024, "shared-memory budget");
};

struct __align__(8) Bars {
    uint64_t full_w[W_STAGES];           // TMA bytes of the weight slot have landed
    uint64_t empty_w[W_STAGES];          // every unpack warp has read the weight slot
    uint64_t full_c[4];                  // TMA bytes of the code slot have landed
    uint64_t cfull[4];                   // INT4: the code warps have widened the slot's codes
    uint64_t empty_c[4];                 // both issuers' MMAs reading the code slot have completed
    uint64_t a_full[A_STAGES][ISSUERS];  // the four unpack warps of a half have written it
    uint64_t a_empty[A_STAGES][ISSUERS]; // the MMAs of that half have completed (commit)
    uint64_t acc_full;                   // every MMA of this CTA has completed (both issuers)
    uint32_t tmem_base;
};
static_assert(sizeof(Bars) <= 512, "barrier area");

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
    uint8_t *wring = smem + C::W_OFF;
    uint8_t *cring = smem + C::C_OFF;
    Bars *bar = reinterpret_cast<Bars *>(smem + C::BAR_OFF);

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
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&bar->full_w[s], 1);
            mbar_init(&bar->empty_w[s], UNPACK_WARPS);
        }
        for (int s = 0; s < C::C_STAGES; ++s) {
            mbar_init(&bar->full_c[s], 1);
            mbar_init(&bar->cfull[s], CODE_WARPS);
            mbar_init(&bar->empty_c[s], ISSUERS);
        }
        for (int a = 0; a < A_STAGES; ++a)
            for (int h = 0; h < ISSUERS; ++h) {
                mbar_init(&bar->a_full[a][h], UNPACK_WARPS / ISSUERS);
                mbar_init(&bar->a_empty[a][h], 1);
            }
        mbar_init(&bar->acc_full, ISSUERS);
        fence_mbar_init();
    }
    if (warp == WARP_WTMA && lane == 0) {
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
    // the next kernel of the stream may be scheduled now; it waits for this grid's completion
    // before it reads anything (griddepcontrol.wait)
    pdl_launch_dependents();

    if (warp == WARP_WTMA) {
        // ------------------------------------------------------------------ weight TMA
        if (lane == 0) {
            // With early_weights the caller guarantees the packed weights were complete before
            // the preceding kernel (the quantiser) started, so they may be requested before that
            // kernel finishes; otherwise every global read waits for it (programmatic dependent
            // launch).
            if (!early_weights) pdl_wait();
            uint32_t issued = 0, ph = 0;  // slots with a load issued, and that load's phase
            for (int it = 0; it < nst; ++it) {
                const int s = it % W_STAGES;
                const uint32_t p = (uint32_t)(it / W_STAGES) & 1;
                if (!mbar_wait(&bar->empty_w[s], p ^ 1, status)) break;
                mbar_arrive_expect_tx(&bar->full_w[s], WBYTES);
                tma_load_2d(wring + (size_t)s * WBYTES, &tmap_w, (kb + it) * (KST / 4), n0,
                            &bar->full_w[s]);
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
            }
            // no copy may still be landing in shared memory when the CTA moves on
            for (int s = 0; s < W_STAGES; ++s)
                if (issued & (1u << s)) mbar_wait(&bar->full_w[s], (ph >> s) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_CTMA) {
        // ------------------------------------------------------------------ code TMA
        if (lane == 0) {
            pdl_wait();
            uint32_t issued = 0, ph = 0;
            for (int it = 0; it < nst; ++it) {
                const int s = it % C::C_STAGES;
                const uint32_t p = (uint32_t)(it / C::C_STAGES) & 1;
                if (!mbar_wait(&bar->empty_c[s], p ^ 1, status)) break;
                uint8_t *st = cring + (size_t)s * C::CBYTES;
                mbar_arrive_expect_tx(&bar->full_c[s], CB);
                const int kx = (kb + it) * KST;  // first weight of the stage
                if constexpr (BITS == 8) {
#pragma unroll
                    for (int j = 0; j < SUBS; ++j)
                        tma_load_2d(st + j * MT * SUB, &tmap_c, kx + j * SUB, 0, &bar->full_c[s]);
                } else {
                    // packed nibbles (256 B per token) into the last two sub-tiles; the code warps
                    // widen them in place
#pragma unroll
                    for (int j = 0; j < 2; ++j)
                        tma_load_2d(st + (2 + j) * MT * SUB, &tmap_c, kx / 2 + j * SUB, 0,
                                    &bar->full_c[s]);
                }
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
            }
            for (int s = 0; s < C::C_STAGES; ++s)
                if (issued & (1u << s)) mbar_wait(&bar->full_c[s], (ph >> s) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_MMA || warp == WARP_MMA + 1) {
        // ------------------------------------------------------------------ MMA issuers
        // issuer i takes code sub-tiles 2i and 2i+1 of every stage (half i of its K, written by
        // unpack warps 4i .. 4i+3) into accumulator i
        if (lane == 0) {
            const int i = warp - WARP_MMA;
            constexpr uint32_t IDESC = idesc_i8_u8s8(FEAT, MT);
            const uint32_t cbase = smem_addr(cring);
            const uint32_t d_tmem = tmem + (uint32_t)(ACC_COL + i * MT);
            for (int it = 0; it < nst; ++it) {
                const int cs = it % C::C_STAGES, as = it % A_STAGES;
                if (!mbar_wait(&bar->a_full[as][i], (uint32_t)(it / A_STAGES) & 1, status)) break;
                if (!mbar_wait(BITS == 8 ? &bar->full_c[cs] : &bar->cfull[cs],
                               (uint32_t)(it / C::C_STAGES) & 1, status))
                    break;
                tc_fence_after();
                const uint32_t cst = cbase + (uint32_t)(cs * C::CBYTES);
#pragma unroll
                for (int jj = 0; jj < SUBS / ISSUERS; ++jj) {
                    const int j = i * (SUBS / ISSUERS) + jj;
                    const uint64_t bdesc = smem_desc_kmajor_sw128(cst + j * MT * SUB);
#pragma unroll
                    for (int kk = 0; kk < SUB / UMMA_K; ++kk)
                        mma_i8_ts(d_tmem,
                                  tmem + (uint32_t)(as * A_COLS + (j * (SUB / UMMA_K) + kk) * 8),
                                  bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                                  (it | jj | kk) != 0 ? 1u : 0u);
                }
                mma_commit(&bar->a_empty[as][i]);
                mma_commit(&bar->empty_c[cs]);
            }
            // arrives once every MMA this thread issued has completed (also after a time-out)
            mma_commit(&bar->acc_full);
        }
        __syncwarp();
    } else if (warp >= WARP_CODE) {
        // ------------------------------------------------------------------ INT4 code widening
        if constexpr (BITS == 4) {
            // thread = token row: its 256 packed bytes (512 codes) sit in sub-tiles 2 and 3.  Half
            // h2 reads packed sub-tile 2 + h2 (codes 256*h2 ..) whole, then writes its 256 int8
            // codes over sub-tiles 2*h2 and 2*h2 + 1 of the row: half 0 writes sub-tiles 0-1 (no
            // input there), half 1 overwrites sub-tile 2 (already read) and 3 (read just before)
            const int row = (warp - WARP_CODE) * 32 + lane;
            const int sx = row & 7;
            for (int it = 0; it < nst; ++it) {
                const int s = it % C::C_STAGES;
                if (!warp_wait(&bar->full_c[s], (uint32_t)(it / C::C_STAGES) & 1, status, lane))
                    break;
                if (row < MT) {
                    uint8_t *crow = cring + (size_t)s * C::CBYTES + row * SUB;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                    uint4 raw[8];
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc)
                        raw[cc] = *reinterpret_cast<const uint4 *>(crow + (2 + h2) * MT * SUB +
                                                                    ((cc ^ sx) << 4));
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        // 32 codes k = 32c .. 32c+31 (c = 8*h2 + cc) -> output chunks 2c (words
                        // x, y) and 2c+1 (z, w)
                        const int c = 8 * h2 + cc;
                        const uint32_t wd[4] = {raw[cc].x, raw[cc].y, raw[cc].z, raw[cc].w};
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
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->cfull[s]);
            }
        }
    } else {
        // ------------------------------------------------------------------ weight unpack
        const int quad = warp & 3, half = warp >> 2;
        const int r = quad * 32 + lane;  // feature row of the block = tensor-memory lane
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        for (int it = 0; it < nst; ++it) {
            const int s = it % W_STAGES, as = it % A_STAGES;
            if (!warp_wait(&bar->full_w[s], (uint32_t)(it / W_STAGES) & 1, status, lane)) break;
            // row r of the weight tile: 128 B, 16-byte chunk c stored at chunk c ^ (r & 7); this
            // warp takes chunks 4*half .. 4*half+3 (k = 256*half .. +255)
            const uint8_t *wrow = wring + (size_t)s * WBYTES + r * (KST / 4);
            uint4 v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                v[c] = *reinterpret_cast<const uint4 *>(wrow + (((4 * half + c) ^ (r & 7)) << 4));
            // the refill is an async-proxy write: without a proxy fence after each lane's plain
            // reads it may overtake them (measured on B200: rows of a slot read after the refill
            // had begun landing)
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->empty_w[s]);  // the slot may be refilled
            if (!warp_wait(&bar->a_empty[as][half], ((uint32_t)(it / A_STAGES) & 1) ^ 1, status,
                           lane))
                break;
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < 2; ++q) {  // words 8q .. 8q+7 of the half -> 32 columns
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
                tmem_st_32x32b_x32(t_lane + (uint32_t)(as * A_COLS + 64 * half + 32 * q), o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->a_full[as][half]);
        }
        if (warp < 4) {
            // ---- this CTA's partial sums (the two accumulators added): tensor memory ->
            // shared memory [MT tokens][FEAT] ----
            warp_wait(&bar->acc_full, 0, status, lane);
            tc_fence_after();
            // the weight ring has been consumed: every unpack warp has read every slot, and the
            // MMAs that followed have completed
            int32_t *red = reinterpret_cast<int32_t *>(wring);
#pragma unroll
            for (int q = 0; q < MT / 16; ++q) {
                uint32_t v0[16], v1[16];
                tmem_ld_32x32b_x16(t_lane + (uint32_t)(ACC_COL + 16 * q), v0);
                tmem_ld_32x32b_x16(t_lane + (uint32_t)(ACC_COL + MT + 16 * q), v1);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    red[(16 * q + j) * FEAT + r] = (int32_t)(v0[j] + v1[j]);
            }
            tc_fence_before();
        }
    }

    // every CTA of the cluster has its partial sums in shared memory
    __syncwarp();
    cluster_sync();

    if (warp < 4) {
        // ------------------------------------------------------------------ epilogue
        // unit = (token m, 8 consecutive features); CTA `rank` takes every S-th group of 128
        pdl_wait();  // scales, code sums and Y belong to the stream order (returns at once here)
        const float gamma = *gamma_ptr;
        const uint32_t red_addr = smem_addr(wring);
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
                                         (int)Cfg<MT>::SMEM);
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
    cfg.dynamicSmemBytes = Cfg<64>::SMEM;
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
    cfg.dynamicSmemBytes = Cfg<MT>::SMEM;
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
