// gemm_tc.cu -- step 4 for many tokens (prefill): the ternary x integer product on the
// 5th-generation tensor cores (tcgen05, kind::i8), accumulating in int32 in tensor memory,
// with the rescale to bf16 fused into the epilogue.
//
// 2B4T article, section 一.2 (W1.58A8 BitLinear; the product needs only additions and
// subtractions) and section 三.3 (GPU kernel: pack-store-load-unpack-compute).  On sm_100a the
// cheapest exact "add/subtract" is the int8 tensor-core MMA: the 2-bit weights are unpacked
// on chip, never in HBM.
//
// Tile: 128 output features (MMA M, operand A) x 128 tokens (MMA N, operand B), K in stages of
// 128.  A persistent CTA per SM walks its tiles; warp roles:
//   warp 0       TMA producer: packed weight tiles [128 rows x 32 B] into a shared-memory ring,
//                and (INT8) code tiles [128 tokens x 128 B] with the 128-byte swizzle straight
//                into the UMMA K-major layout.
//   warp 1       MMA issuer (and TMEM owner): tcgen05.mma.kind::i8 with A from TMEM (unsigned
//                bytes u = q + 1) and B from shared memory (signed codes c), D += u * c;
//                tcgen05.commit frees stages and publishes finished accumulators.
//   warps 4-11   two A-producer warpgroups taking alternate stages, so one group's TMEM store
//                latency hides behind the other's work.  Thread i of a group owns TMEM lane i
//                (output feature n0 + i): it reads its 32 packed bytes from shared memory,
//                expands each 2-bit code to a byte with one shift-and-mask per four weights and
//                writes 32 words into TMEM (tcgen05.st).
//   warps 12-15  epilogue: tcgen05.ld of the int32 accumulator, subtract the token's code sum
//                (sum_k q*c = sum_k u*c - sum_k c), scale by d_m * gamma, round to bf16 (lane
//                pairs swap values so each lane stores one bf16x2 word: conflict-free), stage in
//                shared memory and TMA-store.  Two TMEM accumulators let one tile's epilogue
//                overlap the next tile's main loop.
//   warps 16-19  (INT4 only) B producer: coalesced 16-byte loads of nibble codes, sign-extended
//                to int8 in registers and stored in the swizzled K-major layout.
// Every wait is bounded: after ~1 s a role records BITNET_ERR_TIMEOUT and stops; in-flight TMA
// loads and MMAs are drained before TMEM is released.  No cluster multicast is used.
#include "common.cuh"
#include "kernels.h"

#include <cudaTypedefs.h>

namespace bitnet {
namespace tc {

constexpr int BW = 128;  // output features per tile (MMA M)
constexpr int BT = 128;  // tokens per tile (MMA N)
constexpr int BK = 128;  // K per stage: one 128-byte swizzled row of int8 codes
constexpr int UMMA_K = 32;
constexpr int B_STAGES = 6;
constexpr int W_STAGES = 8;   // packed-weight shared-memory ring
constexpr int A_STAGES = 4;   // TMEM A stages (even ones for group 0, odd ones for group 1)
constexpr int ACC_BUFS = 2;
constexpr int TMEM_COLS = 512;
constexpr int A_COL0 = ACC_BUFS * BT;  // A stages live after the accumulators
constexpr int B_STAGE_BYTES = BT * BK;
constexpr int W_STAGE_BYTES = BW * BK / 4;
constexpr int EPI_BUF_BYTES = 32 * 32 * 4;
constexpr uint32_t IDESC = idesc_i8_u8s8(BW, BT);
static_assert(A_COL0 + A_STAGES * (BK / 4) <= TMEM_COLS, "TMEM budget");
static_assert(A_STAGES % 2 == 0, "two producer groups take alternate stages");

constexpr int WARP_TMA = 0, WARP_MMA = 1, WARP_A0 = 4, WARP_EPI = 12, WARP_B4 = 16;
template <int BITS>
struct Threads {
    static constexpr int value = (BITS == 8 ? 16 : 20) * 32;
};

struct __align__(8) Barriers {
    uint64_t full_b[B_STAGES];
    uint64_t empty_b[B_STAGES];
    uint64_t full_w[W_STAGES];
    uint64_t empty_w[W_STAGES];
    uint64_t full_a[A_STAGES];
    uint64_t empty_a[A_STAGES];
    uint64_t acc_full[ACC_BUFS];
    uint64_t acc_empty[ACC_BUFS];
    uint64_t done;
    uint32_t tmem_base;
};

constexpr size_t OFF_B = 0;
constexpr size_t OFF_W = OFF_B + (size_t)B_STAGES * B_STAGE_BYTES;
constexpr size_t OFF_EPI = OFF_W + (size_t)W_STAGES * W_STAGE_BYTES;
constexpr size_t OFF_SCALE = OFF_EPI + 4 * 2 * EPI_BUF_BYTES;    // [4 warps][BT] floats
constexpr size_t OFF_RSUM = OFF_SCALE + 4 * BT * sizeof(float);  // [4 warps][BT] ints
constexpr size_t OFF_BAR = OFF_RSUM + 4 * BT * sizeof(int32_t);
constexpr size_t SMEM_BYTES = OFF_BAR + sizeof(Barriers) + 1024;  // + alignment slack

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast, __syncwarp orders the
// other lanes after the acquire (needed before warp-collective .sync.aligned tcgen05 ops).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, status);
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// Iteration `it` of this CTA's (tile, k-block) sequence.
__device__ __forceinline__ void iter_coords(int it, int KB, int &tile, int &kb) {
    const int t = it / KB;
    kb = it - t * KB;
    tile = blockIdx.x + t * gridDim.x;
}

template <int BITS, bool OUT_I32>
__global__ void __launch_bounds__(Threads<BITS>::value, 1)
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
    const int KB = K / BK;
    const int my_tiles =
        (int)blockIdx.x < num_tiles ? (num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int total = my_tiles * KB;  // (tile, k-block) iterations of this CTA

    if (threadIdx.x == 0) {
        for (int s = 0; s < B_STAGES; ++s) {
            mbar_init(&bar->full_b[s], BITS == 8 ? 1 : 4);
            mbar_init(&bar->empty_b[s], 1);
        }
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&bar->full_w[s], 1);
            mbar_init(&bar->empty_w[s], 4);
        }
        for (int s = 0; s < A_STAGES; ++s) {
            mbar_init(&bar->full_a[s], 4);
            mbar_init(&bar->empty_a[s], 1);
        }
        for (int s = 0; s < ACC_BUFS; ++s) {
            mbar_init(&bar->acc_full[s], 1);
            mbar_init(&bar->acc_empty[s], 4);
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
            for (int it = 0; it < total; ++it) {
                int tile, kb;
                iter_coords(it, KB, tile, kb);
                const int s_w = it % W_STAGES;
                const uint32_t p_w = (uint32_t)(it / W_STAGES) & 1;
                if (!mbar_wait(&bar->empty_w[s_w], p_w ^ 1, status)) break;
                mbar_arrive_expect_tx(&bar->full_w[s_w], W_STAGE_BYTES);
                tma_load_2d(sw + (size_t)s_w * W_STAGE_BYTES, &tmap_w, kb * (BK / 4),
                            (tile % n_wtiles) * BW, &bar->full_w[s_w]);
                issued_w |= 1u << s_w;
                ph_w = (ph_w & ~(1u << s_w)) | (p_w << s_w);
                if constexpr (BITS == 8) {
                    const int s_b = it % B_STAGES;
                    const uint32_t p_b = (uint32_t)(it / B_STAGES) & 1;
                    if (!mbar_wait(&bar->empty_b[s_b], p_b ^ 1, status)) break;
                    mbar_arrive_expect_tx(&bar->full_b[s_b], B_STAGE_BYTES);
                    tma_load_2d(sb + (size_t)s_b * B_STAGE_BYTES, &tmap_codes, kb * BK,
                                (tile / n_wtiles) * BT, &bar->full_b[s_b]);
                    issued_b |= 1u << s_b;
                    ph_b = (ph_b & ~(1u << s_b)) | (p_b << s_b);
                }
            }
            // no copy may still be writing shared memory when the CTA exits
            for (int t = 0; t < W_STAGES; ++t)
                if (issued_w & (1u << t)) mbar_wait(&bar->full_w[t], (ph_w >> t) & 1, status);
            for (int t = 0; t < B_STAGES; ++t)
                if (issued_b & (1u << t)) mbar_wait(&bar->full_b[t], (ph_b >> t) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t sb_addr = smem_addr(sb);
            bool ok = true;
            int it = 0;
            for (int t = 0; t < my_tiles && ok; ++t) {
                const int ab = t & 1;
                const uint32_t p_acc = (uint32_t)(t >> 1) & 1;
                if (!mbar_wait(&bar->acc_empty[ab], p_acc ^ 1, status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + ab * BT;
                for (int kb = 0; kb < KB; ++kb, ++it) {
                    const int s_a = it % A_STAGES, s_b = it % B_STAGES;
                    if (!mbar_wait(&bar->full_a[s_a], (uint32_t)(it / A_STAGES) & 1, status) ||
                        !mbar_wait(&bar->full_b[s_b], (uint32_t)(it / B_STAGES) & 1, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bdesc =
                        smem_desc_kmajor_sw128(sb_addr + (uint32_t)s_b * B_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        mma_i8_ts(d_tmem, tmem + A_COL0 + s_a * (BK / 4) + kk * (UMMA_K / 4),
                                  bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                                  (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&bar->empty_b[s_b]);
                    mma_commit(&bar->empty_a[s_a]);
                }
                if (!ok) break;
                mma_commit(&bar->acc_full[ab]);
            }
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
            const int s_w = it % W_STAGES, s_a = it % A_STAGES;
            if (!warp_wait(&bar->full_w[s_w], (uint32_t)(it / W_STAGES) & 1, status, lane)) break;
            const uint4 *src = reinterpret_cast<const uint4 *>(sw + (size_t)s_w * W_STAGE_BYTES +
                                                               rr * (BK / 4));
            const uint4 c0 = src[0], c1 = src[1];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->empty_w[s_w]);
            if (!warp_wait(&bar->empty_a[s_a], ((uint32_t)(it / A_STAGES) & 1) ^ 1, status, lane))
                break;
            tc_fence_after();
            const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
            uint32_t out[32];
#pragma unroll
            for (int g = 0; g < 8; ++g)
#pragma unroll
                for (int p = 0; p < 4; ++p) out[4 * g + p] = (w[g] >> (2 * p)) & 0x03030303u;
            tmem_st_32x32b_x32(t_lane + A_COL0 + s_a * (BK / 4), out);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->full_a[s_a]);
        }
    } else if (warp >= WARP_EPI && warp < WARP_EPI + 4) {
        // ------------------------------------------------------------------ epilogue
        const int wq = warp & 3;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        float *w_scale = s_scale + wq * BT;  // this warp's copy: no cross-warp barrier needed
        int32_t *w_rsum = s_rsum + wq * BT;
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
            for (int i = 0; i < BT / 32; ++i) {
                const int ml = i * 32 + lane;
                const int64_t m = (int64_t)mt * BT + ml;
                w_scale[ml] = m < M ? scales[m] * gamma : 0.f;
                w_rsum[ml] = m < M ? rowsum[m] : 0;
            }
            if (!warp_wait(&bar->acc_full[ab], (uint32_t)(t >> 1) & 1, status, lane)) break;
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < BT / 32; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_lane + ab * BT + ch * 32, v);
                tmem_wait_ld();
                uint8_t *stage = sepi + (size_t)(wq * 2 + buf) * EPI_BUF_BYTES;
                if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store is done
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
                        const float y0 = (float)((int)v[i] - w_rsum[m0]) * w_scale[m0];
                        const float y1 = (float)((int)v[i + 1] - w_rsum[m0 + 1]) * w_scale[m0 + 1];
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
                const int x0 = nw * BW + wq * 32, y0 = mt * BT + ch * 32;
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
    } else if (BITS == 4 && warp >= WARP_B4 && warp < WARP_B4 + 4) {
        // ------------------------------------------------------------------ INT4 B producer
        // warp w covers tokens 32w .. 32w+31 of the tile; in sub-step i, lane l loads the
        // 16-byte quarter (l % 4) of token 32w + 8i + l / 4: 8 tokens x 64 B per instruction,
        // fully used sectors.
        const int wq = warp & 3;
        const int q = lane & 3;
        for (int it = 0; it < total; ++it) {
            int tile, kb;
            iter_coords(it, KB, tile, kb);
            const int s_b = it % B_STAGES;
            uint4 raw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = wq * 32 + 8 * i + (lane >> 2);
                const int64_t m = (int64_t)(tile / n_wtiles) * BT + row;
                raw[i] = m < M ? ldg_nc_v4(codes4 + m * (K / 2) + kb * (BK / 2) + q * 16)
                               : make_uint4(0, 0, 0, 0);
            }
            if (!warp_wait(&bar->empty_b[s_b], ((uint32_t)(it / B_STAGES) & 1) ^ 1, status, lane))
                break;
            uint8_t *dst = sb + (size_t)s_b * B_STAGE_BYTES;
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
            if (lane == 0) mbar_arrive(&bar->full_b[s_b]);
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
    kern<<<grid, Threads<BITS>::value, SMEM_BYTES, stream>>>(
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
                  (uint64_t)a.M, (uint64_t)a.K, BK, BT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // packed weights: [N rows][K/4 bytes], one [128 x 32 B] box per stage
    if (encode_2d(encode_fn, &mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, (uint64_t)a.K / 4,
                  (uint64_t)a.N, (uint64_t)a.K / 4, BK / 4, BW,
                  CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
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
