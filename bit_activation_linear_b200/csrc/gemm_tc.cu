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
// 128.  Roles of the 13 warps of a persistent CTA (one per SM):
//   warps 0-3   B producer.  INT8 codes: one thread issues TMA loads of [128 tokens x 128 B]
//               with the 128-byte swizzle straight into the UMMA K-major layout.  INT4 codes:
//               all 128 threads load one token's 64 bytes each, sign-extend the nibbles to
//               int8 in registers and store them in the same swizzled layout.
//   warps 4-7   A producer.  Thread i owns output feature n0 + i (= TMEM lane i): it loads the
//               32 bytes of packed weights of a stage, expands each 2-bit offset code
//               u = q + 1 to a byte with one shift-and-mask per four weights, and writes the 32
//               words into TMEM with tcgen05.st.  The weights never touch shared memory.
//   warp 12     MMA issuer: tcgen05.mma.kind::i8 with A from TMEM (unsigned bytes u) and B
//               from shared memory (signed codes c), D += u * c in TMEM; tcgen05.commit frees
//               the stages and publishes finished accumulators.
//   warps 8-11  epilogue: tcgen05.ld of the int32 accumulator, subtract the token's code sum
//               (sum_k q*c = sum_k u*c - sum_k c), scale by d_m * gamma, round to bf16, stage in
//               shared memory and TMA-store.  Two accumulators in TMEM let the epilogue of one
//               tile overlap the main loop of the next.
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
constexpr int A_STAGES = 4;
constexpr int ACC_BUFS = 2;
constexpr int TMEM_COLS = 512;
constexpr int A_COL0 = ACC_BUFS * BT;  // A stages live after the accumulators
constexpr int NUM_WARPS = 13;
constexpr int NUM_THREADS = NUM_WARPS * 32;
constexpr int B_STAGE_BYTES = BT * BK;
constexpr int EPI_BUF_BYTES = 32 * 32 * 4;
constexpr uint32_t IDESC = idesc_i8_u8s8(BW, BT);
static_assert(A_COL0 + A_STAGES * (BK / 4) <= TMEM_COLS, "TMEM budget");

struct __align__(8) Barriers {
    uint64_t full_b[B_STAGES];
    uint64_t empty_b[B_STAGES];
    uint64_t full_a[A_STAGES];
    uint64_t empty_a[A_STAGES];
    uint64_t acc_full[ACC_BUFS];
    uint64_t acc_empty[ACC_BUFS];
    uint64_t done;
    uint32_t tmem_base;
};

constexpr size_t OFF_B = 0;
constexpr size_t OFF_EPI = OFF_B + (size_t)B_STAGES * B_STAGE_BYTES;
constexpr size_t OFF_SCALE = OFF_EPI + 4 * 2 * EPI_BUF_BYTES;  // [4 warps][BT] floats
constexpr size_t OFF_RSUM = OFF_SCALE + 4 * BT * sizeof(float);  // [4 warps][BT] ints
constexpr size_t OFF_BAR = OFF_RSUM + 4 * BT * sizeof(int32_t);
constexpr int PREFETCH = 4;  // producer register ring depth (stages in flight per thread)
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
__global__ void __launch_bounds__(NUM_THREADS, 1)
    ternary_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                           const __grid_constant__ CUtensorMap tmap_out,
                           const uint8_t *__restrict__ codes4, const uint4 *__restrict__ wp,
                           const float *__restrict__ scales, const int32_t *__restrict__ rowsum,
                           const float *__restrict__ gamma_ptr, int M, int N, int K,
                           int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sb = smem + OFF_B;
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

    if (threadIdx.x == 0) {
        for (int s = 0; s < B_STAGES; ++s) {
            mbar_init(&bar->full_b[s], BITS == 8 ? 1 : 4);
            mbar_init(&bar->empty_b[s], 1);
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
    if (warp == 0 && lane == 0) {
        if (BITS == 8) prefetch_tensormap(&tmap_codes);
        prefetch_tensormap(&tmap_out);
    }
    if (warp == 12) {
        tmem_alloc(&bar->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp < 4) {
        // ------------------------------------------------------------------ B producer
        if constexpr (BITS == 8) {
            if (warp == 0 && lane == 0) {
                int s = 0;
                uint32_t ph = 0;
                uint32_t issued = 0, issued_ph = 0;  // per-stage bits, for the final drain
                bool ok = true;
                for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                    const int mt = tile / n_wtiles;
                    for (int kb = 0; kb < KB; ++kb) {
                        if (!mbar_wait(&bar->empty_b[s], ph ^ 1, status)) { ok = false; break; }
                        mbar_arrive_expect_tx(&bar->full_b[s], B_STAGE_BYTES);
                        tma_load_2d(sb + (size_t)s * B_STAGE_BYTES, &tmap_codes, kb * BK, mt * BT,
                                    &bar->full_b[s]);
                        issued |= 1u << s;
                        issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                        if (++s == B_STAGES) { s = 0; ph ^= 1; }
                    }
                }
                // no copy may still be writing shared memory when the CTA exits
                for (int t = 0; t < B_STAGES; ++t)
                    if (issued & (1u << t)) mbar_wait(&bar->full_b[t], (issued_ph >> t) & 1, status);
            }
        } else {
            // INT4: thread i loads token i of the tile (64 bytes per stage), unpacks to int8
            const int rr = warp * 32 + lane;
            const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
            const int total = my_tiles * KB;
            auto fetch = [&](int it, uint4 (&dst)[4]) {
                if (it < total) {
                    int tile, kb;
                    iter_coords(it, KB, tile, kb);
                    const int64_t m = (int64_t)(tile / n_wtiles) * BT + rr;
                    if (m < M) {
                        const uint4 *src = reinterpret_cast<const uint4 *>(codes4 + m * (K / 2)) + 4 * kb;
#pragma unroll
                        for (int i = 0; i < 4; ++i) dst[i] = ldg_nc_v4(src + i);
                        return;
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(0, 0, 0, 0);
            };
            uint4 ring[PREFETCH][4];
#pragma unroll
            for (int u = 0; u < PREFETCH - 1; ++u) fetch(u, ring[u]);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int it0 = 0; it0 < total && ok; it0 += PREFETCH) {
#pragma unroll
                for (int u = 0; u < PREFETCH; ++u) {
                    const int it = it0 + u;
                    if (it >= total || !ok) break;
                    fetch(it + PREFETCH - 1, ring[(u + PREFETCH - 1) % PREFETCH]);
                    if (!warp_wait(&bar->empty_b[s], ph ^ 1, status, lane)) { ok = false; break; }
                    uint8_t *dst = sb + (size_t)s * B_STAGE_BYTES + rr * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {  // 16 codes k = 16c .. 16c+15
                        const uint4 v = ring[u][c >> 1];
                        const uint32_t w0 = (c & 1) ? v.z : v.x;
                        const uint32_t w1 = (c & 1) ? v.w : v.y;
                        uint4 o;
                        o.x = sext_nibbles(w0 & 0x0F0F0F0Fu);
                        o.y = sext_nibbles((w0 >> 4) & 0x0F0F0F0Fu);
                        o.z = sext_nibbles(w1 & 0x0F0F0F0Fu);
                        o.w = sext_nibbles((w1 >> 4) & 0x0F0F0F0Fu);
                        *reinterpret_cast<uint4 *>(dst + ((c ^ (rr & 7)) << 4)) = o;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar->full_b[s]);
                    if (++s == B_STAGES) { s = 0; ph ^= 1; }
                }
            }
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------------ A producer
        const int wq = warp - 4;  // TMEM lanes 32*wq .. 32*wq+31
        const int rr = wq * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        const int total = my_tiles * KB;
        auto fetch = [&](int it, uint4 (&dst)[2]) {
            if (it < total) {
                int tile, kb;
                iter_coords(it, KB, tile, kb);
                const int64_t n = (int64_t)(tile % n_wtiles) * BW + rr;
                if (n < N) {
                    const uint4 *src = wp + n * (K / 64) + 2 * kb;
                    dst[0] = ldg_nc_v4(src);
                    dst[1] = ldg_nc_v4(src + 1);
                    return;
                }
            }
            dst[0] = make_uint4(0, 0, 0, 0);
            dst[1] = make_uint4(0, 0, 0, 0);
        };
        uint4 ring[PREFETCH][2];
#pragma unroll
        for (int u = 0; u < PREFETCH - 1; ++u) fetch(u, ring[u]);
        int sa = 0;
        uint32_t pha = 0;
        bool ok = true;
        for (int it0 = 0; it0 < total && ok; it0 += PREFETCH) {
#pragma unroll
            for (int u = 0; u < PREFETCH; ++u) {
                const int it = it0 + u;
                if (it >= total || !ok) break;
                fetch(it + PREFETCH - 1, ring[(u + PREFETCH - 1) % PREFETCH]);
                if (!warp_wait(&bar->empty_a[sa], pha ^ 1, status, lane)) { ok = false; break; }
                tc_fence_after();
                const uint32_t w[8] = {ring[u][0].x, ring[u][0].y, ring[u][0].z, ring[u][0].w,
                                       ring[u][1].x, ring[u][1].y, ring[u][1].z, ring[u][1].w};
                uint32_t out[32];
#pragma unroll
                for (int g = 0; g < 8; ++g)
#pragma unroll
                    for (int p = 0; p < 4; ++p) out[4 * g + p] = (w[g] >> (2 * p)) & 0x03030303u;
                tmem_st_32x32b_x32(t_lane + A_COL0 + sa * (BK / 4), out);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar->full_a[sa]);
                if (++sa == A_STAGES) { sa = 0; pha ^= 1; }
            }
        }
    } else if (warp < 12) {
        // ------------------------------------------------------------------ epilogue
        const int wq = warp - 8;
        const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
        float *w_scale = s_scale + wq * BT;  // this warp's copy: no cross-warp barrier needed
        int32_t *w_rsum = s_rsum + wq * BT;
        const float gamma = *gamma_ptr;
        int ab = 0;
        uint32_t phacc = 0;
        int buf = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int nw = tile % n_wtiles;
            const int mt = tile / n_wtiles;
            __syncwarp();  // the previous tile's scales are no longer read
#pragma unroll
            for (int i = 0; i < BT / 32; ++i) {
                const int ml = i * 32 + lane;
                const int64_t m = (int64_t)mt * BT + ml;
                w_scale[ml] = m < M ? scales[m] * gamma : 0.f;
                w_rsum[ml] = m < M ? rowsum[m] : 0;
            }
            if (!warp_wait(&bar->acc_full[ab], phacc, status, lane)) break;
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < BT / 32; ++ch) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(t_lane + ab * BT + ch * 32, v);
                tmem_wait_ld();
                uint8_t *stage = sepi + (size_t)(wq * 2 + buf) * EPI_BUF_BYTES;
                if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store is done
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int ml = ch * 32 + i;
                    const int a = (int)v[i] - w_rsum[ml];
                    if constexpr (OUT_I32) {
                        reinterpret_cast<int32_t *>(stage)[i * 32 + lane] = a;
                    } else {
                        reinterpret_cast<__nv_bfloat16 *>(stage)[i * 32 + lane] =
                            __float2bfloat16_rn((float)a * w_scale[ml]);
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
            if (++ab == ACC_BUFS) { ab = 0; phacc ^= 1; }
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0, sa = 0, ab = 0;
            uint32_t ph = 0, pha = 0, phacc = 0;
            bool ok = true;
            const uint32_t sb_addr = smem_addr(sb);
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(&bar->acc_empty[ab], phacc ^ 1, status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + ab * BT;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(&bar->full_a[sa], pha, status) ||
                        !mbar_wait(&bar->full_b[s], ph, status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bdesc =
                        smem_desc_kmajor_sw128(sb_addr + (uint32_t)s * B_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        mma_i8_ts(d_tmem, tmem + A_COL0 + sa * (BK / 4) + kk * (UMMA_K / 4),
                                  bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                                  (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&bar->empty_b[s]);
                    mma_commit(&bar->empty_a[sa]);
                    if (++s == B_STAGES) { s = 0; ph ^= 1; }
                    if (++sa == A_STAGES) { sa = 0; pha ^= 1; }
                }
                if (!ok) break;
                mma_commit(&bar->acc_full[ab]);
                if (++ab == ACC_BUFS) { ab = 0; phacc ^= 1; }
            }
            // every MMA issued above has finished before TMEM is released
            mma_commit(&bar->done);
            mbar_wait(&bar->done, 0, status);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int BITS, bool OUT_I32>
static cudaError_t launch_tc_t(const GemmArgs &a, const CUtensorMap &mc, const CUtensorMap &mo,
                               int grid, cudaStream_t stream) {
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
        mc, mo, reinterpret_cast<const uint8_t *>(a.codes), reinterpret_cast<const uint4 *>(a.Wp),
        a.scales, a.rowsum, a.gamma, (int)a.M, (int)a.N, (int)a.K, a.status);
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
    CUtensorMap mc, mo;
    memset(&mc, 0, sizeof mc);
    memset(&mo, 0, sizeof mo);
    if (a.act_bits == 8) {
        if (encode_2d(encode_fn, &mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, (uint64_t)a.K,
                      (uint64_t)a.M, (uint64_t)a.K, BK, BT,
                      CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaSuccess;
    if (a.Y) {
        if (encode_2d(encode_fn, &mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Y, (uint64_t)a.N,
                      (uint64_t)a.M, (uint64_t)a.N * 2, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        e = a.act_bits == 8 ? launch_tc_t<8, false>(a, mc, mo, grid, stream)
                            : launch_tc_t<4, false>(a, mc, mo, grid, stream);
        if (e != cudaSuccess) return e;
    }
    if (a.acc) {
        if (encode_2d(encode_fn, &mo, CU_TENSOR_MAP_DATA_TYPE_INT32, a.acc, (uint64_t)a.N,
                      (uint64_t)a.M, (uint64_t)a.N * 4, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        e = a.act_bits == 8 ? launch_tc_t<8, true>(a, mc, mo, grid, stream)
                            : launch_tc_t<4, true>(a, mc, mo, grid, stream);
    }
    return e;
}

}  // namespace bitnet
