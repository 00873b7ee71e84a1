// gemm_pair_ts.cu -- step 4 for prefill token counts on CTA pairs, with the unpacked weights in
// tensor memory: the ternary x integer product as tcgen05.mma.cta_group::2 with operand A read
// from tensor memory.
//
// 2B4T article, section 一.2 (W1.58A8: with ternary weights the product is additions and
// subtractions, exact in int32) and section 三.3 (GPU kernel: pack, store, load, unpack, compute).
// The weights are the MMA's M side and the tokens its N side:
//   D[feature, token] = sum_k u[feature, k] * c[token, k]    (u = q + 1 unsigned, c signed int8)
// accumulated in int32 in tensor memory; the per-token code sum removes the offset, so
// D - sum_k c = sum_k q * c exactly, and the epilogue applies the same fp32 rescale as every other
// product kernel of the library (Y = bf16_rn(float(acc) * (d_m * gamma))).
//
// Why this form.  The packed weights are expanded to int8 by ordinary warps.  Written to shared
// memory (as an SS-form operand) the expanded weights cost a 32 KB write and a 32 KB tensor-core
// read of shared memory per stage and CTA on top of the codes' own traffic; with INT4 codes,
// which are widened on chip too, that left the tensor pipe waiting on the operand pipeline
// (measured on B200: 69 % of the int8 roofline on the 7B down projection, against 84 % for
// INT8 codes, which land ready).  Written with tcgen05.st into tensor memory, where the MMA reads
// its A operand, the weights leave shared memory to the packed weights (8 KB per stage) and the
// tokens' codes, whose ring is then six stages deep.
//
// Tile: a pair computes 256 features x 256 tokens.  CTA r holds features 128r .. 128r+127 (its
// tensor-memory lanes, A and D rows) and tokens 128r .. 128r+127 of the B operand (the pair MMA
// reads both halves).  Tensor memory (512 columns): four A stages of 64 columns (K = 256 as 4
// int8 per column) at columns 0 .. 255 and one 256-column int32 accumulator at 256.  With one
// accumulator a tile's first MMA waits until the previous tile's epilogue has read the
// accumulator out (eight epilogue warps, each 128 tokens of one lane quadrant, release it after
// their last tcgen05.ld); two accumulators would leave no columns for the A stages, and
// 192-token tiles with two accumulators measured slower: the issuing thread pays the same
// ~50 cycles for a 256 x 192 x 32 MMA as for a 256 x 256 x 32 one.  Measured with clock64
// stamps on B200 (7B down projection): a steady 256-deep stage takes ~1500 cycles with the
// operands ready (~90 cycles of barrier tests per stage); the epilogue holds the accumulator
// ~4400 cycles per tile of ~96000.  What it took to get there: each epilogue warp keeps its
// tokens' (d_m * gamma, sum_k c) in a shared-memory table filled while the tile's MMAs run, read
// by broadcast (two shuffles per element before: ~10200 cycles), and the int -> fp32 and
// fp32 -> bf16 conversions, whose unit was the limit, are done on the FMA pipe and two at a time
// (~7700 cycles before), and the accumulator is read two chunks at a time, so that it is
// released after two of a warp's four chunks have been processed (~5400 cycles before).
//
// Warp roles (per CTA):
//   warp 0       code TMA: two [128 tokens x 128 B] boxes per 256-deep stage (INT8; the pair form
//                completes on the even CTA's barrier), or one box of packed nibbles into the
//                stage's second sub-tile (INT4), into a ring of C_STAGES stages;
//   warp 1       tensor-memory allocation (both CTAs); the even CTA's lane 0 issues the MMAs;
//   warp 2       packed-weight TMA: [128 features x 64 B] per stage (64-byte swizzle), a ring of
//                W_STAGES;
//   warps 4-7    unpack: warp w owns tensor-memory lanes 32(w%4) .. +31 (features): 64 packed
//                bytes -> 64 columns of int8 lanes with one shift-and-mask per four weights,
//                tcgen05.st into the A stage;
//   warps 8-15   epilogue: thread = feature, tokens 128 ((w-8)/4) .. +127 of the tile, read 64
//                at a time (tcgen05.ld), then offset, scale, activation and stores 32 at a time
//                (a warp store covers 32 consecutive features of one token);
//   warps 16-19  INT4 only: widen the stage's packed codes in place, thread = token row.
// Every mbarrier wait is bounded (~1 s, then BITNET_ERR_TIMEOUT and the kernel winds down).  No
// TMA multicast is used.
#include "common.cuh"
#include "kernels.h"

#include <cudaTypedefs.h>
#include <string.h>

namespace bitnet {
namespace pts {

constexpr int BF = 256;                 // features per pair tile (MMA M)
constexpr int HF = BF / 2;              // features per CTA (tensor-memory lanes)
constexpr int BT = 256;                 // tokens per pair tile (MMA N)
constexpr int HT = BT / 2;              // tokens of the B operand held by one CTA
constexpr int BK = 256;                 // K per stage
constexpr int SUBK = 128;               // K per code sub-tile: one 128-byte swizzled row
constexpr int UMMA_K = 32;              // K per kind::i8 MMA
constexpr int C_STAGES = 6;             // code stages in flight
constexpr int W_STAGES = 3;             // packed-weight tiles in flight
constexpr int A_STAGES = 4;             // unpacked weight stages in tensor memory, K = 256 each
constexpr int A_COLS = BK / 4;          // 64 columns per A stage
constexpr int ACC_COL = A_STAGES * A_COLS;  // the accumulator's first column
constexpr int TMEM_COLS = 512;
constexpr int SUB_BYTES = HT * SUBK;            // 16 KB: [128 rows x 128 B]
constexpr int C_STAGE_BYTES = 2 * SUB_BYTES;    // 24 KB of codes per CTA and stage
constexpr int W_STAGE_BYTES = HF * BK / 4;      // 8 KB of packed weights per CTA and stage
constexpr uint32_t IDESC = idesc_i8_u8s8(BF, BT);
static_assert(ACC_COL + BT <= TMEM_COLS, "tensor-memory budget");
static_assert(SUB_BYTES % 1024 == 0, "swizzle atoms of whole sub-tiles");

constexpr int WARP_CTMA = 0, WARP_MMA = 1, WARP_WTMA = 2, WARP_UNPACK = 4, UNPACK_WARPS = 4;
constexpr int WARP_EPI = 8, EPI_WARPS = 8, WARP_WIDEN = 16, WIDEN_WARPS = HT / 32;

enum OutMode { OUT_ACC = 0, OUT_BF16 = 1, OUT_RELU2 = 2, OUT_SWIGLU = 3 };

template <int BITS>
constexpr int num_threads() {
    return (BITS == 4 ? WARP_WIDEN + WIDEN_WARPS : WARP_EPI + EPI_WARPS) * 32;
}

struct __align__(8) Barriers {
    uint64_t c_full[C_STAGES];    // even CTA: INT8 the four code boxes' bytes; INT4 the widening
                                  // warps of both CTAs
    uint64_t c_empty[C_STAGES];   // both: the MMAs that read the code stage have completed
    uint64_t c_packed[C_STAGES];  // local, INT4: the stage's packed codes have landed
    uint64_t w_full[W_STAGES];    // local packed-weight ring
    uint64_t w_empty[W_STAGES];   // local: this CTA's unpack warps have read the slot
    uint64_t a_full[A_STAGES];    // even CTA: the stage's unpack warps of both CTAs stored it
    uint64_t a_empty[A_STAGES];   // both: the MMAs that read the A stage have completed
    uint64_t acc_full;            // both
    uint64_t acc_empty;           // even CTA: the epilogue warps of both CTAs
    uint64_t done;                // both: every MMA has completed
    uint32_t tmem_base;
};

// Shared memory, identical offsets in both CTAs (the pair MMA addresses the peer's codes by the
// even CTA's offsets).
constexpr size_t OFF_C = 0;
constexpr size_t OFF_W = OFF_C + (size_t)C_STAGES * C_STAGE_BYTES;
// per epilogue warp: (d_m * gamma, sum_k c) of its 128 tokens of the current tile
constexpr size_t OFF_TOK = OFF_W + (size_t)W_STAGES * W_STAGE_BYTES;
constexpr size_t OFF_BAR = OFF_TOK + (size_t)EPI_WARPS * (BT / 2) * 8;
constexpr size_t SMEM_BYTES = OFF_BAR + sizeof(Barriers) + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared-memory budget");

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast, __syncwarp orders the other
// lanes after the acquire.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, int *status, int lane) {
    bool ok = true;
    if (lane == 0) ok = mbar_wait(bar, parity, status);
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// D (+)= A[tmem] x B[smem]^T on a CTA pair, kind::i8: A rows in both CTAs' tensor memory at the
// same address, B rows split between their shared memories at the same offset.
__device__ __forceinline__ void mma_i8_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int BITS, int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(num_threads<BITS>(), 1)
    ternary_gemm_pair_ts_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                                const __grid_constant__ CUtensorMap tmap_w, void *__restrict__ Yout,
                                const float *__restrict__ scales,
                                const int32_t *__restrict__ rowsum,
                                const float *__restrict__ gamma_ptr, int M, int N, int K,
                                int *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sc = smem + OFF_C;
    uint8_t *sw = smem + OFF_W;
    Barriers *bar = reinterpret_cast<Barriers *>(smem + OFF_BAR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int n_ftiles = (N + BF - 1) / BF;
    const int n_ttiles = (M + BT - 1) / BT;
    const int num_tiles = n_ftiles * n_ttiles;
    const int KS = (K + BK - 1) / BK;  // stages per tile (the last one may be half)
    const int my_tiles = pair < num_tiles ? (num_tiles - 1 - pair) / npairs + 1 : 0;
    const int total = my_tiles * KS;  // (tile, stage) iterations of this pair

    if (threadIdx.x == 0) {
        for (int s = 0; s < C_STAGES; ++s) {
            // INT8: the even CTA's expect-tx arrival; INT4: the widening warps of both CTAs
            mbar_init(&bar->c_full[s], BITS == 8 ? 1 : 2 * WIDEN_WARPS);
            mbar_init(&bar->c_empty[s], 1);
            mbar_init(&bar->c_packed[s], 1);
        }
        for (int s = 0; s < W_STAGES; ++s) {
            mbar_init(&bar->w_full[s], 1);
            mbar_init(&bar->w_empty[s], UNPACK_WARPS);
        }
        for (int s = 0; s < A_STAGES; ++s) {
            mbar_init(&bar->a_full[s], 2 * UNPACK_WARPS);  // one warp per quadrant, both CTAs
            mbar_init(&bar->a_empty[s], 1);
        }
        mbar_init(&bar->acc_full, 1);
        mbar_init(&bar->acc_empty, 2 * EPI_WARPS);
        mbar_init(&bar->done, 1);
        fence_mbar_init();
    }
    if (warp == WARP_CTMA && lane == 0) {
        prefetch_tensormap(&tmap_codes);
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
    // the set-up above overlaps the tail of the kernel that produced the codes (programmatic
    // dependent launch); nothing is read from global memory before this point
    pdl_wait();

    if (warp == WARP_CTMA) {
        // ------------------------------------------------------------------ code TMA
        if (lane == 0) {
            uint32_t issued = 0, ph = 0;
            int s = 0;
            uint32_t p = 0;
            for (int it = 0; it < total; ++it) {
                const int tile = pair + (it / KS) * npairs;
                const int ks = it % KS;
                const int t0 = (tile / n_ftiles) * BT + (int)rank * HT;
                if (!mbar_wait(&bar->c_empty[s], p ^ 1, status)) break;
                uint8_t *dst = sc + (size_t)s * C_STAGE_BYTES;
                if constexpr (BITS == 8) {
                    if (leader) mbar_arrive_expect_tx(&bar->c_full[s], 4 * SUB_BYTES);
                    const uint32_t fb = mapa_shared(smem_addr(&bar->c_full[s]), 0);
                    tma_load_2d_pair(dst, &tmap_codes, ks * BK, t0, fb);
                    tma_load_2d_pair(dst + SUB_BYTES, &tmap_codes, ks * BK + SUBK, t0, fb);
                } else {
                    // the stage's packed nibbles (128 B per token) into its second sub-tile,
                    // widened in place by the widening warps
                    mbar_arrive_expect_tx(&bar->c_packed[s], SUB_BYTES);
                    tma_load_2d(dst + SUB_BYTES, &tmap_codes, ks * (BK / 2), t0, &bar->c_packed[s]);
                }
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
                if (++s == C_STAGES) { s = 0; p ^= 1; }
            }
            // no copy may still be writing shared memory when the CTA exits: wait until the
            // loads have been consumed (or give up after the time limit)
            for (int i = 0; i < C_STAGES; ++i)
                if (issued & (1u << i)) mbar_wait(&bar->c_empty[i], (ph >> i) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_WTMA) {
        // ------------------------------------------------------------------ weight-tile TMA
        if (lane == 0) {
            uint32_t issued = 0, ph = 0;
            int s = 0;
            uint32_t p = 0;
            for (int it = 0; it < total; ++it) {
                const int tile = pair + (it / KS) * npairs;
                const int ks = it % KS;
                if (!mbar_wait(&bar->w_empty[s], p ^ 1, status)) break;
                mbar_arrive_expect_tx(&bar->w_full[s], W_STAGE_BYTES);
                tma_load_2d(sw + (size_t)s * W_STAGE_BYTES, &tmap_w, ks * (BK / 4),
                            (tile % n_ftiles) * BF + (int)rank * HF, &bar->w_full[s]);
                issued |= 1u << s;
                ph = (ph & ~(1u << s)) | (p << s);
                if (++s == W_STAGES) { s = 0; p ^= 1; }
            }
            for (int i = 0; i < W_STAGES; ++i)
                if (issued & (1u << i)) mbar_wait(&bar->w_full[i], (ph >> i) & 1, status);
        }
        __syncwarp();
    } else if (warp == WARP_MMA) {
        // ------------------------------------------------------------------ MMA issuer
        if (leader && lane == 0) {
            const uint32_t sc_addr = smem_addr(sc);
            int cs = 0, as = 0;
            uint32_t cp = 0, ap = 0;
            for (int it = 0; it < total; ++it) {
                const int t = it / KS, ks = it % KS;
                // one accumulator: a tile's first MMA waits until the previous tile's epilogue
                // has read it out
                if (ks == 0 && !mbar_wait(&bar->acc_empty, ((uint32_t)t & 1) ^ 1, status)) break;
                if (!mbar_wait(&bar->a_full[as], ap, status)) break;
                if (!mbar_wait(&bar->c_full[cs], cp, status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + ACC_COL;
                const uint32_t a_tmem = tmem + as * A_COLS;
                const uint32_t c_st = sc_addr + (uint32_t)cs * C_STAGE_BYTES;
#pragma unroll
                for (int sub = 0; sub < 2; ++sub) {
                    const uint64_t bdesc = smem_desc_kmajor_sw128(c_st + sub * SUB_BYTES);
#pragma unroll
                    for (int kk = 0; kk < SUBK / UMMA_K; ++kk)
                        mma_i8_ts_pair(d_tmem, a_tmem + (uint32_t)(sub * (SUBK / 4) + kk * (UMMA_K / 4)),
                                       bdesc + (uint64_t)(kk * UMMA_K / 16), IDESC,
                                       (ks != 0 || sub != 0 || kk != 0) ? 1u : 0u);
                }
                mma_commit_pair(&bar->c_empty[cs], 3);
                mma_commit_pair(&bar->a_empty[as], 3);
                if (ks == KS - 1) mma_commit_pair(&bar->acc_full, 3);
                if (++cs == C_STAGES) { cs = 0; cp ^= 1; }
                if (++as == A_STAGES) { as = 0; ap ^= 1; }
            }
            // every MMA issued above has finished before either CTA releases tensor memory
            mma_commit_pair(&bar->done, 3);
        }
        if (lane == 0) mbar_wait(&bar->done, 0, status);
        __syncwarp();
    } else if (warp >= WARP_UNPACK && warp < WARP_UNPACK + UNPACK_WARPS) {
        // ------------------------------------------------------------------ weight unpack
        const int quad = warp & 3;                    // tensor-memory lanes 32 quad .. +31
        const int rr = quad * 32 + lane;              // feature row of this CTA's half
        const int sx = (rr >> 1) & 3;                 // 64-byte swizzle of the packed tile
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        for (int it = 0; it < total; ++it) {
            const int s_w = it % W_STAGES, as = it % A_STAGES;
            if (!warp_wait(&bar->w_full[s_w], (uint32_t)(it / W_STAGES) & 1, status, lane)) break;
            // row rr of the packed tile: 64 B, 16-byte chunk c stored at chunk c ^ sx
            const uint8_t *wrow = sw + (size_t)s_w * W_STAGE_BYTES + rr * (BK / 4);
            uint4 v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                v[c] = *reinterpret_cast<const uint4 *>(wrow + ((c ^ sx) << 4));
            // the refill is an async-proxy write: each lane's plain reads are fenced before the
            // slot is released
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->w_empty[s_w]);
            if (!warp_wait(&bar->a_empty[as], ((uint32_t)(it / A_STAGES) & 1) ^ 1, status, lane))
                break;
            tc_fence_after();
            // word g of the row holds k = 16g .. 16g+15; (w >> 2p) & 0x03030303 is k = 16g+4p ..
            // +3, i.e. column 4g + p of the A stage
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w[8] = {v[2 * h].x, v[2 * h].y, v[2 * h].z, v[2 * h].w,
                                       v[2 * h + 1].x, v[2 * h + 1].y, v[2 * h + 1].z, v[2 * h + 1].w};
                uint32_t o[32];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    o[4 * g] = w[g] & 0x03030303u;
                    o[4 * g + 1] = (w[g] >> 2) & 0x03030303u;
                    o[4 * g + 2] = (w[g] >> 4) & 0x03030303u;
                    o[4 * g + 3] = (w[g] >> 6) & 0x03030303u;
                }
                tmem_st_32x32b_x32(t_lane + (uint32_t)(as * A_COLS + 32 * h), o);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->a_full[as]), 0));
        }
    } else if (warp >= WARP_EPI && warp < WARP_EPI + EPI_WARPS) {
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;                    // tensor-memory lanes = features
        const int eh = (warp - WARP_EPI) >> 2;        // tokens 128 eh .. +127 of the tile
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const float gamma = *gamma_ptr;
        constexpr int CHUNKS = BT / 2 / 32;
        float2 *tok = reinterpret_cast<float2 *>(smem + OFF_TOK) + (warp - WARP_EPI) * (BT / 2);
        // |sum_k q c| <= 128 K (INT8) or 8 K (INT4): below 2^22 the exact FMA-pipe conversion
        // applies (always for the shapes this kernel takes)
        const bool small_acc = (int64_t)K * (BITS == 8 ? 128 : 8) < (int64_t(1) << 22);
        for (int t = 0; t < my_tiles; ++t) {
            const int tile = pair + t * npairs;
            const int nf = tile % n_ftiles, mt = tile / n_ftiles;
            const int n = nf * BF + (int)rank * HF + quad * 32 + lane;  // this thread's feature
            // the warp's token table, filled while the tile's MMAs run: every element then reads
            // its token's scale and code sum with one broadcast shared-memory load
            __syncwarp();  // the previous tile's reads of the table are done
#pragma unroll
            for (int q = 0; q < CHUNKS; ++q) {
                const int mj = mt * BT + eh * (BT / 2) + q * 32 + lane;
                tok[q * 32 + lane] = make_float2(mj < M ? scales[mj] * gamma : 0.f,
                                                 __int_as_float(mj < M ? rowsum[mj] : 0));
            }
            __syncwarp();
            if (!warp_wait(&bar->acc_full, (uint32_t)t & 1, status, lane)) break;
            tc_fence_after();
            // one chunk (32 tokens) of the accumulator, read into v: offset, scale, activation,
            // stores
            auto process = [&](int ch, const uint32_t (&v)[32]) {
                const int m0 = mt * BT + eh * (BT / 2) + ch * 32;  // first token of the chunk
                if (m0 >= M) return;
                if constexpr (MODE == OUT_ACC) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + j;
                        const int a = (int)v[j] - __float_as_int(tok[ch * 32 + j].y);
                        if (m < M && n < N) reinterpret_cast<int32_t *>(Yout)[(int64_t)m * N + n] = a;
                    }
                } else {
                    // The conversion unit (~16 per clock per SM on B200) set the epilogue's pace
                    // with an int -> fp32 and an fp32 -> bf16 conversion per element: the first
                    // is done exactly on the FMA pipe (|a| < 2^22: the fp32 with bit pattern
                    // 0x4B400000 + a is 1.5 * 2^23 + a), the second two tokens at a time.
                    const bool glu = MODE == OUT_SWIGLU;
                    const bool store = glu ? (lane & 1) == 0 && n < N : n < N;
                    const int64_t ld = glu ? N / 2 : N;
                    unsigned short *yp = reinterpret_cast<unsigned short *>(Yout) +
                                         (int64_t)m0 * ld + (glu ? n / 2 : n);
                    const int rows = store ? min(M - m0, 32) : 0;
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float y[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float2 tk = tok[ch * 32 + j + e];
                            const int a = (int)v[j + e] - __float_as_int(tk.y);
                            const float af = small_acc ? __fsub_rn(__int_as_float(0x4B400000 + a), 12582912.f)
                                                       : (float)a;
                            y[e] = af * tk.x;
                            if constexpr (MODE == OUT_RELU2) y[e] = y[e] > 0.f ? y[e] * y[e] : 0.f;
                            if constexpr (MODE == OUT_SWIGLU) {
                                // features 2p (gate) and 2p + 1 (up) sit in lanes 2p, 2p + 1; the
                                // even lane keeps silu(gate) * up
                                const float up = __shfl_xor_sync(0xFFFFFFFFu, y[e], 1);
                                y[e] = __fdiv_rn(y[e], 1.f + expf(-y[e])) * up;
                            }
                        }
                        const __nv_bfloat162 h = __floats2bfloat162_rn(y[0], y[1]);
                        const uint32_t hw = *reinterpret_cast<const uint32_t *>(&h);
                        if (j < rows) *yp = (unsigned short)(hw & 0xFFFFu);
                        yp += ld;
                        if (j + 1 < rows) *yp = (unsigned short)(hw >> 16);
                        yp += ld;
                    }
                }
            };
            // chunks are read two at a time (64 registers), so the accumulator is released after
            // two chunks have been processed rather than three
#pragma unroll 1
            for (int cp = 0; cp < CHUNKS; cp += 2) {
                uint32_t va[32], vb[32];
                tmem_ld_32x32b_x32(t_lane + (uint32_t)(ACC_COL + eh * (BT / 2) + cp * 32), va);
                tmem_ld_32x32b_x32(t_lane + (uint32_t)(ACC_COL + eh * (BT / 2) + cp * 32 + 32), vb);
                tmem_wait_ld();
                if (cp + 2 == CHUNKS) {
                    // the accumulator is read out: the next tile's MMAs may start
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->acc_empty), 0));
                }
                process(cp, va);
                process(cp + 1, vb);
            }
        }
    } else if (BITS == 4 && warp >= WARP_WIDEN && warp < WARP_WIDEN + WIDEN_WARPS) {
        // ------------------------------------------------------------------ INT4 code widening
        // thread = token row of this CTA's half: its 128 packed bytes (256 codes) sit in the
        // stage's second sub-tile; it reads them all, then writes 256 int8 codes over both
        // sub-tiles (the row's own 128-byte slots, so no other thread's input is overwritten)
        const int row = (warp - WARP_WIDEN) * 32 + lane;
        const int sx = row & 7;
        for (int it = 0; it < total; ++it) {
            const int s = it % C_STAGES;
            if (!warp_wait(&bar->c_packed[s], (uint32_t)(it / C_STAGES) & 1, status, lane)) break;
            uint8_t *crow = sc + (size_t)s * C_STAGE_BYTES + row * SUBK;
            uint4 raw[8];
#pragma unroll
            for (int c = 0; c < 8; ++c)
                raw[c] = *reinterpret_cast<const uint4 *>(crow + SUB_BYTES + ((c ^ sx) << 4));
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                // 32 codes k = 32c .. 32c+31 -> 16-byte chunks 2c (words x, y) and 2c+1 (z, w)
                const uint32_t wd[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint4 o;
                    o.x = sext_nibbles(wd[2 * h] & 0x0F0F0F0Fu);
                    o.y = sext_nibbles((wd[2 * h] >> 4) & 0x0F0F0F0Fu);
                    o.z = sext_nibbles(wd[2 * h + 1] & 0x0F0F0F0Fu);
                    o.w = sext_nibbles((wd[2 * h + 1] >> 4) & 0x0F0F0F0Fu);
                    const int oc = 2 * c + h;  // chunk of the 256-byte row: sub-tile oc / 8
                    *reinterpret_cast<uint4 *>(crow + (oc >> 3) * SUB_BYTES + (((oc & 7) ^ sx) << 4)) = o;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bar->c_full[s]), 0));
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

// Co-resident pairs per device (one pair per two SMs where the GPU's layout allows it), looked up
// once per device and kernel instance.
template <int BITS, int MODE>
static int max_pairs(int num_sms) {
    static int cache[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_sms & ~1), 1, 1);
    cfg.blockDim = dim3(num_threads<BITS>(), 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, ternary_gemm_pair_ts_kernel<BITS, MODE>, &cfg) !=
            cudaSuccess ||
        clusters < 1) {
        (void)cudaGetLastError();
        clusters = num_sms / 2;
    }
    if (dev >= 0 && dev < 64) cache[dev] = clusters;
    return clusters;
}

template <int BITS, int MODE>
static cudaError_t launch_t(const GemmArgs &a, const CUtensorMap &mc, const CUtensorMap &mw,
                            void *out, int64_t tiles, int num_sms, cudaStream_t stream) {
    auto kern = ternary_gemm_pair_ts_kernel<BITS, MODE>;
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
    cfg.blockDim = dim3(num_threads<BITS>(), 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, mc, mw, out, a.scales, a.rowsum, a.gamma, (int)a.M,
                              (int)a.N, (int)a.K, a.status);
}

}  // namespace pts

cudaError_t launch_ternary_gemm_pair_ts(const GemmArgs &a, void *encode_fn, int num_sms,
                                        cudaStream_t stream, int *launches) {
    using namespace pts;
    const int64_t tiles = ((a.N + BF - 1) / BF) * ((a.M + BT - 1) / BT);
    CUtensorMap mc, mw;
    memset(&mc, 0, sizeof mc);
    memset(&mw, 0, sizeof mw);
    // codes: INT8 [M rows][K bytes], two [96 tokens x 128 B] boxes per CTA and stage; INT4
    // [M rows][K/2 bytes], one [96 tokens x 128 B] box of packed nibbles; 128-byte swizzle
    const uint64_t cb = a.act_bits == 8 ? (uint64_t)a.K : (uint64_t)a.K / 2;
    if (encode_tmap_2d(encode_fn, &mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, cb, (uint64_t)a.M,
                       cb, SUBK, HT, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // packed weights: [N rows][K/4 bytes], one [128 features x 64 B] box per stage, 64-byte
    // swizzle
    if (encode_tmap_2d(encode_fn, &mw, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, (uint64_t)a.K / 4,
                       (uint64_t)a.N, (uint64_t)a.K / 4, BK / 4, HF,
                       CU_TENSOR_MAP_SWIZZLE_64B) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (launches) *launches = (a.Y ? 1 : 0) + (a.acc ? 1 : 0);
    if (a.Y) {
        switch (a.activation * 2 + (a.act_bits == 8 ? 1 : 0)) {
            case 0: e = launch_t<4, OUT_BF16>(a, mc, mw, a.Y, tiles, num_sms, stream); break;
            case 1: e = launch_t<8, OUT_BF16>(a, mc, mw, a.Y, tiles, num_sms, stream); break;
            case 2: e = launch_t<4, OUT_RELU2>(a, mc, mw, a.Y, tiles, num_sms, stream); break;
            case 3: e = launch_t<8, OUT_RELU2>(a, mc, mw, a.Y, tiles, num_sms, stream); break;
            case 4: e = launch_t<4, OUT_SWIGLU>(a, mc, mw, a.Y, tiles, num_sms, stream); break;
            case 5: e = launch_t<8, OUT_SWIGLU>(a, mc, mw, a.Y, tiles, num_sms, stream); break;
            default: return cudaErrorInvalidValue;
        }
        if (e != cudaSuccess) return e;
    }
    if (a.acc) {
        e = a.act_bits == 8 ? launch_t<8, OUT_ACC>(a, mc, mw, a.acc, tiles, num_sms, stream)
                            : launch_t<4, OUT_ACC>(a, mc, mw, a.acc, tiles, num_sms, stream);
    }
    return e;
}

}  // namespace bitnet
