// api.cu -- the extern "C" entry points declared in include/bitnet.h: argument checks, the
// per-device state (SM count, status word, tensor-map encoder), workspace layout and the
// choice between the decode and the tensor-core product kernels.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

using namespace bitnet;

__device__ int g_device_status;  // one status word per device (module global)

thread_local char g_last_error[512] = "";
std::atomic<uint64_t> g_launches{0};

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return code;
}

struct DeviceState {
    bool ready = false;
    int status_code = BITNET_OK;
    int num_sms = 0;
    int *status_word = nullptr;
};

constexpr int kMaxDevices = 64;
DeviceState g_dev[kMaxDevices];
std::mutex g_mutex;
void *g_encode = nullptr;

// Per-device set-up on first use: must be an sm_100 device; fetch the address of the status
// word (a host-side symbol name is not a device address) and the SM count.
int device_state(DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(BITNET_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(BITNET_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState &st = g_dev[dev];
    if (!st.ready) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0)
            return fail(BITNET_ERR_UNSUPPORTED,
                        "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                        minor);
        e = cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail(BITNET_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
        e = cudaGetSymbolAddress(reinterpret_cast<void **>(&st.status_word), g_device_status);
        if (e != cudaSuccess)
            return fail(BITNET_ERR_CUDA, "status word address: %s", cudaGetErrorString(e));
        if (!g_encode) {
            cudaDriverEntryPointQueryResult q;
            e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &g_encode, cudaEnableDefault,
                                        &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !g_encode) {
                g_encode = nullptr;
                return fail(BITNET_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
            }
        }
        st.ready = true;
    }
    *out = &st;
    return BITNET_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

int check_shape(int64_t M, int64_t K, int64_t N, bool need_m, bool need_n) {
    if (need_m && M < 1) return fail(BITNET_ERR_INVALID, "M = %lld must be >= 1", (long long)M);
    if (K < 128 || K % 128 != 0)
        return fail(BITNET_ERR_INVALID, "K = %lld must be a positive multiple of 128",
                    (long long)K);
    if (need_n && (N < 8 || N % 8 != 0))
        return fail(BITNET_ERR_INVALID, "N = %lld must be a positive multiple of 8", (long long)N);
    if (M > (int64_t)INT32_MAX || N > (int64_t)INT32_MAX || K > (1 << 20))
        return fail(BITNET_ERR_UNSUPPORTED, "sizes beyond the supported range");
    return BITNET_OK;
}

int log2_exact(int64_t K) {
    int l = 0;
    while ((int64_t(1) << l) < K) ++l;
    return (int64_t(1) << l) == K ? l : -1;
}

int launched(cudaError_t e, int count, const char *what) {
    if (e != cudaSuccess)
        return fail(BITNET_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
    g_launches.fetch_add((uint64_t)count, std::memory_order_relaxed);
    return BITNET_OK;
}

int act_quant_impl(DeviceState *st, const void *X, int64_t M, int64_t K, int hadamard,
                   int act_bits, void *codes, float *scales, int32_t *rowsum, float *zout,
                   cudaStream_t stream, const NormArgs &nrm = NormArgs()) {
    if (hadamard) {
        const int lk = log2_exact(K);
        if (lk < 7 || lk > 15)
            return fail(BITNET_ERR_UNSUPPORTED,
                        "H-BitLinear needs K to be a power of two in [128, 32768], got %lld",
                        (long long)K);
        if (!nrm.on && hadamard_tc_supported(lk))
            return launched(launch_hadamard_tc(X, M, lk, act_bits, codes, scales, rowsum, zout,
                                               st->status_word, g_encode, st->num_sms, stream),
                            1, "hadamard_tc");
        return launched(launch_fwht_quant(X, M, lk, act_bits, nrm, codes, scales, rowsum, zout,
                                          st->status_word, stream),
                        1, "fwht_quant");
    }
    return launched(launch_act_quant_plain(X, M, K, act_bits, nrm, codes, scales, rowsum, zout,
                                           stream),
                    1, "act_quant_plain");
}

int gemm_impl(DeviceState *st, const void *codes, const float *scales, const int32_t *rowsum,
              int64_t M, int64_t K, const void *Wp, const float *gamma, int64_t N, int act_bits,
              int32_t *acc, void *Y, cudaStream_t stream, bool early_weights = false,
              int activation = 0) {
    GemmArgs a;
    a.codes = codes;
    a.scales = scales;
    a.rowsum = rowsum;
    a.Wp = reinterpret_cast<const uint32_t *>(Wp);
    a.gamma = gamma;
    a.M = M;
    a.N = N;
    a.K = K;
    a.act_bits = act_bits;
    a.acc = acc;
    a.Y = Y;
    a.status = st->status_word;
    a.early_weights = early_weights;
    a.activation = activation;
    if (M <= kGemvMaxTokens) return launched(launch_ternary_gemv(a, stream), 1, "ternary_gemv");
    if (M <= kSkinnyMaxTokens)
        return launched(launch_ternary_gemm_skinny(a, g_encode, stream), 1, "ternary_gemm_skinny");
    int n = 0;
    if (use_pair_ts(act_bits, K)) {
        // INT4 codes are widened on chip; with the weights unpacked into tensor memory that
        // widening no longer shares shared memory with the unpacked weights
        const cudaError_t e = launch_ternary_gemm_pair_ts(a, g_encode, st->num_sms, stream, &n);
        return launched(e, n, "ternary_gemm_pair_ts");
    }
    const cudaError_t e = launch_ternary_gemm_tc(a, g_encode, st->num_sms, stream, &n);
    return launched(e, n, "ternary_gemm_tc");
}

int forward_impl(const void *X, int64_t M, int64_t K, const void *Wp, const float *gamma,
                 int64_t N, int act_bits, void *Y, void *ws, size_t ws_bytes, int hadamard,
                 cudaStream_t stream, const NormArgs &nrm = NormArgs(), int activation = 0,
                 bool absmax4 = false) {
    int rc = check_shape(M, K, N, true, true);
    if (rc) return rc;
    if (act_bits != 8 && act_bits != 4)
        return fail(BITNET_ERR_INVALID, "act_bits = %d must be 8 or 4", act_bits);
    if (!X || !Wp || !gamma || !Y || !ws)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X) || !aligned16(Wp) || !aligned16(Y) || !aligned16(ws))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    const size_t need = bitnet_workspace_bytes(M, K, N, act_bits);
    if (ws_bytes < need)
        return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    uint8_t *w = static_cast<uint8_t *>(ws);
    void *codes = w;
    float *scales = reinterpret_cast<float *>(w + round256(bitnet_act_codes_bytes(M, K, act_bits)));
    int32_t *rowsum = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(scales) +
                                                  round256((size_t)M * sizeof(float)));
    if ((rc = act_quant_impl(st, X, M, K, hadamard, absmax4 ? kActInt4Absmax : act_bits, codes,
                             scales, rowsum, nullptr, stream, nrm)))
        return rc;
    // the quantiser above was launched in stream order after whatever wrote Wp
    return gemm_impl(st, codes, scales, rowsum, M, K, Wp, gamma, N, act_bits, nullptr, Y, stream,
                     true, activation);
}

}  // namespace

extern "C" {

const char *bitnet_status_string(int status) {
    switch (status) {
        case BITNET_OK: return "ok";
        case BITNET_ERR_INVALID: return "invalid argument";
        case BITNET_ERR_UNSUPPORTED: return "unsupported shape or device";
        case BITNET_ERR_CUDA: return "CUDA error";
        case BITNET_ERR_TIMEOUT: return "device wait timed out";
        case BITNET_ERR_WORKSPACE: return "workspace too small";
        default: return "unknown status";
    }
}

const char *bitnet_last_error(void) { return g_last_error; }

uint64_t bitnet_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t bitnet_packed_weight_bytes(int64_t N, int64_t K) {
    return (N > 0 && K > 0) ? (size_t)N * (size_t)K / 4 : 0;
}

size_t bitnet_weight_workspace_bytes(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return 0;
    return round256((size_t)absmean_num_partials(N * K) * sizeof(double));
}

int bitnet_quantize_pack_weights(const void *W_dev, int64_t N, int64_t K, void *Wp_dev,
                                 float *gamma_dev, void *ws_dev, size_t ws_bytes,
                                 bitnet_stream_t stream) {
    int rc = check_shape(1, K, N, false, true);
    if (rc) return rc;
    if (!W_dev || !Wp_dev || !gamma_dev || !ws_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(W_dev) || !aligned16(Wp_dev) || !aligned16(ws_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    const size_t need = bitnet_weight_workspace_bytes(N, K);
    if (ws_bytes < need)
        return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    const int64_t n = N * K;
    const int P = absmean_num_partials(n);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    double *partials = static_cast<double *>(ws_dev);
    if ((rc = launched(launch_absmean_partials(W_dev, n, partials, P, s), 1, "absmean_partials")))
        return rc;
    return launched(launch_ternarize_pack(W_dev, n, partials, P,
                                          static_cast<uint32_t *>(Wp_dev), gamma_dev, s),
                    1, "ternarize_pack");
}

int bitnet_quantize_pack_weights_noalloc(const void *W_dev, int64_t N, int64_t K, void *Wp_dev,
                                         float *gamma_dev, bitnet_stream_t stream) {
    int rc = check_shape(1, K, N, false, true);
    if (rc) return rc;
    if (!W_dev || !Wp_dev || !gamma_dev) return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(W_dev) || !aligned16(Wp_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    double *scratch = nullptr;
    size_t scratch_bytes = 0;
    cudaError_t e = noalloc_partials_address(&scratch, &scratch_bytes);
    if (e != cudaSuccess)
        return fail(BITNET_ERR_CUDA, "scratch address: %s", cudaGetErrorString(e));
    const int64_t n = N * K;
    const int P = absmean_num_partials(n);
    if ((size_t)P * sizeof(double) > scratch_bytes)
        return fail(BITNET_ERR_UNSUPPORTED,
                    "%d partial sums need %zu bytes of scratch; the fixed scratch holds %zu", P,
                    (size_t)P * sizeof(double), scratch_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // every partial is written before it is read: the scratch needs no clearing
    if ((rc = launched(launch_absmean_partials(W_dev, n, scratch, P, s), 1, "absmean_partials")))
        return rc;
    return launched(launch_ternarize_pack(W_dev, n, scratch, P, static_cast<uint32_t *>(Wp_dev),
                                          gamma_dev, s),
                    1, "ternarize_pack");
}

size_t bitnet_act_codes_bytes(int64_t M, int64_t K, int act_bits) {
    if (M <= 0 || K <= 0) return 0;
    return act_bits == 4 ? (size_t)M * (size_t)K / 2 : (size_t)M * (size_t)K;
}

int bitnet_act_quant(const void *X_dev, int64_t M, int64_t K, int hadamard, int act_bits,
                     void *codes_dev, float *scales_dev, int32_t *rowsum_dev,
                     bitnet_stream_t stream) {
    int rc = check_shape(M, K, 8, true, false);
    if (rc) return rc;
    if (act_bits != 8 && act_bits != 4)
        return fail(BITNET_ERR_INVALID, "act_bits = %d must be 8 or 4", act_bits);
    if (!X_dev || !codes_dev || !scales_dev || !rowsum_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X_dev) || !aligned16(codes_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return act_quant_impl(st, X_dev, M, K, hadamard, act_bits, codes_dev, scales_dev, rowsum_dev,
                          nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int bitnet_fwht_f32(const void *X_dev, int64_t M, int64_t K, float *Z_dev,
                    bitnet_stream_t stream) {
    int rc = check_shape(M, K, 8, true, false);
    if (rc) return rc;
    if (!X_dev || !Z_dev) return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X_dev) || !aligned16(Z_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return act_quant_impl(st, X_dev, M, K, 1, 8, nullptr, nullptr, nullptr, Z_dev,
                          reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {
int norm_args(const void *gain_dev, float eps, NormArgs *out) {
    if (!(eps > 0.f) || !std::isfinite(eps))
        return fail(BITNET_ERR_INVALID, "eps = %g must be finite and > 0", (double)eps);
    if (gain_dev && !aligned16(gain_dev))
        return fail(BITNET_ERR_INVALID, "the norm gain must be 16-byte aligned");
    out->on = true;
    out->gain = gain_dev;
    out->eps = eps;
    return BITNET_OK;
}
}  // namespace

extern "C" {

int bitnet_act_quant_norm(const void *X_dev, int64_t M, int64_t K, const void *norm_gain_dev,
                          float eps, int hadamard, int act_bits, void *codes_dev,
                          float *scales_dev, int32_t *rowsum_dev, bitnet_stream_t stream) {
    int rc = check_shape(M, K, 8, true, false);
    if (rc) return rc;
    if (act_bits != 8 && act_bits != 4)
        return fail(BITNET_ERR_INVALID, "act_bits = %d must be 8 or 4", act_bits);
    if (!X_dev || !codes_dev || !scales_dev || !rowsum_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X_dev) || !aligned16(codes_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    NormArgs nrm;
    if ((rc = norm_args(norm_gain_dev, eps, &nrm))) return rc;
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return act_quant_impl(st, X_dev, M, K, hadamard, act_bits, codes_dev, scales_dev, rowsum_dev,
                          nullptr, reinterpret_cast<cudaStream_t>(stream), nrm);
}

int bitnet_norm_transform_f32(const void *X_dev, int64_t M, int64_t K, const void *norm_gain_dev,
                              float eps, int hadamard, float *Z_dev, bitnet_stream_t stream) {
    int rc = check_shape(M, K, 8, true, false);
    if (rc) return rc;
    if (!X_dev || !Z_dev) return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X_dev) || !aligned16(Z_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    NormArgs nrm;
    if ((rc = norm_args(norm_gain_dev, eps, &nrm))) return rc;
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return act_quant_impl(st, X_dev, M, K, hadamard, 8, nullptr, nullptr, nullptr, Z_dev,
                          reinterpret_cast<cudaStream_t>(stream), nrm);
}

int bitnet_norm_bitlinear_forward(const void *X_dev, int64_t M, int64_t K,
                                  const void *norm_gain_dev, float eps, int hadamard,
                                  const void *Wp_dev, const float *gamma_dev, int64_t N,
                                  int act_bits, void *Y_dev, void *ws_dev, size_t ws_bytes,
                                  bitnet_stream_t stream) {
    NormArgs nrm;
    int rc = norm_args(norm_gain_dev, eps, &nrm);
    if (rc) return rc;
    return forward_impl(X_dev, M, K, Wp_dev, gamma_dev, N, act_bits, Y_dev, ws_dev, ws_bytes,
                        hadamard ? 1 : 0, reinterpret_cast<cudaStream_t>(stream), nrm);
}

}  // extern "C"

namespace {
int check_activation(int activation, int64_t N) {
    if (activation != BITNET_ACT_RELU2 && activation != BITNET_ACT_SWIGLU)
        return fail(BITNET_ERR_INVALID, "activation = %d must be %d (squared ReLU) or %d (SwiGLU)",
                    activation, (int)BITNET_ACT_RELU2, (int)BITNET_ACT_SWIGLU);
    if (activation == BITNET_ACT_SWIGLU && N % 16 != 0)
        return fail(BITNET_ERR_INVALID, "SwiGLU needs N %% 16 == 0, got N = %lld", (long long)N);
    return BITNET_OK;
}
}  // namespace

extern "C" {

int bitnet_ternary_gemm_act(const void *codes_dev, const float *scales_dev,
                            const int32_t *rowsum_dev, int64_t M, int64_t K, const void *Wp_dev,
                            const float *gamma_dev, int64_t N, int act_bits, int activation,
                            void *Y_dev, bitnet_stream_t stream) {
    int rc = check_shape(M, K, N, true, true);
    if (rc) return rc;
    if ((rc = check_activation(activation, N))) return rc;
    if (act_bits != 8 && act_bits != 4)
        return fail(BITNET_ERR_INVALID, "act_bits = %d must be 8 or 4", act_bits);
    if (!codes_dev || !scales_dev || !rowsum_dev || !Wp_dev || !gamma_dev || !Y_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(codes_dev) || !aligned16(Wp_dev) || !aligned16(Y_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return gemm_impl(st, codes_dev, scales_dev, rowsum_dev, M, K, Wp_dev, gamma_dev, N, act_bits,
                     nullptr, Y_dev, reinterpret_cast<cudaStream_t>(stream), false, activation);
}

int bitnet_bitlinear_forward_act(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                                 const float *gamma_dev, int64_t N, int act_bits, int hadamard,
                                 int activation, void *Y_dev, void *ws_dev, size_t ws_bytes,
                                 bitnet_stream_t stream) {
    int rc = check_activation(activation, N);
    if (rc) return rc;
    return forward_impl(X_dev, M, K, Wp_dev, gamma_dev, N, act_bits, Y_dev, ws_dev, ws_bytes,
                        hadamard ? 1 : 0, reinterpret_cast<cudaStream_t>(stream), NormArgs(),
                        activation);
}

int bitnet_ternary_gemm(const void *codes_dev, const float *scales_dev,
                        const int32_t *rowsum_dev, int64_t M, int64_t K, const void *Wp_dev,
                        const float *gamma_dev, int64_t N, int act_bits, int32_t *acc_dev,
                        void *Y_dev, bitnet_stream_t stream) {
    int rc = check_shape(M, K, N, true, true);
    if (rc) return rc;
    if (act_bits != 8 && act_bits != 4)
        return fail(BITNET_ERR_INVALID, "act_bits = %d must be 8 or 4", act_bits);
    if (!codes_dev || !scales_dev || !rowsum_dev || !Wp_dev || !gamma_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!acc_dev && !Y_dev) return fail(BITNET_ERR_INVALID, "neither acc nor Y requested");
    if (!aligned16(codes_dev) || !aligned16(Wp_dev) || (acc_dev && !aligned16(acc_dev)) ||
        (Y_dev && !aligned16(Y_dev)))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return gemm_impl(st, codes_dev, scales_dev, rowsum_dev, M, K, Wp_dev, gamma_dev, N, act_bits,
                     acc_dev, Y_dev, reinterpret_cast<cudaStream_t>(stream));
}

int bitnet_product_plan(int64_t M, int64_t K, int64_t N, int act_bits, int *path,
                        int *k_split) {
    int rc = check_shape(M, K, N, true, true);
    if (rc) return rc;
    if (act_bits != 8 && act_bits != 4)
        return fail(BITNET_ERR_INVALID, "act_bits = %d must be 8 or 4", act_bits);
    if (!path || !k_split) return fail(BITNET_ERR_INVALID, "null pointer argument");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    if (M <= kGemvMaxTokens) {
        *path = BITNET_PATH_DECODE;
        *k_split = 1;
        return BITNET_OK;
    }
    if (M <= kSkinnyMaxTokens) {
        *path = BITNET_PATH_TC_SKINNY;
        *k_split = ternary_gemm_skinny_split(N, K);
        return BITNET_OK;
    }
    *path = use_pair_ts(act_bits, K) ? BITNET_PATH_TC_TMEM : BITNET_PATH_TC;
    *k_split = 1;
    return BITNET_OK;
}

int bitnet_act_quant_plan(int64_t K, int hadamard, int norm, int *path) {
    int rc = check_shape(1, K, 8, false, false);
    if (rc) return rc;
    if (!path) return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!hadamard) {
        *path = BITNET_QUANT_PLAIN;
        return BITNET_OK;
    }
    const int lk = log2_exact(K);
    if (lk < 7 || lk > 15)
        return fail(BITNET_ERR_UNSUPPORTED,
                    "H-BitLinear needs K to be a power of two in [128, 32768], got %lld",
                    (long long)K);
    *path = !norm && hadamard_tc_supported(lk) ? BITNET_QUANT_HADAMARD_TC : BITNET_QUANT_FWHT;
    return BITNET_OK;
}

size_t bitnet_workspace_bytes(int64_t M, int64_t K, int64_t N, int act_bits) {
    (void)N;
    if (M <= 0 || K <= 0) return 0;
    return round256(bitnet_act_codes_bytes(M, K, act_bits)) + round256((size_t)M * 4) +
           round256((size_t)M * 4);
}

int bitnet_bitlinear_forward(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                             const float *gamma_dev, int64_t N, int act_bits, void *Y_dev,
                             void *ws_dev, size_t ws_bytes, bitnet_stream_t stream) {
    return forward_impl(X_dev, M, K, Wp_dev, gamma_dev, N, act_bits, Y_dev, ws_dev, ws_bytes, 0,
                        reinterpret_cast<cudaStream_t>(stream));
}

int bitnet_hbitlinear_forward(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                              const float *gamma_dev, int64_t N, int act_bits, void *Y_dev,
                              void *ws_dev, size_t ws_bytes, bitnet_stream_t stream) {
    return forward_impl(X_dev, M, K, Wp_dev, gamma_dev, N, act_bits, Y_dev, ws_dev, ws_bytes, 1,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t bitnet_weight_workspace_bytes_rotated(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return 0;
    return round256((size_t)N * (size_t)K * sizeof(float)) + bitnet_weight_workspace_bytes(N, K);
}

int bitnet_quantize_pack_weights_rotated(const void *W_dev, int64_t N, int64_t K, void *Wp_dev,
                                         float *gamma_dev, void *ws_dev, size_t ws_bytes,
                                         bitnet_stream_t stream) {
    int rc = check_shape(N, K, 8, true, false);  // N rows are transformed like M token rows
    if (rc) return rc;
    if (N % 8 != 0)
        return fail(BITNET_ERR_INVALID, "N = %lld must be a positive multiple of 8", (long long)N);
    if (!W_dev || !Wp_dev || !gamma_dev || !ws_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(W_dev) || !aligned16(Wp_dev) || !aligned16(ws_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    const size_t need = bitnet_weight_workspace_bytes_rotated(N, K);
    if (ws_bytes < need)
        return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float *rot = static_cast<float *>(ws_dev);
    double *partials = reinterpret_cast<double *>(static_cast<uint8_t *>(ws_dev) +
                                                  round256((size_t)N * (size_t)K * sizeof(float)));
    // the rotated rows W' = W H / sqrt(K): the transform of the activation path, on weight rows
    if ((rc = act_quant_impl(st, W_dev, N, K, 1, 8, nullptr, nullptr, nullptr, rot, s)))
        return rc;
    const int P = absmean_num_partials(N * K);
    return launched(launch_ternarize_pack_f32(rot, N * K, partials, P,
                                              static_cast<uint32_t *>(Wp_dev), gamma_dev, s),
                    2, "ternarize_pack_f32");
}

int bitnet_act_quant_absmax4(const void *X_dev, int64_t M, int64_t K, int hadamard,
                              void *codes_dev, float *scales_dev, int32_t *rowsum_dev,
                              bitnet_stream_t stream) {
    int rc = check_shape(M, K, 8, true, false);
    if (rc) return rc;
    if (!X_dev || !codes_dev || !scales_dev || !rowsum_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X_dev) || !aligned16(codes_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return act_quant_impl(st, X_dev, M, K, hadamard ? 1 : 0, kActInt4Absmax, codes_dev,
                          scales_dev, rowsum_dev, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

int bitnet_bitlinear_forward_absmax4(const void *X_dev, int64_t M, int64_t K, const void *Wp_dev,
                                      const float *gamma_dev, int64_t N, int hadamard, void *Y_dev,
                                      void *ws_dev, size_t ws_bytes, bitnet_stream_t stream) {
    return forward_impl(X_dev, M, K, Wp_dev, gamma_dev, N, 4, Y_dev, ws_dev, ws_bytes,
                        hadamard ? 1 : 0, reinterpret_cast<cudaStream_t>(stream), NormArgs(), 0,
                        true);
}

size_t bitnet_base3_weight_bytes(int64_t N, int64_t K) {
    return (N > 0 && K > 0) ? (size_t)N * (size_t)((K + 19) / 20) * 4 : 0;
}

int bitnet_quantize_pack_weights_base3(const void *W_dev, int64_t N, int64_t K, void *Wp3_dev,
                                       float *gamma_dev, void *ws_dev, size_t ws_bytes,
                                       bitnet_stream_t stream) {
    int rc = check_shape(1, K, N, false, true);
    if (rc) return rc;
    if (!W_dev || !Wp3_dev || !gamma_dev || !ws_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(W_dev) || !aligned16(Wp3_dev) || !aligned16(ws_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    const size_t need = bitnet_weight_workspace_bytes(N, K);
    if (ws_bytes < need)
        return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    const int P = absmean_num_partials(N * K);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    double *partials = static_cast<double *>(ws_dev);
    if ((rc = launched(launch_absmean_partials(W_dev, N * K, partials, P, s), 1,
                       "absmean_partials")))
        return rc;
    return launched(launch_ternarize_pack_base3(W_dev, N, K, partials, P,
                                                static_cast<uint32_t *>(Wp3_dev), gamma_dev, s),
                    1, "ternarize_pack_base3");
}

}  // extern "C"

namespace {
int check_base3(int64_t M, int64_t K, int64_t N, int activation) {
    int rc = check_shape(M, K, N, true, true);
    if (rc) return rc;
    if (M > kGemvMaxTokens)
        return fail(BITNET_ERR_UNSUPPORTED, "base-3 weights serve M <= %d tokens, got M = %lld",
                    kGemvMaxTokens, (long long)M);
    if (activation != 0) return check_activation(activation, N);
    return BITNET_OK;
}

int gemv_base3_impl(DeviceState *st, const void *codes, const float *scales,
                    const int32_t *rowsum, int64_t M, int64_t K, const void *Wp3,
                    const float *gamma, int64_t N, int activation, int32_t *acc, void *Y,
                    bool early_weights, cudaStream_t stream) {
    GemmArgs a;
    a.codes = codes;
    a.scales = scales;
    a.rowsum = rowsum;
    a.Wp = reinterpret_cast<const uint32_t *>(Wp3);
    a.gamma = gamma;
    a.M = M;
    a.N = N;
    a.K = K;
    a.act_bits = 8;
    a.acc = acc;
    a.Y = Y;
    a.status = st->status_word;
    a.early_weights = early_weights;
    a.activation = activation;
    return launched(launch_ternary_gemv_base3(a, stream), 1, "ternary_gemv_base3");
}
}  // namespace

extern "C" {

int bitnet_ternary_gemv_base3(const void *codes_dev, const float *scales_dev,
                              const int32_t *rowsum_dev, int64_t M, int64_t K,
                              const void *Wp3_dev, const float *gamma_dev, int64_t N,
                              int activation, int32_t *acc_dev, void *Y_dev,
                              bitnet_stream_t stream) {
    int rc = check_base3(M, K, N, activation);
    if (rc) return rc;
    if (!codes_dev || !scales_dev || !rowsum_dev || !Wp3_dev || !gamma_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!acc_dev && !Y_dev) return fail(BITNET_ERR_INVALID, "neither acc nor Y requested");
    if (acc_dev && activation != 0)
        return fail(BITNET_ERR_INVALID, "acc is the product before the activation: pass "
                                        "activation 0 with acc");
    if (!aligned16(codes_dev) || !aligned16(Wp3_dev) || (acc_dev && !aligned16(acc_dev)) ||
        (Y_dev && !aligned16(Y_dev)))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    return gemv_base3_impl(st, codes_dev, scales_dev, rowsum_dev, M, K, Wp3_dev, gamma_dev, N,
                           activation, acc_dev, Y_dev, false,
                           reinterpret_cast<cudaStream_t>(stream));
}

int bitnet_bitlinear_forward_base3(const void *X_dev, int64_t M, int64_t K, const void *Wp3_dev,
                                   const float *gamma_dev, int64_t N, int hadamard,
                                   int activation, void *Y_dev, void *ws_dev, size_t ws_bytes,
                                   bitnet_stream_t stream) {
    int rc = check_base3(M, K, N, activation);
    if (rc) return rc;
    if (!X_dev || !Wp3_dev || !gamma_dev || !Y_dev || !ws_dev)
        return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X_dev) || !aligned16(Wp3_dev) || !aligned16(Y_dev) || !aligned16(ws_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    const size_t need = bitnet_workspace_bytes(M, K, N, 8);
    if (ws_bytes < need)
        return fail(BITNET_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
    DeviceState *st = nullptr;
    if ((rc = device_state(&st))) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *w = static_cast<uint8_t *>(ws_dev);
    float *scales = reinterpret_cast<float *>(w + round256(bitnet_act_codes_bytes(M, K, 8)));
    int32_t *rowsum = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(scales) +
                                                  round256((size_t)M * sizeof(float)));
    if ((rc = act_quant_impl(st, X_dev, M, K, hadamard ? 1 : 0, 8, w, scales, rowsum, nullptr,
                             s)))
        return rc;
    // the quantiser was launched in stream order after whatever wrote Wp3
    return gemv_base3_impl(st, w, scales, rowsum, M, K, Wp3_dev, gamma_dev, N, activation,
                           nullptr, Y_dev, true, s);
}

size_t bitnet_state_codes_bytes(int64_t M, int64_t C, int bits) {
    if (M <= 0 || C <= 0 || bits < 2 || bits > 8) return 0;
    return (size_t)M * (size_t)C * (size_t)bits / 8;
}

int bitnet_quant_states(const void *X_dev, int64_t M, int64_t C, int64_t group, int bits,
                        void *codes_dev, float *scales_dev, bitnet_stream_t stream) {
    if (M < 1 || M > (int64_t)INT32_MAX)
        return fail(BITNET_ERR_INVALID, "M = %lld must be in 1 .. 2^31-1", (long long)M);
    if (group < 32 || group % 32 != 0 || group > (1 << 20))
        return fail(BITNET_ERR_INVALID, "group = %lld must be a positive multiple of 32",
                    (long long)group);
    if (C < group || C % group != 0 || C > (1 << 24))
        return fail(BITNET_ERR_INVALID, "C = %lld must be a multiple of group = %lld",
                    (long long)C, (long long)group);
    if (bits < 2 || bits > 8) return fail(BITNET_ERR_INVALID, "bits = %d must be in 2 .. 8", bits);
    if (!X_dev || !codes_dev || !scales_dev) return fail(BITNET_ERR_INVALID, "null pointer argument");
    if (!aligned16(X_dev) || !aligned16(codes_dev))
        return fail(BITNET_ERR_INVALID, "device pointers must be 16-byte aligned");
    DeviceState *st = nullptr;
    int rc = device_state(&st);
    if (rc) return rc;
    return launched(launch_quant_states(X_dev, M, C, group, bits, codes_dev, scales_dev,
                                        reinterpret_cast<cudaStream_t>(stream)),
                    1, "quant_states");
}

int bitnet_selftest_wait_timeout(int64_t limit_cycles, bitnet_stream_t stream) {
    if (limit_cycles < 1 || limit_cycles > kWaitLimitCycles)
        return fail(BITNET_ERR_INVALID, "limit_cycles = %lld must be in 1 .. %lld",
                    (long long)limit_cycles, (long long)kWaitLimitCycles);
    DeviceState *st = nullptr;
    int rc = device_state(&st);
    if (rc) return rc;
    return launched(launch_selftest_wait_timeout((long long)limit_cycles, st->status_word,
                                                 reinterpret_cast<cudaStream_t>(stream)),
                    1, "selftest_wait_timeout");
}

int bitnet_sync_status(bitnet_stream_t stream) {
    DeviceState *st = nullptr;
    int rc = device_state(&st);
    if (rc) return rc;
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return fail(BITNET_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
    int word = 0;
    e = cudaMemcpy(&word, st->status_word, sizeof word, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(BITNET_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (word != 0) {
        const int zero = 0;
        cudaMemcpy(st->status_word, &zero, sizeof zero, cudaMemcpyHostToDevice);
        return fail(word, "a kernel reported: %s", bitnet_status_string(word));
    }
    return BITNET_OK;
}

}  // extern "C"
