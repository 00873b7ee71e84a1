"""CPU oracle for the BitLinear / H-BitLinear forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this package.  The product library never does: it shares no
code with the oracle, and its Python binding fails loudly instead of falling back here.

The arithmetic lives in ``bitnet_oracle.c`` (plain loops, double precision, int64
accumulation); this module compiles it with gcc on first use and wraps it with numpy.  Each
wrapper names the page and section whose step it states; the readings taken where the pages
print no formula are listed at the top of the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bitnet_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# -ffp-contract=off keeps every product and sum a separately rounded IEEE operation.
CFLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile ``bitnet_oracle.c`` into ``liboracle.so`` next to it (gcc + OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            L = ctypes.CDLL(path)
            i64, vp, f32, f64, i32 = (ctypes.c_int64, ctypes.c_void_p, ctypes.c_float,
                                      ctypes.c_double, ctypes.c_int)
            sig = {
                "oracle_double_to_bf16": (ctypes.c_uint16, [f64]),
                "oracle_bf16_to_double": (f64, [ctypes.c_uint16]),
                "oracle_num_threads": (i32, []),
                "oracle_abs_sum_bf16": (f64, [vp, i64]),
                "oracle_absmean_gamma": (f32, [vp, i64]),
                "oracle_ternarize": (None, [vp, i64, f32, vp]),
                "oracle_absmean_gamma_f32": (f32, [vp, i64]),
                "oracle_ternarize_f32": (None, [vp, i64, f32, vp]),
                "oracle_pack_ternary": (None, [vp, i64, i64, vp]),
                "oracle_unpack_ternary": (i64, [vp, i64, i64, vp]),
                "oracle_pack_base3": (None, [vp, i64, vp]),
                "oracle_pack_ternary_base3": (None, [vp, i64, i64, vp]),
                "oracle_unpack_ternary_base3": (i64, [vp, i64, i64, vp]),
                "oracle_unpack_base3": (None, [vp, i64, vp]),
                "oracle_fwht": (None, [vp, i64, i64, vp]),
                "oracle_rmsnorm": (None, [vp, i64, i64, vp, f64, vp]),
                "oracle_bitlinear_forward_norm": (i32, [vp, i64, i64, vp, i64, i32, i32, i32,
                                                        i32, vp, f64, vp, vp, vp, vp, vp, vp,
                                                        vp]),
                "oracle_quant_act": (None, [vp, i64, i64, i32, vp, vp, vp, vp]),
                "oracle_quant_act_absmean4": (None, [vp, i64, i64, vp, vp, vp, vp]),
                "oracle_quant_states": (None, [vp, i64, i64, i64, i32, vp, vp, vp]),
                "oracle_pack_bits": (None, [vp, i64, i64, i32, vp]),
                "oracle_unpack_bits": (None, [vp, i64, i64, i32, vp]),
                "oracle_pack_int4": (None, [vp, i64, i64, vp]),
                "oracle_unpack_int4": (None, [vp, i64, i64, vp]),
                "oracle_gemm_i64": (None, [vp, vp, i64, i64, i64, vp]),
                "oracle_gemm_addsub": (None, [vp, vp, i64, i64, i64, vp]),
                "oracle_dequant": (None, [vp, vp, f32, i64, i64, vp]),
                "oracle_dequant_act": (None, [vp, vp, f32, i64, i64, i32, vp]),
                "oracle_bitlinear_forward": (i32, [vp, i64, i64, vp, i64, i32, i32, vp,
                                                   vp, vp, vp, vp, vp, vp]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def num_threads() -> int:
    """Host threads the oracle's OpenMP loops use."""
    return int(lib().oracle_num_threads())


# --------------------------------------------------------------------------------------
# bf16 helpers (bf16 values are carried as uint16 bit patterns)
# --------------------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values straight to bf16 (ties to even); returns uint16 bit patterns."""
    L = lib()
    flat = np.ascontiguousarray(x, dtype=np.float64).ravel()
    out = np.fromiter((L.oracle_double_to_bf16(float(v)) for v in flat), dtype=np.uint16,
                      count=flat.size)
    return out.reshape(np.shape(x))


# --------------------------------------------------------------------------------------
# Step 1: absmean ternarisation  (b1.58 summary, 方法论 / 方法详解; 2B4T article, 一.2)
# --------------------------------------------------------------------------------------

def absmean_gamma(w_bf16: np.ndarray) -> np.float32:
    """gamma = fp32(max(mean|W|, 1e-5)) over the whole tensor."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    return np.float32(lib().oracle_absmean_gamma(_p(w), w.size))


def ternarize(w_bf16: np.ndarray, gamma) -> np.ndarray:
    """q = clip(rint(w / gamma), -1, 1), decided in IEEE fp32.  Returns int8 of W's shape."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    q = np.empty(w.shape, dtype=np.int8)
    lib().oracle_ternarize(_p(w), w.size, ctypes.c_float(float(gamma)), _p(q))
    return q


def absmean_gamma_f32(w_f32: np.ndarray) -> np.float32:
    """absmean scale of fp32 weights (the Hadamard-rotated rows): fp32(max(mean|w|, 1e-5)),
    the sum in double."""
    w = np.ascontiguousarray(w_f32, dtype=np.float32)
    return np.float32(lib().oracle_absmean_gamma_f32(_p(w), w.size))


def ternarize_f32(w_f32: np.ndarray, gamma) -> np.ndarray:
    """RoundClip(w / gamma, -1, 1) on fp32 weights, decided in fp32.  int8, same shape."""
    w = np.ascontiguousarray(w_f32, dtype=np.float32)
    q = np.empty(w.shape, dtype=np.int8)
    lib().oracle_ternarize_f32(_p(w), w.size, float(gamma), _p(q))
    return q


def rotate_weights(w_bf16: np.ndarray) -> np.ndarray:
    """Weight half of the weight + activation rotation: W' = W H / sqrt(K) row by row (H is
    symmetric, so W' x' = W x for x' = H x / sqrt(K)), in double, rounded to fp32 once."""
    return fwht(bf16_to_f64(w_bf16)).astype(np.float32)


def pack_ternary(q: np.ndarray) -> np.ndarray:
    """2-bit offset codes, interleaved words: [N, K/16] uint32 (see bitnet_oracle.c)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    N, K = q.shape
    out = np.empty((N, K // 16), dtype=np.uint32)
    lib().oracle_pack_ternary(_p(q), N, K, _p(out))
    return out


def unpack_ternary(wp: np.ndarray, K: int):
    """Inverse of pack_ternary.  Returns (q int8 [N, K], count of fields holding code 3)."""
    wp = np.ascontiguousarray(wp, dtype=np.uint32).reshape(-1, K // 16)
    N = wp.shape[0]
    q = np.empty((N, K), dtype=np.int8)
    bad = lib().oracle_unpack_ternary(_p(wp), N, K, _p(q))
    return q, int(bad)


def pack_base3(digits: np.ndarray) -> np.ndarray:
    """Five base-3 digits per byte, first digit most significant (2B4T article, 一.1)."""
    d = np.ascontiguousarray(digits, dtype=np.uint8).ravel()
    out = np.empty((d.size + 4) // 5, dtype=np.uint8)
    lib().oracle_pack_base3(_p(d), d.size, _p(out))
    return out


def unpack_base3(b: np.ndarray, n: int) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(n, dtype=np.uint8)
    lib().oracle_unpack_base3(_p(b), n, _p(out))
    return out


# --------------------------------------------------------------------------------------
# Step 2: online Hadamard transform  (BitNet v2 write-up, H-BitLinear paragraphs)
# --------------------------------------------------------------------------------------

def pack_ternary_base3(q: np.ndarray) -> np.ndarray:
    """Ternary int8 [N, K] -> base-3 rows, uint32 [N, ceil(K/20)] (BitNet b1.58 2B4T article,
    一.1: five ternary weights per byte; this library's row layout for the decode product)."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    N, K = q.shape
    out = np.zeros((N, (K + 19) // 20), dtype=np.uint32)
    lib().oracle_pack_ternary_base3(_p(q), N, K, _p(out))
    return out


def unpack_ternary_base3(words: np.ndarray, K: int):
    """Inverse of pack_ternary_base3: (q int8 [N, K], count of invalid bytes or padding)."""
    words = np.ascontiguousarray(words, dtype=np.uint32)
    N = words.shape[0]
    q = np.empty((N, K), dtype=np.int8)
    bad = lib().oracle_unpack_ternary_base3(_p(words), N, K, _p(q))
    return q, int(bad)


def rmsnorm(x: np.ndarray, gain_bf16: np.ndarray | None = None, eps: float = 1e-5) -> np.ndarray:
    """y = x * g / sqrt(mean(x^2) + eps) per row, in double (BitNet b1.58 2B4T article, 一.3:
    subln normalisation; BitNet v2 write-up: RMS normalisation).  x: [M, K] float64; gain: bf16
    bits [K] or None (unit gain)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    if x.ndim == 1:
        return rmsnorm(x[None, :], gain_bf16, eps)[0]
    M, K = x.shape
    y = np.empty_like(x)
    g = None if gain_bf16 is None else np.ascontiguousarray(gain_bf16, dtype=np.uint16)
    lib().oracle_rmsnorm(_p(x), M, K, None if g is None else _p(g), float(eps), _p(y))
    return y


def fwht(x: np.ndarray) -> np.ndarray:
    """z = H_K x / sqrt(K) per row, Sylvester order, in double.  x: [M, K] float64."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    if x.ndim == 1:
        return fwht(x[None, :])[0]
    M, K = x.shape
    z = np.empty_like(x)
    lib().oracle_fwht(_p(x), M, K, _p(z))
    return z


# --------------------------------------------------------------------------------------
# Step 3: per-token quantisation  (2B4T article, 一.2: absmax for 8-bit activations; BitNet v2
# write-up, INT8/INT4 paragraph: each width takes its own strategy -- absmean for INT4, the
# reading taken here)
# --------------------------------------------------------------------------------------

def quant_act_for_bits(z_f32: np.ndarray, bits: int):
    """The forward's quantiser for the width: absmax to INT8 (bits 8), absmean to INT4 (bits 4).
    Returns (codes, d, pre, rowsum) as quant_act."""
    return quant_act(z_f32, 8) if bits == 8 else quant_act_absmean4(z_f32)


def quant_act(z_f32: np.ndarray, bits: int):
    """Per-token absmax codes decided in fp32 (INT8; with bits 4, the absmax INT4 variant).

    Returns (codes int8 [M, K], d float32 [M], pre float64 [M, K], rowsum int64 [M]) where
    ``pre`` is the unrounded z * Q / max|z| in double.
    """
    z = np.ascontiguousarray(z_f32, dtype=np.float32)
    M, K = z.shape
    codes = np.empty((M, K), dtype=np.int8)
    d = np.empty(M, dtype=np.float32)
    pre = np.empty((M, K), dtype=np.float64)
    rowsum = np.empty(M, dtype=np.int64)
    lib().oracle_quant_act(_p(z), M, K, int(bits), _p(codes), _p(d), _p(pre), _p(rowsum))
    return codes, d, pre, rowsum


def quant_act_absmean4(z_f32: np.ndarray):
    """INT4 codes with a per-token absmean scale (the mean |z| maps to code sqrt(7)), decided in
    fp32 and clipped to [-8, 7]: the forward's INT4 quantiser.

    Returns (codes int8 [M, K], d float32 [M], pre float64 [M, K], rowsum int64 [M]) where
    ``pre`` is z * s in double, the value the rounding decides on.
    """
    z = np.ascontiguousarray(z_f32, dtype=np.float32)
    M, K = z.shape
    codes = np.empty((M, K), dtype=np.int8)
    d = np.empty(M, dtype=np.float32)
    pre = np.empty((M, K), dtype=np.float64)
    rowsum = np.empty(M, dtype=np.int64)
    lib().oracle_quant_act_absmean4(_p(z), M, K, _p(codes), _p(d), _p(pre), _p(rowsum))
    return codes, d, pre, rowsum


def pack_int4(c: np.ndarray) -> np.ndarray:
    """Nibble storage of INT4 codes: [M, K/2] uint8 (see bitnet_oracle.c)."""
    c = np.ascontiguousarray(c, dtype=np.int8)
    M, K = c.shape
    out = np.empty((M, K // 2), dtype=np.uint8)
    lib().oracle_pack_int4(_p(c), M, K, _p(out))
    return out


def unpack_int4(b: np.ndarray, K: int) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8).reshape(-1, K // 2)
    M = b.shape[0]
    c = np.empty((M, K), dtype=np.int8)
    lib().oracle_unpack_int4(_p(b), M, K, _p(c))
    return c


# --------------------------------------------------------------------------------------
# Low-bit Q / K / V states  (BitNet v2 write-up, Tables 2 and 3: the QKV states' bit width
# varies; a 3-bit KV cache matches full precision)
# --------------------------------------------------------------------------------------

def quant_states(x_bf16: np.ndarray, group: int, bits: int = 3):
    """Per-token (group = C) or per-head (group = head_dim) absmax codes of bf16 states [M, C],
    Q = 2^(bits-1) - 1, decided in fp32.  Returns (codes int8 [M, C], d float32 [M, C/group],
    pre float64 [M, C])."""
    x = bf16_to_f64(x_bf16).astype(np.float32)
    M, C = x.shape
    codes = np.empty((M, C), dtype=np.int8)
    d = np.empty((M, C // group), dtype=np.float32)
    pre = np.empty((M, C), dtype=np.float64)
    lib().oracle_quant_states(_p(x), M, C, int(group), int(bits), _p(codes), _p(d), _p(pre))
    return codes, d, pre


def pack_bits(c: np.ndarray, bits: int) -> np.ndarray:
    """Rows of `bits`-bit codes as little-endian bit streams: [M, C * bits / 8] uint8."""
    c = np.ascontiguousarray(c, dtype=np.int8)
    M, C = c.shape
    out = np.empty((M, C * bits // 8), dtype=np.uint8)
    lib().oracle_pack_bits(_p(c), M, C, int(bits), _p(out))
    return out


def unpack_bits(b: np.ndarray, C: int, bits: int) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8).reshape(-1, C * bits // 8)
    M = b.shape[0]
    c = np.empty((M, C), dtype=np.int8)
    lib().oracle_unpack_bits(_p(b), M, C, int(bits), _p(c))
    return c


# --------------------------------------------------------------------------------------
# Step 4: ternary x integer product  (2B4T article, 一.2: +1 adds, -1 subtracts, 0 skips)
# --------------------------------------------------------------------------------------

def gemm_i64(c: np.ndarray, q: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k c[m, k] q[n, k] in int64."""
    c = np.ascontiguousarray(c, dtype=np.int8)
    q = np.ascontiguousarray(q, dtype=np.int8)
    M, K = c.shape
    N = q.shape[0]
    acc = np.empty((M, N), dtype=np.int64)
    lib().oracle_gemm_i64(_p(c), _p(q), M, N, K, _p(acc))
    return acc


def gemm_addsub(c: np.ndarray, q: np.ndarray) -> np.ndarray:
    """The same product as add / subtract / skip, without multiplications."""
    c = np.ascontiguousarray(c, dtype=np.int8)
    q = np.ascontiguousarray(q, dtype=np.int8)
    M, K = c.shape
    N = q.shape[0]
    acc = np.empty((M, N), dtype=np.int64)
    lib().oracle_gemm_addsub(_p(c), _p(q), M, N, K, _p(acc))
    return acc


# --------------------------------------------------------------------------------------
# Step 5: rescale to bf16
# --------------------------------------------------------------------------------------

def dequant(acc: np.ndarray, d: np.ndarray, gamma) -> np.ndarray:
    """Y = bf16_rn(acc * d * gamma) (product in double); returns uint16 bf16 bit patterns."""
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    d = np.ascontiguousarray(d, dtype=np.float32)
    M, N = acc.shape
    Y = np.empty((M, N), dtype=np.uint16)
    lib().oracle_dequant(_p(acc), _p(d), ctypes.c_float(float(gamma)), M, N, _p(Y))
    return Y


# --------------------------------------------------------------------------------------
# The whole forward
# --------------------------------------------------------------------------------------

RELU2, SWIGLU = 1, 2


def dequant_act(acc: np.ndarray, d: np.ndarray, gamma, act: int) -> np.ndarray:
    """Rescale then activation (2B4T article, 一.3: squared ReLU; BitNet v2 write-up: SwishGLU),
    rounded to bf16 bits.  act RELU2: [M, N]; SWIGLU: rows interleaved gate/up, [M, N/2]."""
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    d = np.ascontiguousarray(d, dtype=np.float32)
    M, N = acc.shape
    Y = np.empty((M, N if act == RELU2 else N // 2), dtype=np.uint16)
    lib().oracle_dequant_act(_p(acc), _p(d), float(np.float32(gamma)), M, N, int(act), _p(Y))
    return Y


def bitlinear_forward(x_bf16: np.ndarray, w_bf16: np.ndarray, hadamard: bool, bits: int,
                      norm_gain: np.ndarray | None = None, norm_eps: float | None = None,
                      int4_absmax: bool = False):
    """Y = (H-)BitLinear(X) from bf16 X [M, K] and latent bf16 W [N, K].  bits 8: absmax INT8
    codes; bits 4: absmean INT4 codes (int4_absmax: the absmax variant).  With norm_eps given,
    every token row is RMS-normalised first (gain norm_gain, bf16 bits [K], or unit gain).

    Returns a dict with every stage: gamma, q, z, codes, d, acc, y (uint16 bf16 bits).
    """
    X = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    W = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    M, K = X.shape
    N = W.shape[0]
    Y = np.empty((M, N), dtype=np.uint16)
    gamma = np.zeros(1, dtype=np.float32)
    q = np.empty((N, K), dtype=np.int8)
    z = np.empty((M, K), dtype=np.float64)
    codes = np.empty((M, K), dtype=np.int8)
    d = np.empty(M, dtype=np.float32)
    acc = np.empty((M, N), dtype=np.int64)
    g = None if norm_gain is None else np.ascontiguousarray(norm_gain, dtype=np.uint16)
    rc = lib().oracle_bitlinear_forward_norm(
        _p(X), M, K, _p(W), N, int(bool(hadamard)), int(bits), int(bool(int4_absmax)),
        int(norm_eps is not None),
        None if g is None else _p(g), float(norm_eps or 0.0),
        _p(Y), _p(gamma), _p(q), _p(z), _p(codes), _p(d), _p(acc))
    if rc != 0:
        raise MemoryError("oracle_bitlinear_forward could not allocate its buffers")
    return {"gamma": np.float32(gamma[0]), "q": q, "z": z, "codes": codes, "d": d,
            "acc": acc, "y": Y}
