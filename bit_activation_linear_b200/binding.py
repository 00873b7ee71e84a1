"""Python binding of libbitnet_b200.so: argument marshalling only.

Every function here has the name of the C entry point it calls (include/bitnet.h), takes torch
CUDA tensors, checks dtype / device / contiguity, allocates outputs and workspace with torch
(the library itself never allocates) and passes raw pointers plus the current torch stream.  All
arithmetic runs in the library's kernels; there is no fallback of any kind: if the shared
library is missing or cannot load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbitnet_b200.so")
_lock = threading.Lock()
_lib = None

OK, ERR_INVALID, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = 0, -1, -2, -3, -4, -5
ACT_RELU2, ACT_SWIGLU = 1, 2  # bitnet_activation
PATH_DECODE, PATH_TC, PATH_TC_SKINNY, PATH_TC_TMEM = 1, 2, 3, 4  # bitnet_product_path
QUANT_PLAIN, QUANT_FWHT, QUANT_HADAMARD_TC = 1, 2, 3  # bitnet_quant_path


class BitnetError(RuntimeError):
    """A non-zero status from the library, with its text and the library's detail message."""

    def __init__(self, status: int, where: str):
        lib = load_library()
        self.status = status
        text = lib.bitnet_status_string(status).decode()
        detail = lib.bitnet_last_error().decode()
        super().__init__(f"{where}: {text} ({status}): {detail}")


_SIGS = {
    "bitnet_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bitnet_last_error": (ctypes.c_char_p, []),
    "bitnet_launch_count": (ctypes.c_uint64, []),
    "bitnet_packed_weight_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "bitnet_weight_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "bitnet_quantize_pack_weights": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                    ctypes.c_int64, ctypes.c_void_p,
                                                    ctypes.c_void_p, ctypes.c_void_p,
                                                    ctypes.c_size_t, ctypes.c_void_p]),
    "bitnet_quantize_pack_weights_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                            ctypes.c_int64, ctypes.c_void_p,
                                                            ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_act_codes_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]),
    "bitnet_act_quant": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_fwht_f32": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_ternary_gemm": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                 ctypes.c_int]),
    "bitnet_product_plan": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                           ctypes.POINTER(ctypes.c_int)]),
    "bitnet_act_quant_plan": (ctypes.c_int, [ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                             ctypes.POINTER(ctypes.c_int)]),
    "bitnet_bitlinear_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                                ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p]),
    "bitnet_hbitlinear_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                                 ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_size_t, ctypes.c_void_p]),
    "bitnet_act_quant_norm": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_float, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_norm_transform_f32": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                 ctypes.c_void_p, ctypes.c_float, ctypes.c_int,
                                                 ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_norm_bitlinear_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                     ctypes.c_int64, ctypes.c_void_p,
                                                     ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                                     ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                                     ctypes.c_void_p, ctypes.c_void_p,
                                                     ctypes.c_size_t, ctypes.c_void_p]),
    "bitnet_ternary_gemm_act": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                               ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_bitlinear_forward_act": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                    ctypes.c_int64, ctypes.c_void_p,
                                                    ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                                    ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                                    ctypes.c_void_p, ctypes.c_size_t,
                                                    ctypes.c_void_p]),
    "bitnet_weight_workspace_bytes_rotated": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "bitnet_quantize_pack_weights_rotated": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                            ctypes.c_int64, ctypes.c_void_p,
                                                            ctypes.c_void_p, ctypes.c_void_p,
                                                            ctypes.c_size_t, ctypes.c_void_p]),
    "bitnet_act_quant_absmax4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                 ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_bitlinear_forward_absmax4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                         ctypes.c_int64, ctypes.c_void_p,
                                                         ctypes.c_void_p, ctypes.c_int64,
                                                         ctypes.c_int, ctypes.c_void_p,
                                                         ctypes.c_void_p, ctypes.c_size_t,
                                                         ctypes.c_void_p]),
    "bitnet_base3_weight_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "bitnet_quantize_pack_weights_base3": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                          ctypes.c_int64, ctypes.c_void_p,
                                                          ctypes.c_void_p, ctypes.c_void_p,
                                                          ctypes.c_size_t, ctypes.c_void_p]),
    "bitnet_ternary_gemv_base3": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                                 ctypes.c_void_p, ctypes.c_void_p,
                                                 ctypes.c_void_p]),
    "bitnet_bitlinear_forward_base3": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                      ctypes.c_int64, ctypes.c_void_p,
                                                      ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                                      ctypes.c_int, ctypes.c_void_p,
                                                      ctypes.c_void_p, ctypes.c_size_t,
                                                      ctypes.c_void_p]),
    "bitnet_state_codes_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]),
    "bitnet_quant_states": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_int, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p]),
    "bitnet_sync_status": (ctypes.c_int, [ctypes.c_void_p]),
    "bitnet_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int64, ctypes.c_void_p]),
}

EXPORTED = tuple(_SIGS)


def load_library(path: str | None = None):
    """Load (once) and return the ctypes handle of libbitnet_b200.so.  Raises if it is absent."""
    global _lib
    with _lock:
        if _lib is None:
            p = path or LIB_PATH
            if not os.path.exists(p):
                raise RuntimeError(
                    f"{p} is missing: build it with `python -m bit_activation_linear_b200.build`"
                    " (nvcc, sm_100a). There is no fallback implementation.")
            lib = ctypes.CDLL(p)
            for name, (res, args) in _SIGS.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(t: torch.Tensor, name: str, dtype=None, dim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions")


def _nbytes_at_least(t: torch.Tensor, need: int, name: str):
    have = t.numel() * t.element_size()
    if have < need:
        raise ValueError(f"{name} holds {have} bytes, {need} needed")


def _rc(status: int, where: str):
    if status != OK:
        raise BitnetError(status, where)


def bitnet_launch_count() -> int:
    return int(load_library().bitnet_launch_count())


def bitnet_packed_weight_bytes(N: int, K: int) -> int:
    return int(load_library().bitnet_packed_weight_bytes(N, K))


def bitnet_weight_workspace_bytes(N: int, K: int) -> int:
    return int(load_library().bitnet_weight_workspace_bytes(N, K))


def bitnet_act_codes_bytes(M: int, K: int, act_bits: int) -> int:
    return int(load_library().bitnet_act_codes_bytes(M, K, act_bits))


def bitnet_workspace_bytes(M: int, K: int, N: int, act_bits: int) -> int:
    return int(load_library().bitnet_workspace_bytes(M, K, N, act_bits))


def bitnet_product_plan(M: int, K: int, N: int, act_bits: int):
    """(path, k_split) of the product of this shape on the current device (PATH_* values)."""
    path, split = ctypes.c_int(0), ctypes.c_int(0)
    _rc(load_library().bitnet_product_plan(M, K, N, int(act_bits), ctypes.byref(path),
                                           ctypes.byref(split)), "bitnet_product_plan")
    return path.value, split.value


def bitnet_act_quant_plan(K: int, hadamard: bool, norm: bool = False) -> int:
    """Which kernel quantises a K-wide row (QUANT_* values); host only, no device needed."""
    path = ctypes.c_int(0)
    _rc(load_library().bitnet_act_quant_plan(K, int(bool(hadamard)), int(bool(norm)),
                                             ctypes.byref(path)), "bitnet_act_quant_plan")
    return path.value


def bitnet_quantize_pack_weights(W: torch.Tensor, Wp: torch.Tensor | None = None,
                                 gamma: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                                 stream=None):
    """absmean-ternarise and pack bf16 W [N, K].  Returns (Wp uint8 [N, K/4], gamma float [1])."""
    L = load_library()
    _check(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    if Wp is None:
        Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    need = int(L.bitnet_weight_workspace_bytes(N, K))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=W.device)
    _rc(L.bitnet_quantize_pack_weights(W.data_ptr(), N, K, Wp.data_ptr(), gamma.data_ptr(),
                                       ws.data_ptr(), ws.numel() * ws.element_size(),
                                       _stream(stream)), "bitnet_quantize_pack_weights")
    return Wp, gamma


def bitnet_quantize_pack_weights_noalloc(W: torch.Tensor, Wp: torch.Tensor | None = None,
                                         gamma: torch.Tensor | None = None, stream=None):
    """As bitnet_quantize_pack_weights, with the library's fixed device scratch instead of a
    workspace (for callers that cannot allocate device memory).  Returns (Wp, gamma)."""
    L = load_library()
    _check(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    if Wp is None:
        Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    _rc(L.bitnet_quantize_pack_weights_noalloc(W.data_ptr(), N, K, Wp.data_ptr(),
                                               gamma.data_ptr(), _stream(stream)),
        "bitnet_quantize_pack_weights_noalloc")
    return Wp, gamma


def bitnet_act_quant(X: torch.Tensor, hadamard: bool, act_bits: int, codes=None, scales=None,
                     rowsum=None, stream=None):
    """Per-token (Hadamard +) quantisation: absmax INT8 or absmean INT4.  Returns (codes,
    scales, rowsum)."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    if codes is None:
        codes = torch.empty((M, K if act_bits == 8 else K // 2),
                            dtype=torch.int8 if act_bits == 8 else torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty(M, dtype=torch.float32, device=X.device)
    if rowsum is None:
        rowsum = torch.empty(M, dtype=torch.int32, device=X.device)
    _nbytes_at_least(codes, int(L.bitnet_act_codes_bytes(M, K, act_bits)), "codes")
    _nbytes_at_least(scales, 4 * M, "scales")
    _nbytes_at_least(rowsum, 4 * M, "rowsum")
    _rc(L.bitnet_act_quant(X.data_ptr(), M, K, int(bool(hadamard)), int(act_bits),
                           codes.data_ptr(), scales.data_ptr(), rowsum.data_ptr(),
                           _stream(stream)), "bitnet_act_quant")
    return codes, scales, rowsum


def bitnet_fwht_f32(X: torch.Tensor, Z: torch.Tensor | None = None, stream=None):
    """Z = H_K X / sqrt(K) per row in fp32 (debug / parity entry)."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    if Z is None:
        Z = torch.empty((M, K), dtype=torch.float32, device=X.device)
    _rc(L.bitnet_fwht_f32(X.data_ptr(), M, K, Z.data_ptr(), _stream(stream)), "bitnet_fwht_f32")
    return Z


def bitnet_ternary_gemm(codes: torch.Tensor, scales: torch.Tensor, rowsum: torch.Tensor, K: int,
                        Wp: torch.Tensor, gamma: torch.Tensor, act_bits: int, want_acc=False,
                        want_y=True, acc=None, Y=None, stream=None):
    """Ternary x integer product (+ rescale).  Returns (acc int32 [M, N] or None, Y bf16 or None)."""
    L = load_library()
    for t, n in ((codes, "codes"), (scales, "scales"), (rowsum, "rowsum"), (Wp, "Wp"),
                 (gamma, "gamma")):
        _check(t, n)
    M = scales.numel()
    N = Wp.shape[0]
    _nbytes_at_least(codes, int(L.bitnet_act_codes_bytes(M, K, act_bits)), "codes")
    _nbytes_at_least(rowsum, 4 * M, "rowsum")
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if want_acc and acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=codes.device)
    if want_y and Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=codes.device)
    _rc(L.bitnet_ternary_gemm(codes.data_ptr(), scales.data_ptr(), rowsum.data_ptr(), M, K,
                              Wp.data_ptr(), gamma.data_ptr(), N, int(act_bits),
                              acc.data_ptr() if acc is not None else None,
                              Y.data_ptr() if Y is not None else None, _stream(stream)),
        "bitnet_ternary_gemm")
    return acc, Y


def _forward(fn_name: str, X, Wp, gamma, act_bits, Y, ws, stream):
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    _check(Wp, "Wp")
    _check(gamma, "gamma", torch.float32)
    M, K = X.shape
    N = Wp.shape[0]
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _nbytes_at_least(Y, 2 * M * N, "Y")
    need = int(L.bitnet_workspace_bytes(M, K, N, act_bits))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _rc(getattr(L, fn_name)(X.data_ptr(), M, K, Wp.data_ptr(), gamma.data_ptr(), N,
                            int(act_bits), Y.data_ptr(), ws.data_ptr(),
                            ws.numel() * ws.element_size(), _stream(stream)), fn_name)
    return Y


def bitnet_bitlinear_forward(X, Wp, gamma, act_bits=8, Y=None, ws=None, stream=None):
    """Y = BitLinear(X) for bf16 X [M, K] and packed ternary Wp [N, K/4]."""
    return _forward("bitnet_bitlinear_forward", X, Wp, gamma, act_bits, Y, ws, stream)


def bitnet_hbitlinear_forward(X, Wp, gamma, act_bits=8, Y=None, ws=None, stream=None):
    """Y = H-BitLinear(X): online Hadamard transform, then BitLinear."""
    return _forward("bitnet_hbitlinear_forward", X, Wp, gamma, act_bits, Y, ws, stream)


def _act_cols(N: int, activation: int) -> int:
    return N // 2 if activation == ACT_SWIGLU else N


def bitnet_ternary_gemm_act(codes, scales, rowsum, K: int, Wp, gamma, act_bits: int,
                            activation: int, Y=None, stream=None):
    """Y = activation(rescaled product): squared ReLU [M, N] or SwiGLU over interleaved gate/up
    features [M, N/2] (bf16)."""
    L = load_library()
    for t, n in ((codes, "codes"), (scales, "scales"), (rowsum, "rowsum"), (Wp, "Wp"),
                 (gamma, "gamma")):
        _check(t, n)
    M = scales.numel()
    N = Wp.shape[0]
    _nbytes_at_least(codes, int(L.bitnet_act_codes_bytes(M, K, act_bits)), "codes")
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if Y is None:
        Y = torch.empty((M, _act_cols(N, activation)), dtype=torch.bfloat16, device=Wp.device)
    _nbytes_at_least(Y, 2 * M * _act_cols(N, activation), "Y")
    _rc(L.bitnet_ternary_gemm_act(codes.data_ptr(), scales.data_ptr(), rowsum.data_ptr(), M, K,
                                  Wp.data_ptr(), gamma.data_ptr(), N, int(act_bits),
                                  int(activation), Y.data_ptr(), _stream(stream)),
        "bitnet_ternary_gemm_act")
    return Y


def bitnet_bitlinear_forward_act(X, Wp, gamma, act_bits, hadamard, activation, Y=None, ws=None,
                                 stream=None):
    """Y = activation((H-)BitLinear(X)) with the activation in the product's epilogue."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    _check(Wp, "Wp")
    _check(gamma, "gamma", torch.float32)
    M, K = X.shape
    N = Wp.shape[0]
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if Y is None:
        Y = torch.empty((M, _act_cols(N, activation)), dtype=torch.bfloat16, device=X.device)
    _nbytes_at_least(Y, 2 * M * _act_cols(N, activation), "Y")
    need = int(L.bitnet_workspace_bytes(M, K, N, act_bits))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _rc(L.bitnet_bitlinear_forward_act(X.data_ptr(), M, K, Wp.data_ptr(), gamma.data_ptr(), N,
                                       int(act_bits), int(bool(hadamard)), int(activation),
                                       Y.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                                       _stream(stream)),
        "bitnet_bitlinear_forward_act")
    return Y


def _gain_ptr(gain, K):
    if gain is None:
        return None
    _check(gain, "norm_gain", torch.bfloat16, 1)
    if gain.numel() != K:
        raise ValueError(f"norm_gain has {gain.numel()} entries, K = {K}")
    return gain.data_ptr()


def bitnet_act_quant_norm(X: torch.Tensor, norm_gain, eps: float, hadamard: bool, act_bits: int,
                          codes=None, scales=None, rowsum=None, stream=None):
    """RMS normalisation (gain norm_gain bf16 [K] or None, eps) fused with per-token
    (Hadamard +) absmax quantisation.  Returns (codes, scales, rowsum)."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    if codes is None:
        codes = torch.empty((M, K if act_bits == 8 else K // 2),
                            dtype=torch.int8 if act_bits == 8 else torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty(M, dtype=torch.float32, device=X.device)
    if rowsum is None:
        rowsum = torch.empty(M, dtype=torch.int32, device=X.device)
    _nbytes_at_least(codes, int(L.bitnet_act_codes_bytes(M, K, act_bits)), "codes")
    _nbytes_at_least(scales, 4 * M, "scales")
    _nbytes_at_least(rowsum, 4 * M, "rowsum")
    _rc(L.bitnet_act_quant_norm(X.data_ptr(), M, K, _gain_ptr(norm_gain, K), float(eps),
                                int(bool(hadamard)), int(act_bits), codes.data_ptr(),
                                scales.data_ptr(), rowsum.data_ptr(), _stream(stream)),
        "bitnet_act_quant_norm")
    return codes, scales, rowsum


def bitnet_norm_transform_f32(X: torch.Tensor, norm_gain, eps: float, hadamard: bool,
                              Z: torch.Tensor | None = None, stream=None):
    """The normalised rows (and their Hadamard transform) in fp32 (debug / parity entry)."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    if Z is None:
        Z = torch.empty((M, K), dtype=torch.float32, device=X.device)
    _rc(L.bitnet_norm_transform_f32(X.data_ptr(), M, K, _gain_ptr(norm_gain, K), float(eps),
                                    int(bool(hadamard)), Z.data_ptr(), _stream(stream)),
        "bitnet_norm_transform_f32")
    return Z


def bitnet_norm_bitlinear_forward(X, norm_gain, eps, hadamard, Wp, gamma, act_bits=8, Y=None,
                                  ws=None, stream=None):
    """Y = (H-)BitLinear(RMSNorm(X)) with the normalisation fused into the quantiser."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    _check(Wp, "Wp")
    _check(gamma, "gamma", torch.float32)
    M, K = X.shape
    N = Wp.shape[0]
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _nbytes_at_least(Y, 2 * M * N, "Y")
    need = int(L.bitnet_workspace_bytes(M, K, N, act_bits))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _rc(L.bitnet_norm_bitlinear_forward(X.data_ptr(), M, K, _gain_ptr(norm_gain, K), float(eps),
                                        int(bool(hadamard)), Wp.data_ptr(), gamma.data_ptr(), N,
                                        int(act_bits), Y.data_ptr(), ws.data_ptr(),
                                        ws.numel() * ws.element_size(), _stream(stream)),
        "bitnet_norm_bitlinear_forward")
    return Y


def bitnet_weight_workspace_bytes_rotated(N: int, K: int) -> int:
    return int(load_library().bitnet_weight_workspace_bytes_rotated(N, K))


def bitnet_quantize_pack_weights_rotated(W: torch.Tensor, Wp: torch.Tensor | None = None,
                                         gamma: torch.Tensor | None = None,
                                         ws: torch.Tensor | None = None, stream=None):
    """Weight half of the weight + activation Hadamard rotation: ternarise and pack the rows of
    W H / sqrt(K).  Returns (Wp uint8 [N, K/4], gamma float [1]) for bitnet_hbitlinear_forward."""
    L = load_library()
    _check(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    if Wp is None:
        Wp = torch.empty((N, K // 4), dtype=torch.uint8, device=W.device)
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    need = int(L.bitnet_weight_workspace_bytes_rotated(N, K))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=W.device)
    _rc(L.bitnet_quantize_pack_weights_rotated(W.data_ptr(), N, K, Wp.data_ptr(),
                                               gamma.data_ptr(), ws.data_ptr(),
                                               ws.numel() * ws.element_size(), _stream(stream)),
        "bitnet_quantize_pack_weights_rotated")
    return Wp, gamma


def bitnet_act_quant_absmax4(X: torch.Tensor, hadamard: bool, codes=None, scales=None,
                             rowsum=None, stream=None):
    """Variant INT4 quantiser with a per-token absmax scale (Q = 7).  Returns (codes uint8
    [M, K/2] nibbles, scales, rowsum), consumed by the product with act_bits 4."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    if codes is None:
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty(M, dtype=torch.float32, device=X.device)
    if rowsum is None:
        rowsum = torch.empty(M, dtype=torch.int32, device=X.device)
    _nbytes_at_least(codes, int(L.bitnet_act_codes_bytes(M, K, 4)), "codes")
    _nbytes_at_least(scales, 4 * M, "scales")
    _nbytes_at_least(rowsum, 4 * M, "rowsum")
    _rc(L.bitnet_act_quant_absmax4(X.data_ptr(), M, K, int(bool(hadamard)), codes.data_ptr(),
                                   scales.data_ptr(), rowsum.data_ptr(), _stream(stream)),
        "bitnet_act_quant_absmax4")
    return codes, scales, rowsum


def bitnet_bitlinear_forward_absmax4(X, Wp, gamma, hadamard: bool, Y=None, ws=None, stream=None):
    """Y = (H-)BitLinear(X) with the variant absmax INT4 activation quantiser."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    _check(Wp, "Wp")
    _check(gamma, "gamma", torch.float32)
    M, K = X.shape
    N = Wp.shape[0]
    _nbytes_at_least(Wp, int(L.bitnet_packed_weight_bytes(N, K)), "Wp")
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _nbytes_at_least(Y, 2 * M * N, "Y")
    need = int(L.bitnet_workspace_bytes(M, K, N, 4))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _rc(L.bitnet_bitlinear_forward_absmax4(X.data_ptr(), M, K, Wp.data_ptr(), gamma.data_ptr(),
                                           N, int(bool(hadamard)), Y.data_ptr(), ws.data_ptr(),
                                           ws.numel() * ws.element_size(), _stream(stream)),
        "bitnet_bitlinear_forward_absmax4")
    return Y


def bitnet_base3_weight_bytes(N: int, K: int) -> int:
    return int(load_library().bitnet_base3_weight_bytes(N, K))


def bitnet_quantize_pack_weights_base3(W: torch.Tensor, Wp3: torch.Tensor | None = None,
                                       gamma: torch.Tensor | None = None,
                                       ws: torch.Tensor | None = None, stream=None):
    """absmean-ternarise bf16 W [N, K] into base-3 rows (five weights a byte).
    Returns (Wp3 uint8 [N, 4 * ceil(K/20)], gamma float [1])."""
    L = load_library()
    _check(W, "W", torch.bfloat16, 2)
    N, K = W.shape
    if Wp3 is None:
        Wp3 = torch.empty((N, 4 * ((K + 19) // 20)), dtype=torch.uint8, device=W.device)
    _nbytes_at_least(Wp3, int(L.bitnet_base3_weight_bytes(N, K)), "Wp3")
    if gamma is None:
        gamma = torch.empty(1, dtype=torch.float32, device=W.device)
    need = int(L.bitnet_weight_workspace_bytes(N, K))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=W.device)
    _rc(L.bitnet_quantize_pack_weights_base3(W.data_ptr(), N, K, Wp3.data_ptr(),
                                             gamma.data_ptr(), ws.data_ptr(),
                                             ws.numel() * ws.element_size(), _stream(stream)),
        "bitnet_quantize_pack_weights_base3")
    return Wp3, gamma


def bitnet_ternary_gemv_base3(codes, scales, rowsum, K: int, Wp3, gamma, activation: int = 0,
                              want_acc=False, want_y=True, acc=None, Y=None, stream=None):
    """Product of INT8 codes (M <= 8 tokens) with base-3 weights Wp3 [N, 4 * ceil(K/20)].
    Returns (acc int32 [M, N] or None, Y bf16 [M, N] ([M, N/2] for SwiGLU) or None)."""
    L = load_library()
    for t, n in ((codes, "codes"), (scales, "scales"), (rowsum, "rowsum"), (Wp3, "Wp3"),
                 (gamma, "gamma")):
        _check(t, n)
    M = scales.numel()
    N = Wp3.shape[0]
    _nbytes_at_least(codes, int(L.bitnet_act_codes_bytes(M, K, 8)), "codes")
    _nbytes_at_least(rowsum, 4 * M, "rowsum")
    _nbytes_at_least(Wp3, int(L.bitnet_base3_weight_bytes(N, K)), "Wp3")
    if want_acc and acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=codes.device)
    if want_y and Y is None:
        Y = torch.empty((M, _act_cols(N, activation)), dtype=torch.bfloat16, device=codes.device)
    if Y is not None:
        _nbytes_at_least(Y, 2 * M * _act_cols(N, activation), "Y")
    _rc(L.bitnet_ternary_gemv_base3(codes.data_ptr(), scales.data_ptr(), rowsum.data_ptr(), M, K,
                                    Wp3.data_ptr(), gamma.data_ptr(), N, int(activation),
                                    acc.data_ptr() if acc is not None else None,
                                    Y.data_ptr() if Y is not None else None, _stream(stream)),
        "bitnet_ternary_gemv_base3")
    return acc, Y


def bitnet_bitlinear_forward_base3(X, Wp3, gamma, hadamard: bool, activation: int = 0, Y=None,
                                   ws=None, stream=None):
    """Y = activation((H-)BitLinear(X)) for M <= 8 tokens on base-3 weights, INT8 activations."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    _check(Wp3, "Wp3")
    _check(gamma, "gamma", torch.float32)
    M, K = X.shape
    N = Wp3.shape[0]
    _nbytes_at_least(Wp3, int(L.bitnet_base3_weight_bytes(N, K)), "Wp3")
    if Y is None:
        Y = torch.empty((M, _act_cols(N, activation)), dtype=torch.bfloat16, device=X.device)
    _nbytes_at_least(Y, 2 * M * _act_cols(N, activation), "Y")
    need = int(L.bitnet_workspace_bytes(M, K, N, 8))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=X.device)
    _rc(L.bitnet_bitlinear_forward_base3(X.data_ptr(), M, K, Wp3.data_ptr(), gamma.data_ptr(), N,
                                         int(bool(hadamard)), int(activation), Y.data_ptr(),
                                         ws.data_ptr(), ws.numel() * ws.element_size(),
                                         _stream(stream)),
        "bitnet_bitlinear_forward_base3")
    return Y


def bitnet_state_codes_bytes(M: int, C: int, bits: int) -> int:
    return int(load_library().bitnet_state_codes_bytes(M, C, bits))


def bitnet_quant_states(X: torch.Tensor, group: int, bits: int = 3, codes=None, scales=None,
                        stream=None):
    """Low-bit absmax codes of bf16 Q/K/V states [M, C], per group of `group` features.
    Returns (codes uint8 [M, C * bits / 8] bit streams, scales float [M, C / group])."""
    L = load_library()
    _check(X, "X", torch.bfloat16, 2)
    M, C = X.shape
    if codes is None:
        codes = torch.empty((M, C * bits // 8), dtype=torch.uint8, device=X.device)
    if scales is None:
        scales = torch.empty((M, max(C // group, 1)), dtype=torch.float32, device=X.device)
    _nbytes_at_least(codes, int(L.bitnet_state_codes_bytes(M, C, bits)), "codes")
    _nbytes_at_least(scales, 4 * M * (C // group), "scales")
    _rc(L.bitnet_quant_states(X.data_ptr(), M, C, int(group), int(bits), codes.data_ptr(),
                              scales.data_ptr(), _stream(stream)), "bitnet_quant_states")
    return codes, scales


def bitnet_selftest_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Enqueue the failure-detection self-test: one bounded wait that runs out after
    limit_cycles SM cycles and records a time-out for the next bitnet_sync_status()."""
    st = load_library().bitnet_selftest_wait_timeout(int(limit_cycles), _stream(stream))
    _rc(st, "bitnet_selftest_wait_timeout")


def bitnet_sync_status(stream=None) -> int:
    """Synchronise the stream and raise BitnetError if a kernel reported a fault or time-out."""
    st = load_library().bitnet_sync_status(_stream(stream))
    _rc(st, "bitnet_sync_status")
    return st
