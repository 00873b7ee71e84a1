"""The C-ABI library loads and exports what include/bitnet.h declares (no GPU needed).

Only calls that never reach the device run here: size queries, status strings and the argument
checks that reject a call before any CUDA work.
"""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bitnet.h")


@pytest.fixture(scope="module")
def lib():
    from bit_activation_linear_b200 import build, binding
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bitnet_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("bitnet_quantize_pack_weights", "bitnet_bitlinear_forward",
                     "bitnet_hbitlinear_forward", "bitnet_act_quant", "bitnet_fwht_f32",
                     "bitnet_ternary_gemm", "bitnet_sync_status"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from bit_activation_linear_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (bitnet_[a-z0-9_]+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # the binding wraps every exported entry point under the same name
    for name in declared_functions():
        assert name in binding.EXPORTED


def test_library_targets_sm100a_only():
    from bit_activation_linear_b200 import binding
    out = subprocess.run(["cuobjdump", "--list-elf", binding.LIB_PATH], capture_output=True,
                         text=True).stdout
    assert "sm_100a" in out
    assert not re.search(r"sm_(?!100a)\d+", out)


def test_size_queries(lib):
    assert lib.bitnet_packed_weight_bytes(2048, 2048) == 2048 * 2048 // 4
    assert lib.bitnet_act_codes_bytes(16, 256, 8) == 16 * 256
    assert lib.bitnet_act_codes_bytes(16, 256, 4) == 16 * 128
    ws = lib.bitnet_workspace_bytes(4096, 2048, 2048, 8)
    assert ws >= 4096 * 2048 + 2 * 4096 * 4 and ws % 256 == 0
    assert lib.bitnet_weight_workspace_bytes(2048, 2048) % 256 == 0
    assert lib.bitnet_weight_workspace_bytes(2048, 2048) >= 8


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5):
        assert lib.bitnet_status_string(code).decode()
    assert lib.bitnet_status_string(0).decode() == "ok"


@pytest.mark.parametrize("M,K,N,bits", [
    (0, 256, 256, 8),      # no tokens
    (16, 100, 256, 8),     # K not a multiple of 128
    (16, 256, 12, 8),      # N not a multiple of 8
    (16, 256, 256, 5),     # act_bits
])
def test_forward_rejects_bad_shapes_before_touching_the_device(lib, M, K, N, bits):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the call must fail in the host check
    rc = lib.bitnet_hbitlinear_forward(fake, M, K, fake, fake, N, bits, fake, fake, 1 << 30, None)
    assert rc == -1
    assert lib.bitnet_last_error().decode()


def test_forward_rejects_null_and_misaligned_pointers(lib):
    good = ctypes.c_void_p(1 << 20)
    rc = lib.bitnet_bitlinear_forward(None, 16, 256, good, good, 256, 8, good, good, 1 << 30, None)
    assert rc == -1
    bad = ctypes.c_void_p((1 << 20) + 4)
    rc = lib.bitnet_bitlinear_forward(bad, 16, 256, good, good, 256, 8, good, good, 1 << 30, None)
    assert rc == -1
    assert "aligned" in lib.bitnet_last_error().decode()


def test_forward_rejects_small_workspace(lib):
    good = ctypes.c_void_p(1 << 20)
    rc = lib.bitnet_hbitlinear_forward(good, 16, 256, good, good, 256, 8, good, good, 64, None)
    assert rc == -5


def test_binding_raises_without_library(tmp_path):
    from bit_activation_linear_b200 import binding
    code = ("import bit_activation_linear_b200.binding as b\n"
            f"try:\n    b.load_library({str(tmp_path / 'missing.so')!r})\n"
            "except RuntimeError as e:\n    print('raised', 'no fallback' in str(e).lower())\n")
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert "raised True" in out.stdout, out.stdout + out.stderr


def test_selftest_rejects_bad_limits_before_touching_the_device(lib):
    for limit in (0, -5, 3_000_000_000):
        assert lib.bitnet_selftest_wait_timeout(ctypes.c_int64(limit), None) == -1  # INVALID


def test_activation_entries_reject_bad_arguments_before_the_device(lib):
    p = ctypes.c_void_p(16)
    # unknown activation
    rc = lib.bitnet_ternary_gemm_act(p, p, p, 8, 256, p, p, 256, 8, 3, p, None)
    assert rc == -1
    # SwiGLU needs N % 16 == 0
    rc = lib.bitnet_ternary_gemm_act(p, p, p, 8, 256, p, p, 264, 8, 2, p, None)
    assert rc == -1
    rc = lib.bitnet_bitlinear_forward_act(p, 8, 256, p, p, 264, 8, 0, 2, p, p, 1 << 20, None)
    assert rc == -1


def test_base3_entries_size_and_rejections_before_the_device(lib):
    # five weights a byte, rows of ceil(K/20) 32-bit words
    assert lib.bitnet_base3_weight_bytes(2048, 2048) == 2048 * 4 * 103
    assert lib.bitnet_base3_weight_bytes(8, 640) == 8 * 4 * 32
    assert lib.bitnet_base3_weight_bytes(0, 640) == 0
    p = ctypes.c_void_p(16)
    # more than 8 tokens: unsupported (the tensor-core product takes the 2-bit layout)
    assert lib.bitnet_ternary_gemv_base3(p, p, p, 9, 256, p, p, 256, 0, None, p, None) == -2
    assert lib.bitnet_bitlinear_forward_base3(p, 9, 256, p, p, 256, 0, 0, p, p, 1 << 20,
                                              None) == -2
    # unknown activation; an activation together with the int32 product; neither output
    assert lib.bitnet_ternary_gemv_base3(p, p, p, 4, 256, p, p, 256, 3, None, p, None) == -1
    assert lib.bitnet_ternary_gemv_base3(p, p, p, 4, 256, p, p, 256, 1, p, p, None) == -1
    assert lib.bitnet_ternary_gemv_base3(p, p, p, 4, 256, p, p, 256, 0, None, None, None) == -1
    # K not a multiple of 128; misaligned weights
    assert lib.bitnet_ternary_gemv_base3(p, p, p, 4, 200, p, p, 256, 0, None, p, None) == -1
    q = ctypes.c_void_p(20)
    assert lib.bitnet_quantize_pack_weights_base3(p, 256, 256, q, p, p, 1 << 20, None) == -1
    assert lib.bitnet_quantize_pack_weights_base3(p, 256, 256, p, p, p, 0, None) == -5


def test_absmax4_entries_reject_bad_arguments_before_the_device(lib):
    p = ctypes.c_void_p(16)
    assert lib.bitnet_act_quant_absmax4(p, 4, 200, 1, p, p, p, None) == -1      # K % 128
    assert lib.bitnet_act_quant_absmax4(p, 0, 256, 1, p, p, p, None) == -1      # M < 1
    assert lib.bitnet_act_quant_absmax4(None, 4, 256, 1, p, p, p, None) == -1   # null X
    q = ctypes.c_void_p(24)
    assert lib.bitnet_act_quant_absmax4(q, 4, 256, 1, p, p, p, None) == -1      # misaligned
    assert lib.bitnet_bitlinear_forward_absmax4(p, 4, 256, p, p, 256, 1, p, p, 0, None) == -5


def test_rotated_weight_entries_size_and_rejections_before_the_device(lib):
    ws = lib.bitnet_weight_workspace_bytes_rotated(2048, 2048)
    assert ws >= 4 * 2048 * 2048 + lib.bitnet_weight_workspace_bytes(2048, 2048)
    assert ws % 256 == 0 and lib.bitnet_weight_workspace_bytes_rotated(0, 128) == 0
    p = ctypes.c_void_p(16)
    assert lib.bitnet_quantize_pack_weights_rotated(p, 256, 200, p, p, p, 1 << 30, None) == -1
    assert lib.bitnet_quantize_pack_weights_rotated(p, 12, 256, p, p, p, 1 << 30, None) == -1
    assert lib.bitnet_quantize_pack_weights_rotated(p, 256, 256, p, p, p, 1024, None) == -5
    q = ctypes.c_void_p(24)
    assert lib.bitnet_quantize_pack_weights_rotated(p, 256, 256, q, p, p, 1 << 30, None) == -1


def test_state_quant_size_and_rejections_before_the_device(lib):
    assert lib.bitnet_state_codes_bytes(16, 4096, 3) == 16 * 4096 * 3 // 8
    assert lib.bitnet_state_codes_bytes(16, 4096, 9) == 0
    p = ctypes.c_void_p(16)
    assert lib.bitnet_quant_states(p, 4, 4096, 100, 3, p, p, None) == -1    # group % 32
    assert lib.bitnet_quant_states(p, 4, 4000, 128, 3, p, p, None) == -1    # C % group
    assert lib.bitnet_quant_states(p, 4, 4096, 128, 1, p, p, None) == -1    # bits
    assert lib.bitnet_quant_states(p, 0, 4096, 128, 3, p, p, None) == -1    # M
    assert lib.bitnet_quant_states(None, 4, 4096, 128, 3, p, p, None) == -1  # null X
    q = ctypes.c_void_p(20)
    assert lib.bitnet_quant_states(q, 4, 4096, 128, 3, p, p, None) == -1    # misaligned


def test_act_quant_plan_host_only():
    """The quantiser plan is a host query: it needs no device and names the kernel each case
    takes (the tensor-core Hadamard only for K = 8192 / 16384 without the RMS norm)."""
    from bit_activation_linear_b200 import binding as B
    assert B.bitnet_act_quant_plan(4096, False) == B.QUANT_PLAIN
    assert B.bitnet_act_quant_plan(2048, True) == B.QUANT_FWHT
    assert B.bitnet_act_quant_plan(8192, True) == B.QUANT_HADAMARD_TC
    assert B.bitnet_act_quant_plan(16384, True) == B.QUANT_HADAMARD_TC
    assert B.bitnet_act_quant_plan(16384, True, norm=True) == B.QUANT_FWHT
    assert B.bitnet_act_quant_plan(32768, True) == B.QUANT_FWHT
    lib = B.load_library()
    out = ctypes.c_int(0)
    assert lib.bitnet_act_quant_plan(3 * 128, 1, 0, ctypes.byref(out)) == -2   # not 2^k
    assert lib.bitnet_act_quant_plan(100, 0, 0, ctypes.byref(out)) == -1       # K % 128
    assert lib.bitnet_act_quant_plan(4096, 1, 0, None) == -1                   # null path
