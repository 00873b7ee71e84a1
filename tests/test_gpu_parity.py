"""GPU parity: every stage of the CUDA path against the CPU oracle, through the C ABI.

Tolerances (written here, from the contract of the forward):
  * packed weights and gamma: bit-exact;
  * Hadamard output (fp32): per row, max|z - z_ref| <= 1e-5 * max|z_ref|;
  * activation codes: a code may differ by +-1 only where the oracle's unrounded value lies
    within 1e-4 of a .5 boundary, and on at most 1e-4 of the codes;
  * int32 accumulators: bit-exact against the oracle fed the same codes;
  * bf16 output: elementwise relative error <= 1e-2 against the oracle fed the same codes, and
    ||Y - Y_ref||_F / ||Y_ref||_F <= 1e-2 against the fully independent oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_activation_linear_b200 import synth

pytestmark = pytest.mark.gpu

CODE_BOUNDARY = 1e-4
CODE_FRACTION = 1e-4
FWHT_REL = 1e-5
Y_REL = 1e-2


@pytest.fixture(scope="module")
def B():
    from bit_activation_linear_b200 import build, binding
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    binding.load_library()
    return binding


def dev_bf16(bits):
    return synth.to_torch_bf16(bits).cuda()


def to_np_bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def check_codes(codes_gpu, codes_ref, pre):
    diff = codes_gpu.astype(np.int32) - codes_ref.astype(np.int32)
    bad = diff != 0
    if bad.any():
        assert np.abs(diff).max() <= 1
        dist = np.abs(np.abs(pre[bad] - np.floor(pre[bad])) - 0.5)
        assert np.all(dist < CODE_BOUNDARY), dist.max()
        assert bad.mean() <= CODE_FRACTION
    return int(bad.sum())


# ----------------------------------------------------------------------------------------
# step 1: weights
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(256, 256), (8, 128), (264, 384), (2048, 2048), (2048, 8192)])
def test_weights_bit_exact(B, N, K):
    W = synth.latent_weights(N, K, seed=N + K)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    B.bitnet_sync_status()
    g_ref = oracle.absmean_gamma(W)
    assert np.float32(gamma.item()) == g_ref
    ref = oracle.pack_ternary(oracle.ternarize(W, g_ref))
    np.testing.assert_array_equal(Wp.cpu().numpy().view(np.uint32).reshape(N, K // 16), ref)


def test_weights_degenerate(B):
    Z = np.zeros((16, 128), np.uint16)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(Z))
    assert np.float32(gamma.item()) == np.float32(1e-5)
    q, bad = oracle.unpack_ternary(Wp.cpu().numpy().view(np.uint32), 128)
    assert bad == 0 and not q.any()


# ----------------------------------------------------------------------------------------
# steps 2-3: Hadamard transform and quantisation
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("K", [128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768])
def test_fwht_matches_oracle(B, K):
    M = 37 if K <= 8192 else 9
    X = synth.sharp_activations(M, K, seed=K)
    Z = B.bitnet_fwht_f32(dev_bf16(X)).cpu().numpy().astype(np.float64)
    ref = oracle.fwht(oracle.bf16_to_f64(X))
    err = np.abs(Z - ref).max(axis=1) / np.abs(ref).max(axis=1)
    assert err.max() <= FWHT_REL, err.max()


@pytest.mark.parametrize("K", [128, 256, 2048, 8192, 16384])
@pytest.mark.parametrize("bits", [8, 4])
def test_hadamard_quant_codes(B, K, bits):
    M = 45 if K <= 8192 else 11
    X = synth.sharp_activations(M, K, seed=3 * K + bits)
    Xd = dev_bf16(X)
    z = B.bitnet_fwht_f32(Xd).cpu().numpy()
    codes, scales, rowsum = B.bitnet_act_quant(Xd, True, bits)
    c_ref, d_ref, pre, rs_ref = oracle.quant_act(z, bits)
    c = codes.cpu().numpy()
    c = c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)
    n_diff = check_codes(c, c_ref, pre)
    assert n_diff == 0, f"{n_diff} codes differ (within the boundary tolerance)"
    np.testing.assert_allclose(scales.cpu().numpy(), d_ref, rtol=1e-6)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), c.astype(np.int64).sum(axis=1))


@pytest.mark.parametrize("K", [128, 640, 4096])
@pytest.mark.parametrize("bits", [8, 4])
def test_plain_quant_codes_exact(B, K, bits):
    M = 21
    X = synth.gaussian_activations(M, K, seed=K + bits)
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), False, bits)
    z = oracle.bf16_to_f64(X).astype(np.float32)
    c_ref, d_ref, _, rs_ref = oracle.quant_act(z, bits)
    c = codes.cpu().numpy()
    c = c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)
    np.testing.assert_array_equal(c, c_ref)
    np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), rs_ref)


def test_quant_zero_rows(B):
    X = np.zeros((5, 256), np.uint16)
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), True, 8)
    assert not codes.cpu().numpy().any()
    assert np.all(scales.cpu().numpy() == np.float32(np.float32(1e-5) / np.float32(127)))
    assert not rowsum.cpu().numpy().any()


# ----------------------------------------------------------------------------------------
# step 4: product, staged on the GPU's own codes
# ----------------------------------------------------------------------------------------

def staged_product(B, M, K, N, bits, seed):
    X = synth.sharp_activations(M, K, seed=seed)
    W = synth.latent_weights(N, K, seed=seed + 1)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    hadamard = (K & (K - 1)) == 0
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), hadamard, bits)
    acc, Y = B.bitnet_ternary_gemm(codes, scales, rowsum, K, Wp, gamma, bits, want_acc=True,
                                   want_y=True)
    B.bitnet_sync_status()
    c = codes.cpu().numpy()
    c = c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)
    q, bad = oracle.unpack_ternary(Wp.cpu().numpy().view(np.uint32), K)
    assert bad == 0
    return c, q, scales.cpu().numpy(), np.float32(gamma.item()), acc.cpu().numpy(), Y


@pytest.mark.parametrize("M,K,N", [
    (1, 256, 256), (3, 384, 136), (8, 2048, 264),          # decode kernel
    (1, 8320, 136), (2, 4096, 8), (6, 8320, 264),           # decode, rows split over 2 / 4 warps
    (8, 16384, 520), (4, 32768, 16),                        # (17 steps: uneven split)
    (7, 4096, 8200),                                        # decode, 4-row groups
    (9, 256, 256), (130, 384, 136), (300, 2048, 264),       # tensor-core kernel, ragged tiles
    (64, 8192, 2048), (17, 4096, 1032),                     # tensor cores with the K split
    (256, 1024, 1024), (513, 128, 8),
    (1000, 640, 520),                                       # several tiles, 2.5 K stages
])
@pytest.mark.parametrize("bits", [8, 4])
def test_product_int32_exact_and_bf16(B, M, K, N, bits):
    c, q, d, gamma, acc, Y = staged_product(B, M, K, N, bits, seed=M * 7 + N)
    acc_ref = oracle.gemm_i64(c, q)
    np.testing.assert_array_equal(acc.astype(np.int64), acc_ref)
    y_ref = oracle.bf16_to_f64(oracle.dequant(acc_ref, d, gamma))
    y = oracle.bf16_to_f64(to_np_bits(Y))
    rel = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), 1e-30)
    assert np.all((rel <= Y_REL) | (y_ref == 0)), rel.max()
    assert np.all(y[y_ref == 0] == 0)


# ----------------------------------------------------------------------------------------
# the whole layer against the independent oracle, on every workload shape
# ----------------------------------------------------------------------------------------

def forward_case(B, wl, sample_rows, seed=0):
    X = wl.activations(seed=seed)
    W = wl.weights(seed=seed)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    fwd = B.bitnet_hbitlinear_forward if wl.hadamard else B.bitnet_bitlinear_forward
    Y = fwd(dev_bf16(X), Wp, gamma, wl.act_bits)
    B.bitnet_sync_status()
    rows = np.arange(wl.M) if sample_rows is None else np.sort(
        np.random.default_rng(seed).choice(wl.M, size=sample_rows, replace=False))
    ref = oracle.bitlinear_forward(X[rows], W, wl.hadamard, wl.act_bits)
    assert np.float32(gamma.item()) == ref["gamma"]
    y = oracle.bf16_to_f64(to_np_bits(Y)[rows])
    y_ref = oracle.bf16_to_f64(ref["y"])
    fro = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert fro <= Y_REL, fro
    return fro


@pytest.mark.parametrize("name,rows", [
    ("tiny", None),
    ("wo_2048", 64),
    ("wdown_8192", 24),
    ("decode_m1_k8192", None), ("decode_m8_k8192", None), ("decode_m32_k8192", None),
    ("decode_m64_k8192", None), ("decode_m1_k2048", None), ("decode_m64_k2048", None),
])
def test_forward_end_to_end(B, name, rows):
    forward_case(B, synth.WORKLOADS[name], rows)


@pytest.mark.parametrize("name,rows", [("down_7b", 6), ("up_7b", 8)])
def test_forward_end_to_end_7b(B, name, rows):
    forward_case(B, synth.WORKLOADS[name], rows)


def test_forward_equals_staged_calls(B):
    wl = synth.WORKLOADS["wo_2048"]
    X = dev_bf16(wl.activations(rows=640))
    W = dev_bf16(wl.weights())
    Wp, gamma = B.bitnet_quantize_pack_weights(W)
    Y = B.bitnet_hbitlinear_forward(X, Wp, gamma, 8)
    codes, scales, rowsum = B.bitnet_act_quant(X, True, 8)
    _, Y2 = B.bitnet_ternary_gemm(codes, scales, rowsum, wl.K, Wp, gamma, 8)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_errors_are_reported(B):
    X = torch.zeros((4, 384), dtype=torch.bfloat16, device="cuda")
    Wp = torch.zeros((8, 96), dtype=torch.uint8, device="cuda")
    gamma = torch.ones(1, device="cuda")
    with pytest.raises(B.BitnetError) as e:
        B.bitnet_hbitlinear_forward(X, Wp, gamma, 8)  # 384 is not a power of two
    assert e.value.status == B.ERR_UNSUPPORTED
    Y = B.bitnet_bitlinear_forward(X, Wp, gamma, 8)  # fine without the transform
    B.bitnet_sync_status()
    assert not Y.float().abs().sum().item()


# ----------------------------------------------------------------------------------------
# failure detection: a bounded device wait that runs out is reported, and nothing is lost
# ----------------------------------------------------------------------------------------

def test_bounded_wait_time_out_is_reported_and_context_survives(B):
    B.bitnet_sync_status()                       # nothing pending
    B.bitnet_selftest_wait_timeout(2_000_000)    # ~1 ms of waiting on a barrier nobody arrives on
    with pytest.raises(B.BitnetError) as err:
        B.bitnet_sync_status()
    assert err.value.status == B.ERR_TIMEOUT
    assert B.bitnet_sync_status() == B.OK        # the flag was cleared
    # the context is still usable: a small forward matches the oracle
    wl = synth.WORKLOADS["tiny"]
    forward_case(B, wl, None)


# ----------------------------------------------------------------------------------------
# RMS normalisation fused into the quantiser (2B4T article, 一.3: subln normalisation;
# BitNet v2 write-up: RMS normalisation).  The normalised rows are fp32 on the GPU and double
# in the oracle, so they are held to the transform's tolerance; codes are then exact on the
# GPU's own rows.
# ----------------------------------------------------------------------------------------

NORM_EPS = 1e-5


def gain_bits(K, seed):
    g = np.random.default_rng(seed).uniform(0.5, 1.5, K).astype(np.float32)
    return synth.f32_to_bf16_bits(g)


def dev_gain(bits):
    return None if bits is None else synth.to_torch_bf16(bits).cuda()


NORM_CASES = [(128, True), (2048, True), (8192, True), (16384, True),
              (384, False), (2048, False)]


@pytest.mark.parametrize("K,hadamard", NORM_CASES)
@pytest.mark.parametrize("with_gain", [True, False])
def test_norm_transform_matches_oracle(B, K, hadamard, with_gain):
    M = 29 if K <= 8192 else 7
    X = synth.sharp_activations(M, K, seed=K + 5)
    g = gain_bits(K, K) if with_gain else None
    Z = B.bitnet_norm_transform_f32(dev_bf16(X), dev_gain(g), NORM_EPS, hadamard)
    Z = Z.cpu().numpy().astype(np.float64)
    ref = oracle.rmsnorm(oracle.bf16_to_f64(X), g, NORM_EPS)
    if hadamard:
        ref = oracle.fwht(ref)
    err = np.abs(Z - ref).max(axis=1) / np.abs(ref).max(axis=1)
    assert err.max() <= FWHT_REL, err.max()


@pytest.mark.parametrize("K,hadamard", NORM_CASES)
@pytest.mark.parametrize("bits", [8, 4])
def test_norm_quant_codes_exact_on_the_gpu_rows(B, K, hadamard, bits):
    M = 33 if K <= 8192 else 9
    X = synth.sharp_activations(M, K, seed=7 * K + bits)
    g = gain_bits(K, K + 1)
    Xd, gd = dev_bf16(X), dev_gain(g)
    z = B.bitnet_norm_transform_f32(Xd, gd, NORM_EPS, hadamard).cpu().numpy()
    codes, scales, rowsum = B.bitnet_act_quant_norm(Xd, gd, NORM_EPS, hadamard, bits)
    c_ref, d_ref, pre, rs_ref = oracle.quant_act(z, bits)
    c = codes.cpu().numpy()
    c = c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)
    assert check_codes(c, c_ref, pre) == 0
    np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), rs_ref)


@pytest.mark.parametrize("name,hadamard,rows", [
    ("wo_2048", True, 48), ("wdown_8192", True, 16), ("decode_m8_k8192", True, None),
    ("tiny", False, None), ("decode_m32_k2048", False, None),
])
def test_norm_forward_end_to_end(B, name, hadamard, rows):
    wl = synth.WORKLOADS[name]
    X, W = wl.activations(seed=1), wl.weights(seed=1)
    g = gain_bits(wl.K, 99)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    Y = B.bitnet_norm_bitlinear_forward(dev_bf16(X), dev_gain(g), NORM_EPS, hadamard, Wp, gamma,
                                        wl.act_bits)
    B.bitnet_sync_status()
    sel = np.arange(wl.M) if rows is None else np.sort(
        np.random.default_rng(1).choice(wl.M, size=rows, replace=False))
    ref = oracle.bitlinear_forward(X[sel], W, hadamard, wl.act_bits, norm_gain=g,
                                   norm_eps=NORM_EPS)
    y = oracle.bf16_to_f64(to_np_bits(Y)[sel])
    y_ref = oracle.bf16_to_f64(ref["y"])
    assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) <= Y_REL


def test_norm_rejects_bad_eps(B):
    X = dev_bf16(synth.sharp_activations(4, 256, seed=1))
    for eps in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(B.BitnetError) as err:
            B.bitnet_act_quant_norm(X, None, eps, True, 8)
        assert err.value.status == B.ERR_INVALID


# ----------------------------------------------------------------------------------------
# activations fused into the product's epilogue (2B4T article, 一.3: squared ReLU; BitNet v2
# write-up: SwishGLU), staged on the GPU's codes and end to end
# ----------------------------------------------------------------------------------------

def check_act(Y, y_ref_bits):
    y = oracle.bf16_to_f64(to_np_bits(Y))
    y_ref = oracle.bf16_to_f64(y_ref_bits)
    assert y.shape == y_ref.shape
    rel = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), 1e-30)
    assert np.all((rel <= Y_REL) | (y_ref == 0)), rel.max()
    # squared ReLU: zeros exactly where the accumulator is <= 0; SwiGLU: silu(0) * u = 0
    assert np.all(np.abs(y[y_ref == 0]) <= 1e-30)


@pytest.mark.parametrize("M,K,N", [
    (1, 256, 256), (5, 2048, 272), (8, 384, 528),               # decode kernel
    (8, 8320, 272), (2, 4096, 528),                             # decode, split rows
    (8, 2048, 8192),                                            # decode, 4-row groups
    (9, 256, 256), (300, 2048, 272), (1000, 640, 528),          # tensor-core kernel
])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("act", [1, 2])
def test_product_activation_matches_oracle(B, M, K, N, bits, act):
    X = synth.sharp_activations(M, K, seed=M + K)
    W = synth.latent_weights(N, K, seed=N + 3)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    hadamard = (K & (K - 1)) == 0
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), hadamard, bits)
    acc, _ = B.bitnet_ternary_gemm(codes, scales, rowsum, K, Wp, gamma, bits, want_acc=True,
                                   want_y=False)
    Y = B.bitnet_ternary_gemm_act(codes, scales, rowsum, K, Wp, gamma, bits, act)
    B.bitnet_sync_status()
    c = codes.cpu().numpy()
    c = c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)
    q, _ = oracle.unpack_ternary(Wp.cpu().numpy().view(np.uint32), K)
    acc_ref = oracle.gemm_i64(c, q)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    check_act(Y, oracle.dequant_act(acc_ref, scales.cpu().numpy(), np.float32(gamma.item()), act))


@pytest.mark.parametrize("name,act", [("up_7b", 1), ("up_7b", 2), ("tiny", 2),
                                      ("decode_m8_k2048", 1), ("decode_m1_k8192", 2)])
def test_forward_activation_end_to_end(B, name, act):
    wl = synth.WORKLOADS[name]
    rows = 24 if wl.M > 64 else None
    X, W = wl.activations(seed=2), wl.weights(seed=2)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    Y = B.bitnet_bitlinear_forward_act(dev_bf16(X), Wp, gamma, wl.act_bits, wl.hadamard, act)
    B.bitnet_sync_status()
    sel = np.arange(wl.M) if rows is None else np.sort(
        np.random.default_rng(2).choice(wl.M, size=rows, replace=False))
    ref = oracle.bitlinear_forward(X[sel], W, wl.hadamard, wl.act_bits)
    y_ref = oracle.bf16_to_f64(oracle.dequant_act(ref["acc"], ref["d"], ref["gamma"], act))
    y = oracle.bf16_to_f64(to_np_bits(Y)[sel])
    assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) <= Y_REL


# ----------------------------------------------------------------------------------------
# base-3 weights for decode (2B4T article, section 一.1: five ternary weights a byte)
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(256, 256), (8, 128), (264, 384), (16, 640), (2048, 2048),
                                 (520, 8192), (8, 32768)])
def test_base3_weights_bit_exact(B, N, K):
    W = synth.latent_weights(N, K, seed=N + 2 * K)
    Wp3, gamma = B.bitnet_quantize_pack_weights_base3(dev_bf16(W))
    B.bitnet_sync_status()
    g_ref = oracle.absmean_gamma(W)
    assert np.float32(gamma.item()) == g_ref
    words = (K + 19) // 20
    ref = oracle.pack_ternary_base3(oracle.ternarize(W, g_ref))
    got = Wp3.cpu().numpy().view(np.uint32).reshape(N, words)
    np.testing.assert_array_equal(got, ref)


def test_base3_weights_degenerate(B):
    # all-zero weights: gamma = 1e-5, every weight q = 0 (u = 1), padding too: byte 121
    Z = np.zeros((16, 128), np.uint16)
    Wp3, gamma = B.bitnet_quantize_pack_weights_base3(dev_bf16(Z))
    B.bitnet_sync_status()
    assert np.float32(gamma.item()) == np.float32(1e-5)
    assert np.all(Wp3.cpu().numpy() == 121)


@pytest.mark.parametrize("M,K,N", [
    (1, 128, 8), (1, 2048, 264), (2, 384, 136), (3, 640, 256), (4, 8192, 520),
    (5, 256, 8), (8, 2048, 1032), (8, 32768, 16), (1, 10880, 136), (6, 5120, 264),
])
def test_base3_product_int32_exact_and_bf16(B, M, K, N):
    X = synth.sharp_activations(M, K, seed=M * 3 + K)
    W = synth.latent_weights(N, K, seed=N + 5)
    Wp3, gamma = B.bitnet_quantize_pack_weights_base3(dev_bf16(W))
    hadamard = (K & (K - 1)) == 0
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), hadamard, 8)
    acc, Y = B.bitnet_ternary_gemv_base3(codes, scales, rowsum, K, Wp3, gamma, want_acc=True)
    B.bitnet_sync_status()
    c = codes.cpu().numpy().view(np.int8)
    q, bad = oracle.unpack_ternary_base3(Wp3.cpu().numpy().view(np.uint32), K)
    assert bad == 0
    np.testing.assert_array_equal(q, oracle.ternarize(W, oracle.absmean_gamma(W)))
    acc_ref = oracle.gemm_i64(c, q)
    np.testing.assert_array_equal(acc.cpu().numpy().astype(np.int64), acc_ref)
    y_ref = oracle.bf16_to_f64(oracle.dequant(acc_ref, scales.cpu().numpy(),
                                              np.float32(gamma.item())))
    y = oracle.bf16_to_f64(to_np_bits(Y))
    rel = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), 1e-30)
    assert np.all((rel <= Y_REL) | (y_ref == 0)), rel.max()
    assert np.all(y[y_ref == 0] == 0)


@pytest.mark.parametrize("M,K,N", [(1, 2048, 272), (4, 640, 528), (8, 8192, 1040),
                                   (8, 1280, 8208)])
@pytest.mark.parametrize("act", [1, 2])
def test_base3_product_activation_matches_oracle(B, M, K, N, act):
    X = synth.sharp_activations(M, K, seed=M + 2 * K)
    W = synth.latent_weights(N, K, seed=N + 7)
    Wp3, gamma = B.bitnet_quantize_pack_weights_base3(dev_bf16(W))
    hadamard = (K & (K - 1)) == 0
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), hadamard, 8)
    _, Y = B.bitnet_ternary_gemv_base3(codes, scales, rowsum, K, Wp3, gamma, act)
    B.bitnet_sync_status()
    q = oracle.ternarize(W, oracle.absmean_gamma(W))
    acc_ref = oracle.gemm_i64(codes.cpu().numpy().view(np.int8), q)
    check_act(Y, oracle.dequant_act(acc_ref, scales.cpu().numpy(), np.float32(gamma.item()), act))


@pytest.mark.parametrize("name,act", [("decode_m1_k8192", 0), ("decode_m8_k8192", 0),
                                      ("decode_m1_k2048", 0), ("decode_m8_k2048", 2),
                                      ("decode_m1_k8192", 1)])
def test_base3_forward_end_to_end(B, name, act):
    wl = synth.WORKLOADS[name]
    assert wl.act_bits == 8
    X, W = wl.activations(seed=4), wl.weights(seed=4)
    Wp3, gamma = B.bitnet_quantize_pack_weights_base3(dev_bf16(W))
    Y = B.bitnet_bitlinear_forward_base3(dev_bf16(X), Wp3, gamma, wl.hadamard, act)
    B.bitnet_sync_status()
    ref = oracle.bitlinear_forward(X, W, wl.hadamard, 8)
    assert np.float32(gamma.item()) == ref["gamma"]
    y_ref = ref["y"] if act == 0 else oracle.dequant_act(ref["acc"], ref["d"], ref["gamma"], act)
    y_ref = oracle.bf16_to_f64(y_ref)
    y = oracle.bf16_to_f64(to_np_bits(Y))
    assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) <= Y_REL


def test_base3_product_equals_two_bit_product(B):
    # the same ternary matrix in both layouts gives the same integers and the same bf16 outputs
    M, K, N = 8, 4096, 776
    X = synth.sharp_activations(M, K, seed=11)
    W = dev_bf16(synth.latent_weights(N, K, seed=12))
    Wp, g2 = B.bitnet_quantize_pack_weights(W)
    Wp3, g3 = B.bitnet_quantize_pack_weights_base3(W)
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), True, 8)
    a2, y2 = B.bitnet_ternary_gemm(codes, scales, rowsum, K, Wp, g2, 8, want_acc=True)
    a3, y3 = B.bitnet_ternary_gemv_base3(codes, scales, rowsum, K, Wp3, g3, want_acc=True)
    B.bitnet_sync_status()
    assert g2.item() == g3.item()
    assert torch.equal(a2, a3)
    assert torch.equal(y2.view(torch.int16), y3.view(torch.int16))


# ----------------------------------------------------------------------------------------
# variant INT4 quantiser with a per-token absmean scale
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("K", [128, 256, 2048, 4096, 8192, 16384, 32768])
def test_absmean4_hadamard_codes(B, K):
    M = 37 if K <= 8192 else 9
    X = synth.sharp_activations(M, K, seed=5 * K + 1)
    Xd = dev_bf16(X)
    z = B.bitnet_fwht_f32(Xd).cpu().numpy()
    codes, scales, rowsum = B.bitnet_act_quant_absmean4(Xd, True)
    B.bitnet_sync_status()
    c_ref, d_ref, pre, _ = oracle.quant_act_absmean4(z)
    c = oracle.unpack_int4(codes.cpu().numpy().view(np.uint8), K)
    n_diff = check_codes(c, c_ref, pre)
    assert n_diff == 0, f"{n_diff} codes differ (within the boundary tolerance)"
    np.testing.assert_allclose(scales.cpu().numpy(), d_ref, rtol=1e-6)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), c.astype(np.int64).sum(axis=1))
    assert (c == 7).any() or (c == -8).any()  # the clip is exercised


@pytest.mark.parametrize("K", [128, 640, 4096])
def test_absmean4_plain_codes(B, K):
    M = 19
    X = synth.gaussian_activations(M, K, seed=K + 17)
    X[3] = 0  # a zero row: zero codes, guarded scale
    codes, scales, rowsum = B.bitnet_act_quant_absmean4(dev_bf16(X), False)
    B.bitnet_sync_status()
    z = oracle.bf16_to_f64(X).astype(np.float32)
    c_ref, d_ref, pre, rs_ref = oracle.quant_act_absmean4(z)
    c = oracle.unpack_int4(codes.cpu().numpy().view(np.uint8), K)
    assert check_codes(c, c_ref, pre) == 0
    np.testing.assert_allclose(scales.cpu().numpy(), d_ref, rtol=1e-6)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), rs_ref)
    assert not c[3].any()


@pytest.mark.parametrize("name,rows", [("wdown_8192", 16), ("tiny", None)])
def test_absmean4_forward_end_to_end(B, name, rows):
    wl = synth.WORKLOADS[name]
    X, W = wl.activations(seed=6), wl.weights(seed=6)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    Y = B.bitnet_bitlinear_forward_absmean4(dev_bf16(X), Wp, gamma, wl.hadamard)
    B.bitnet_sync_status()
    sel = np.arange(wl.M) if rows is None else np.sort(
        np.random.default_rng(6).choice(wl.M, size=rows, replace=False))
    x = oracle.bf16_to_f64(X[sel])
    z = (oracle.fwht(x) if wl.hadamard else x).astype(np.float32)
    codes, d, _, _ = oracle.quant_act_absmean4(z)
    g = oracle.absmean_gamma(W)
    assert np.float32(gamma.item()) == g
    acc = oracle.gemm_i64(codes, oracle.ternarize(W, g))
    y_ref = oracle.bf16_to_f64(oracle.dequant(acc, d, g))
    y = oracle.bf16_to_f64(to_np_bits(Y)[sel])
    assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) <= Y_REL


# ----------------------------------------------------------------------------------------
# variant: weight + activation Hadamard rotation (the weight half)
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(256, 256), (8, 128), (264, 2048), (1032, 8192), (16, 32768)])
def test_rotated_weights_bit_exact_on_the_gpu_rotation(B, N, K):
    W = synth.latent_weights(N, K, seed=N + 3 * K)
    Wd = dev_bf16(W)
    Wp, gamma = B.bitnet_quantize_pack_weights_rotated(Wd)
    Wr = B.bitnet_fwht_f32(Wd).cpu().numpy()  # the same transform, as fp32 rows
    B.bitnet_sync_status()
    g_ref = oracle.absmean_gamma_f32(Wr)
    assert np.float32(gamma.item()) == g_ref
    ref = oracle.pack_ternary(oracle.ternarize_f32(Wr, g_ref))
    np.testing.assert_array_equal(Wp.cpu().numpy().view(np.uint32).reshape(N, K // 16), ref)
    # the GPU rotation against the oracle's double transform
    Wr_ref = oracle.rotate_weights(W)
    err = np.abs(Wr - Wr_ref).max(axis=1) / np.abs(Wr_ref).max(axis=1)
    assert err.max() <= FWHT_REL


def test_rotated_weights_degenerate(B):
    Wp, gamma = B.bitnet_quantize_pack_weights_rotated(dev_bf16(np.zeros((16, 256), np.uint16)))
    B.bitnet_sync_status()
    assert np.float32(gamma.item()) == np.float32(1e-5)
    q, bad = oracle.unpack_ternary(Wp.cpu().numpy().view(np.uint32), 256)
    assert bad == 0 and not q.any()


@pytest.mark.parametrize("name,rows", [("tiny", None), ("wo_2048", 32), ("wdown_8192", 8)])
def test_rotated_forward_end_to_end(B, name, rows):
    wl = synth.WORKLOADS[name]
    X, W = wl.activations(seed=8), wl.weights(seed=8)
    Wp, gamma = B.bitnet_quantize_pack_weights_rotated(dev_bf16(W))
    Y = B.bitnet_hbitlinear_forward(dev_bf16(X), Wp, gamma, wl.act_bits)
    B.bitnet_sync_status()
    sel = np.arange(wl.M) if rows is None else np.sort(
        np.random.default_rng(8).choice(wl.M, size=rows, replace=False))
    z = oracle.fwht(oracle.bf16_to_f64(X[sel])).astype(np.float32)
    codes, d, _, _ = oracle.quant_act(z, wl.act_bits)
    Wr = oracle.rotate_weights(W)
    g = oracle.absmean_gamma_f32(Wr)
    assert abs(np.float32(gamma.item()) / g - 1) <= 1e-6
    acc = oracle.gemm_i64(codes, oracle.ternarize_f32(Wr, g))
    y_ref = oracle.bf16_to_f64(oracle.dequant(acc, d, g))
    y = oracle.bf16_to_f64(to_np_bits(Y)[sel])
    assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) <= Y_REL
