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
import math

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
    """Codes may differ by +-1 only within CODE_BOUNDARY of a .5 boundary, on at most a fraction
    CODE_FRACTION of the elements: at most floor(CODE_FRACTION * n) of n codes, and at least one
    allowed (below 10^4 codes a single near-tie flip already exceeds the rate)."""
    diff = codes_gpu.astype(np.int32) - codes_ref.astype(np.int32)
    bad = diff != 0
    if bad.any():
        assert np.abs(diff).max() <= 1
        dist = np.abs(np.abs(pre[bad] - np.floor(pre[bad])) - 0.5)
        assert np.all(dist < CODE_BOUNDARY), dist.max()
        assert bad.sum() <= max(1, math.floor(CODE_FRACTION * bad.size)), bad.sum()
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
    c_ref, d_ref, pre, rs_ref = oracle.quant_act_for_bits(z, bits)
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
    X[3] = 0  # a zero row: zero codes, guarded scale
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), False, bits)
    z = oracle.bf16_to_f64(X).astype(np.float32)
    c_ref, d_ref, pre, rs_ref = oracle.quant_act_for_bits(z, bits)
    c = codes.cpu().numpy()
    c = c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)
    assert check_codes(c, c_ref, pre) == 0
    if bits == 8:
        np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)
    else:  # the absmean sum is taken in double in another order: the scale may move by an ulp
        np.testing.assert_allclose(scales.cpu().numpy(), d_ref, rtol=1e-6)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), rs_ref)
    assert not c[3].any()


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
    (9, 256, 256), (64, 8192, 2048), (17, 4096, 1032),      # skinny tensor-core kernel
    (130, 384, 136), (300, 2048, 264),                      # 256 x 256 tiles, ragged
    (256, 1024, 1024), (513, 128, 8),
    (1000, 640, 520),                                       # several tiles, 2.5 K stages
    (65, 8192, 8), (700, 8448, 264),                        # INT4: tensor-memory kernel
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


def sample_rows(M, count, seed):
    """A seeded sorted sample of token rows that always holds the first and the last row (the
    ragged tail of the last tile)."""
    if count is None or count >= M:
        return np.arange(M)
    rows = np.random.default_rng(seed).choice(np.arange(1, M - 1), size=count - 2, replace=False)
    return np.sort(np.concatenate([[0, M - 1], rows]))


def codes_rows(codes, rows, K, bits):
    c = codes[torch.from_numpy(rows).to(codes.device)].cpu().numpy()
    return c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)


# The skinny tensor-core product (9 <= M <= 64: 128 features per CTA, weights unpacked into
# tensor memory, K split over a cluster and summed through distributed shared memory): every
# token tile (16 / 32 / 64), ragged token counts, ragged N, K with a partial last 512-stage, both
# code widths and every cluster size the launcher picks.  int32 bit-exact on all rows.
@pytest.mark.parametrize("M,K,N", [
    (9, 128, 8), (16, 640, 136), (17, 2048, 8192), (32, 8192, 2048), (33, 1152, 264),
    (48, 16384, 4096), (63, 4096, 1032), (64, 2048, 8192), (64, 8192, 2048), (40, 384, 16384),
])
@pytest.mark.parametrize("bits", [8, 4])
def test_skinny_product_int32_exact_and_bf16(B, M, K, N, bits):
    path, split = B.bitnet_product_plan(M, K, N, bits)
    assert path == B.PATH_TC_SKINNY and 1 <= split <= min(8, (K + 511) // 512)
    c, q, d, gamma, acc, Y = staged_product(B, M, K, N, bits, seed=M * 11 + N)
    acc_ref = oracle.gemm_i64(c, q)
    np.testing.assert_array_equal(acc.astype(np.int64), acc_ref)
    y_ref = oracle.bf16_to_f64(oracle.dequant(acc_ref, d, gamma))
    y = oracle.bf16_to_f64(to_np_bits(Y))
    rel = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), 1e-30)
    assert np.all((rel <= Y_REL) | (y_ref == 0)), rel.max()
    assert np.all(y[y_ref == 0] == 0)


def test_product_paths_by_token_count(B):
    for M, path in ((1, B.PATH_DECODE), (8, B.PATH_DECODE), (9, B.PATH_TC_SKINNY),
                    (64, B.PATH_TC_SKINNY), (65, B.PATH_TC), (4096, B.PATH_TC)):
        assert B.bitnet_product_plan(M, 2048, 2048, 8)[0] == path, M
    for M, path in ((8, B.PATH_DECODE), (64, B.PATH_TC_SKINNY), (65, B.PATH_TC_TMEM),
                    (16384, B.PATH_TC_TMEM)):
        assert B.bitnet_product_plan(M, 8192, 2048, 4)[0] == path, M
    # INT4 below K = 8192 stays on the shared-memory kernel
    assert B.bitnet_product_plan(4096, 4096, 2048, 4)[0] == B.PATH_TC


def test_concurrent_forwards_on_two_streams(B):
    """Two decode-size forwards (skinny tensor-core product, K split over clusters) issued on two
    streams with no ordering between them: no state is shared, so both match the oracle."""
    wls = [synth.WORKLOADS["decode_m64_k8192"], synth.WORKLOADS["decode_m32_k2048"]]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    inputs = []
    for i, wl in enumerate(wls):
        X, W = wl.activations(seed=20 + i), wl.weights(seed=20 + i)
        Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
        inputs.append((X, W, dev_bf16(X), Wp, gamma))
    torch.cuda.synchronize()
    outs = []
    for _ in range(3):  # several rounds so the launches overlap
        for (X, W, Xd, Wp, gamma), wl, st in zip(inputs, wls, streams):
            with torch.cuda.stream(st):
                outs.append(B.bitnet_hbitlinear_forward(Xd, Wp, gamma, wl.act_bits, stream=st))
    torch.cuda.synchronize()
    B.bitnet_sync_status()
    for r in range(3):
        for i, ((X, W, _, _, _), wl) in enumerate(zip(inputs, wls)):
            ref = oracle.bitlinear_forward(X, W, wl.hadamard, wl.act_bits)
            y = oracle.bf16_to_f64(to_np_bits(outs[2 * r + i]))
            y_ref = oracle.bf16_to_f64(ref["y"])
            assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) <= Y_REL


# The one-pass tensor-core product at the sizes the benchmark runs: many K stages per tile
# (the operand rings wrap), more tiles than SM pairs (the persistent tile loop and both
# accumulator buffers of tensor memory are used), ragged token and feature tails, and a half
# last stage (K % 256 == 128).  int32 bit-exact on a seeded sample of rows x all features;
# bf16 elementwise on the same rows.
@pytest.mark.parametrize("M,K,N,bits,name", [
    (4096, 2048, 2048, 8, "wo_2048"),
    (8192, 8192, 2048, 4, "wdown_8192"),
    (16384, 16384, 4096, 4, "down_7b"),
    (4000, 2048, 2056, 8, None),
    (3000, 1152, 3080, 4, None),
    (3000, 8320, 3080, 4, None),   # tensor-memory kernel: ragged M and N, half last stage
])
def test_product_one_pass_full_size_bit_exact(B, M, K, N, bits, name):
    path, split = B.bitnet_product_plan(M, K, N, bits)
    expect = B.PATH_TC_TMEM if bits == 4 and K >= 8192 else B.PATH_TC
    assert (path, split) == (expect, 1), "this shape must take the one-pass kernel"
    if name is not None:
        wl = synth.WORKLOADS[name]
        X, W = wl.activations(seed=3), wl.weights(seed=3)
    else:
        X = synth.sharp_activations(M, K, seed=M + K)
        W = synth.latent_weights(N, K, seed=N + K)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    hadamard = (K & (K - 1)) == 0
    Xd = dev_bf16(X)
    del X
    codes, scales, rowsum = B.bitnet_act_quant(Xd, hadamard, bits)
    acc, Y = B.bitnet_ternary_gemm(codes, scales, rowsum, K, Wp, gamma, bits, want_acc=True,
                                   want_y=True)
    B.bitnet_sync_status()
    rows = sample_rows(M, 64, seed=M)
    sel = torch.from_numpy(rows).cuda()
    c = codes_rows(codes, rows, K, bits)
    q, bad = oracle.unpack_ternary(Wp.cpu().numpy().view(np.uint32), K)
    assert bad == 0
    acc_ref = oracle.gemm_i64(c, q)
    np.testing.assert_array_equal(acc[sel].cpu().numpy().astype(np.int64), acc_ref)
    y_ref = oracle.bf16_to_f64(oracle.dequant(acc_ref, scales[sel].cpu().numpy(),
                                              np.float32(gamma.item())))
    y = oracle.bf16_to_f64(to_np_bits(Y[sel]))
    rel = np.abs(y - y_ref) / np.maximum(np.abs(y_ref), 1e-30)
    assert np.all((rel <= Y_REL) | (y_ref == 0)), rel.max()
    assert np.all(y[y_ref == 0] == 0)


# ----------------------------------------------------------------------------------------
# the whole layer against the independent oracle, on every workload shape
# ----------------------------------------------------------------------------------------

def forward_case(B, wl, sample_count, seed=0):
    """The GPU forward against the fully independent oracle on sampled rows.

    Besides the Frobenius bound, every sampled element is checked: the GPU's codes may differ
    from the oracle's by +-1 at near-ties (the GPU's fp32 transform is not the oracle's double
    one), and each such code moves an accumulator by at most 1, i.e. y by at most d * gamma.
    So |y - y_ref| <= Y_REL |y_ref| + flips(m) * d_m * gamma, flips(m) being the number of
    codes of row m that differ (themselves held to the code tolerance)."""
    X = wl.activations(seed=seed)
    W = wl.weights(seed=seed)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    fwd = B.bitnet_hbitlinear_forward if wl.hadamard else B.bitnet_bitlinear_forward
    Xd = dev_bf16(X)
    Y = fwd(Xd, Wp, gamma, wl.act_bits)
    codes, _, _ = B.bitnet_act_quant(Xd, wl.hadamard, wl.act_bits)  # the forward's own codes
    B.bitnet_sync_status()
    rows = sample_rows(wl.M, sample_count, seed)
    ref = oracle.bitlinear_forward(X[rows], W, wl.hadamard, wl.act_bits)
    assert np.float32(gamma.item()) == ref["gamma"]
    c = codes_rows(codes, rows, wl.K, wl.act_bits)
    _, _, pre, _ = oracle.quant_act_for_bits(ref["z"].astype(np.float32), wl.act_bits)
    check_codes(c, ref["codes"], pre)
    flips = (c != ref["codes"]).sum(axis=1)
    y = oracle.bf16_to_f64(to_np_bits(Y)[rows])
    y_ref = oracle.bf16_to_f64(ref["y"])
    fro = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert fro <= Y_REL, fro
    slack = flips[:, None] * ref["d"][:, None].astype(np.float64) * float(ref["gamma"])
    bound = Y_REL * np.abs(y_ref) + slack * (1 + 1e-6)
    assert np.all(np.abs(y - y_ref) <= bound), np.abs(y - y_ref).max()
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


# ----------------------------------------------------------------------------------------
# the method's edge cases on the GPU
# ----------------------------------------------------------------------------------------

def bf16_exact(a):
    """bf16 bits of values that bf16 holds exactly (asserted)."""
    a = np.asarray(a, np.float32)
    bits = synth.f32_to_bf16_bits(a)
    assert np.array_equal(oracle.bf16_to_f64(bits), a.astype(np.float64))
    return bits


def test_weights_on_the_ternary_threshold(B):
    """Weights exactly at |w| = gamma / 2 and at the bf16 neighbours of that value.

    3/8 of the weights are +-1, half are +-1/4 and 1/8 are zero, so gamma = 1/2 exactly and
    1/4 lies on the threshold: w / gamma = 0.5 rounds to the even 0.  Triples (1/4 + 2^-9,
    1/4 - 2^-10, 1/4 - 2^-10) keep the sum, and so gamma, unchanged: the first is the bf16 value
    just above the threshold (code +-1), the others just below it (code 0)."""
    N, K = 64, 256
    rng = np.random.default_rng(21)
    kinds = np.array([1.0] * 3 + [0.25] * 4 + [0.0])          # per 8 weights
    w = np.stack([rng.permutation(kinds) for _ in range(N * K // 8)]).reshape(N, K)
    flat = w.reshape(-1)
    quarter = np.flatnonzero(flat == 0.25)
    trip = rng.choice(quarter, size=(300, 3), replace=False)
    flat[trip[:, 0]] = 0.25 + 2.0 ** -9
    flat[trip[:, 1:]] = 0.25 - 2.0 ** -10
    sign = np.where(rng.random(flat.shape) < 0.5, -1.0, 1.0)
    W = bf16_exact((flat * sign).reshape(N, K))
    g_ref = oracle.absmean_gamma(W)
    assert g_ref == np.float32(0.5)
    q_ref = oracle.ternarize(W, g_ref)
    a = np.abs(oracle.bf16_to_f64(W))
    assert np.all(q_ref[a == 0.25] == 0) and np.all(q_ref[a == 0.25 - 2.0 ** -10] == 0)
    assert np.all(np.abs(q_ref[a == 0.25 + 2.0 ** -9]) == 1)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    B.bitnet_sync_status()
    assert np.float32(gamma.item()) == g_ref
    np.testing.assert_array_equal(Wp.cpu().numpy().view(np.uint32).reshape(N, K // 16),
                                  oracle.pack_ternary(q_ref))


def test_weights_near_the_threshold_of_a_random_gamma(B):
    """A random matrix whose gamma is not a power of two, with probes at the bf16 values around
    gamma / 2, where the fp32 division w / gamma decides between 0 and +-1 by one rounding."""
    N, K = 256, 1024
    W = synth.latent_weights(N, K, seed=33)
    probes = np.random.default_rng(33).choice(N * K, size=4096, replace=False)
    for _ in range(6):  # settle gamma: the probes' own magnitudes move it slightly
        g = float(oracle.absmean_gamma(W))
        h = np.float32(g / 2)
        nb = synth.f32_to_bf16_bits(np.array([h], np.float32)).astype(np.int32)[0] & 0x7FFF
        cand = np.array([nb - 2, nb - 1, nb, nb + 1, nb + 2], np.int32)
        mags = cand[np.arange(probes.size) % 5]
        signs = np.where(np.arange(probes.size) % 2 == 0, 0, 0x8000)
        flat = W.reshape(-1).copy()
        flat[probes] = (mags | signs).astype(np.uint16)
        W = flat.reshape(N, K)
    g_ref = oracle.absmean_gamma(W)
    q_ref = oracle.ternarize(W, g_ref)
    a = np.abs(oracle.bf16_to_f64(W.reshape(-1)[probes]))
    qa = np.abs(q_ref.reshape(-1)[probes])
    # the probes straddle the threshold: some decide 0, some +-1, within two bf16 steps
    assert (qa == 0).any() and (qa == 1).any()
    assert a.max() / a.min() < 1.04
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    B.bitnet_sync_status()
    assert np.float32(gamma.item()) == g_ref
    np.testing.assert_array_equal(Wp.cpu().numpy().view(np.uint32).reshape(N, K // 16),
                                  oracle.pack_ternary(q_ref))


@pytest.mark.parametrize("bits", [8, 4])
def test_activation_codes_at_exact_ties_plain(B, bits):
    """Plain rows with max |x| = Q/2 or Q/4, so s = 2 or 4 exactly, and every other x equal to
    (k + 1/2) / s: x * s lands exactly on a .5 for each of them.  The codes must round half to
    even, as the oracle does, with zero differences.  (INT4: the absmax variant, whose scale a
    row's maximum fixes.)"""
    Q = 127 if bits == 8 else 7
    K = 256
    rng = np.random.default_rng(bits)
    rows = []
    for s in (2, 4):
        x = (rng.integers(-Q, Q, size=K) + 0.5) / s       # x * s = k + 1/2, |k + 1/2| < Q
        x[rng.integers(K)] = Q / s
        rows.append(x)
    X = bf16_exact(np.stack(rows))
    if bits == 8:
        codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), False, 8)
    else:
        codes, scales, rowsum = B.bitnet_act_quant_absmax4(dev_bf16(X), False)
    B.bitnet_sync_status()
    z = oracle.bf16_to_f64(X).astype(np.float32)
    c_ref, d_ref, pre, rs_ref = oracle.quant_act(z, bits)
    assert (pre - np.floor(pre) == 0.5).sum() > K  # most elements are exact ties
    np.testing.assert_array_equal(codes_rows(codes, np.arange(2), K, bits), c_ref)
    np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), rs_ref)


def hadamard_rows_from_z(z_rows, K):
    """x = H z / sqrt(K), so that the transform gives back z exactly (H H = K I)."""
    H = np.array([[(-1) ** bin(i & j).count("1") for j in range(K)] for i in range(K)], np.float64)
    return (np.asarray(z_rows, np.float64) @ H) / math.sqrt(K)


def test_activation_codes_at_exact_ties_hadamard(B):
    """H-BitLinear rows built so that z = 63.5 e_0 + 0.25 e_a + 0.75 e_b (signs varied): every x is
    a bf16 value, the fp32 transform is exact, s = 127 / 63.5 = 2, and z * s = 127, 0.5, 1.5,
    which round to 127, 0 and 2."""
    K = 256
    rng = np.random.default_rng(5)
    zs = []
    for t in range(12):
        z = np.zeros(K)
        a, b = rng.choice(np.arange(1, K), size=2, replace=False)
        z[0] = 63.5 * (1 if t % 2 == 0 else -1)
        z[a] = 0.25 * (1 if t % 3 else -1)
        z[b] = 0.75 * (1 if t % 4 < 2 else -1)
        zs.append(z)
    X = bf16_exact(hadamard_rows_from_z(zs, K))
    Xd = dev_bf16(X)
    Z = B.bitnet_fwht_f32(Xd).cpu().numpy().astype(np.float64)
    np.testing.assert_array_equal(Z, np.array(zs))
    codes, scales, rowsum = B.bitnet_act_quant(Xd, True, 8)
    B.bitnet_sync_status()
    ref = oracle.bitlinear_forward(X, synth.latent_weights(8, K, seed=1), True, 8)
    c = codes.cpu().numpy().view(np.int8)
    np.testing.assert_array_equal(c, ref["codes"])
    expect = np.rint(np.array(zs) * 2).astype(np.int8)  # numpy rint: half to even
    np.testing.assert_array_equal(c, expect)
    assert set(np.unique(np.abs(expect))) == {0, 2, 127}
    np.testing.assert_array_equal(scales.cpu().numpy(), ref["d"])


@pytest.mark.parametrize("K", [256, 2048, 8192])
@pytest.mark.parametrize("bits", [8, 4])
def test_single_spike_and_constant_rows(B, K, bits):
    """x = c * (column j of H): z = c sqrt(K) e_j, one non-zero; a constant row is the j = 0
    case.  Codes are the oracle's (Q or the clipped absmean code at j, zero elsewhere), bit for
    bit, and the scales match."""
    js = [0, 1, K // 2 + 3, K - 1]
    rows = []
    for t, j in enumerate(js):
        col = np.array([(-1) ** bin(i & j).count("1") for i in range(K)], np.float64)
        rows.append((0.5 if t % 2 == 0 else -0.125) * col)
    rows.append(np.full(K, 0.75))                          # constant row
    X = bf16_exact(np.stack(rows))
    codes, scales, rowsum = B.bitnet_act_quant(dev_bf16(X), True, bits)
    B.bitnet_sync_status()
    ref = oracle.bitlinear_forward(X, synth.latent_weights(8, K, seed=2), True, bits)
    c = codes_rows(codes, np.arange(len(rows)), K, bits)
    np.testing.assert_array_equal(c, ref["codes"])
    for t, j in enumerate(js + [0]):
        nz = np.flatnonzero(c[t])
        assert list(nz) == [j]
    # 1/sqrt(K) is inexact for odd powers of two: the scale may differ in its last bit
    np.testing.assert_allclose(scales.cpu().numpy(), ref["d"], rtol=1e-6)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), c.astype(np.int64).sum(axis=1))


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
    c_ref, d_ref, pre, rs_ref = oracle.quant_act_for_bits(z, bits)
    c = codes.cpu().numpy()
    c = c.view(np.int8) if bits == 8 else oracle.unpack_int4(c.view(np.uint8), K)
    assert check_codes(c, c_ref, pre) == 0
    if bits == 8:
        np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)
    else:  # absmean: a double sum in another order
        np.testing.assert_allclose(scales.cpu().numpy(), d_ref, rtol=1e-6)
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
    (9, 256, 256), (32, 8192, 2064), (64, 2048, 8192),          # skinny tensor-core kernel
    (300, 2048, 272), (1000, 640, 528),                         # 256 x 256 tiles
    (300, 8192, 528),                                           # INT4: tensor-memory kernel
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
# INT4: the absmean rule of act_bits 4 (the clip is exercised), and the absmax variant
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("K", [128, 256, 2048, 4096, 8192, 16384, 32768])
def test_int4_absmean_hadamard_codes(B, K):
    M = 37 if K <= 8192 else 9
    X = synth.sharp_activations(M, K, seed=5 * K + 1)
    Xd = dev_bf16(X)
    z = B.bitnet_fwht_f32(Xd).cpu().numpy()
    codes, scales, rowsum = B.bitnet_act_quant(Xd, True, 4)
    B.bitnet_sync_status()
    c_ref, d_ref, pre, _ = oracle.quant_act_absmean4(z)
    c = oracle.unpack_int4(codes.cpu().numpy().view(np.uint8), K)
    n_diff = check_codes(c, c_ref, pre)
    assert n_diff == 0, f"{n_diff} codes differ (within the boundary tolerance)"
    np.testing.assert_allclose(scales.cpu().numpy(), d_ref, rtol=1e-6)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), c.astype(np.int64).sum(axis=1))
    assert (c == 7).any() or (c == -8).any()  # the clip is exercised


@pytest.mark.parametrize("K", [128, 256, 2048, 8192, 16384])
def test_absmax4_hadamard_codes(B, K):
    M = 37 if K <= 8192 else 9
    X = synth.sharp_activations(M, K, seed=5 * K + 2)
    Xd = dev_bf16(X)
    z = B.bitnet_fwht_f32(Xd).cpu().numpy()
    codes, scales, rowsum = B.bitnet_act_quant_absmax4(Xd, True)
    B.bitnet_sync_status()
    c_ref, d_ref, pre, _ = oracle.quant_act(z, 4)
    c = oracle.unpack_int4(codes.cpu().numpy().view(np.uint8), K)
    assert check_codes(c, c_ref, pre) == 0
    np.testing.assert_allclose(scales.cpu().numpy(), d_ref, rtol=1e-6)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), c.astype(np.int64).sum(axis=1))


@pytest.mark.parametrize("K", [128, 640, 4096])
def test_absmax4_plain_codes(B, K):
    M = 19
    X = synth.gaussian_activations(M, K, seed=K + 17)
    X[3] = 0  # a zero row: zero codes, guarded scale
    codes, scales, rowsum = B.bitnet_act_quant_absmax4(dev_bf16(X), False)
    B.bitnet_sync_status()
    z = oracle.bf16_to_f64(X).astype(np.float32)
    c_ref, d_ref, _, rs_ref = oracle.quant_act(z, 4)
    c = oracle.unpack_int4(codes.cpu().numpy().view(np.uint8), K)
    np.testing.assert_array_equal(c, c_ref)
    np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)
    np.testing.assert_array_equal(rowsum.cpu().numpy(), rs_ref)
    assert not c[3].any()


@pytest.mark.parametrize("name,rows", [("wdown_8192", 16), ("tiny", None)])
def test_absmax4_forward_end_to_end(B, name, rows):
    wl = synth.WORKLOADS[name]
    X, W = wl.activations(seed=6), wl.weights(seed=6)
    Wp, gamma = B.bitnet_quantize_pack_weights(dev_bf16(W))
    Y = B.bitnet_bitlinear_forward_absmax4(dev_bf16(X), Wp, gamma, wl.hadamard)
    B.bitnet_sync_status()
    sel = sample_rows(wl.M, rows, 6)
    ref = oracle.bitlinear_forward(X[sel], W, wl.hadamard, 4, int4_absmax=True)
    assert np.float32(gamma.item()) == ref["gamma"]
    y = oracle.bf16_to_f64(to_np_bits(Y)[sel])
    y_ref = oracle.bf16_to_f64(ref["y"])
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
    codes, d, _, _ = oracle.quant_act_for_bits(z, wl.act_bits)
    Wr = oracle.rotate_weights(W)
    g = oracle.absmean_gamma_f32(Wr)
    assert abs(np.float32(gamma.item()) / g - 1) <= 1e-6
    acc = oracle.gemm_i64(codes, oracle.ternarize_f32(Wr, g))
    y_ref = oracle.bf16_to_f64(oracle.dequant(acc, d, g))
    y = oracle.bf16_to_f64(to_np_bits(Y)[sel])
    assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) <= Y_REL


# ----------------------------------------------------------------------------------------
# low-bit Q / K / V states (BitNet v2 write-up, Tables 2 and 3): packed bit streams and scales
# bit-exact against the oracle
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("M,C,group", [(37, 4096, 128), (16, 2048, 64), (9, 4096, 4096),
                                       (5, 96, 32), (300, 1024, 1024)])
@pytest.mark.parametrize("bits", [3, 2, 4, 8])
def test_state_quant_bit_exact(B, M, C, group, bits):
    rng = np.random.default_rng(M + C + bits)
    x = rng.standard_normal((M, C)).astype(np.float32)
    x[:, rng.choice(C, size=max(1, C // 64), replace=False)] *= 20.0  # outlier channels
    x[1, :group] = 0.0                                                 # an all-zero group
    X = synth.f32_to_bf16_bits(x)
    codes, scales = B.bitnet_quant_states(dev_bf16(X), group, bits)
    B.bitnet_sync_status()
    c_ref, d_ref, _ = oracle.quant_states(X, group, bits)
    np.testing.assert_array_equal(codes.cpu().numpy(), oracle.pack_bits(c_ref, bits))
    np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)


def test_state_quant_exact_ties(B):
    # groups with max 1.5: s = 2 exactly, so 0.25, 0.75, 1.25 -> 0.5, 1.5, 2.5 -> 0, 2, 2
    K = 64
    vals = np.array([0.25, 0.75, 1.25, -0.25, -0.75, -1.25, 0.5, 1.0])
    row = np.tile(vals, K // len(vals))
    row[0] = 1.5
    X = bf16_exact(np.stack([row, -row]))
    codes, scales = B.bitnet_quant_states(dev_bf16(X), K, 3)
    B.bitnet_sync_status()
    c = oracle.unpack_bits(codes.cpu().numpy(), K, 3)
    c_ref, d_ref, pre = oracle.quant_states(X, K, 3)
    np.testing.assert_array_equal(c, c_ref)
    assert (pre - np.floor(pre) == 0.5).sum() >= K
    np.testing.assert_array_equal(scales.cpu().numpy(), d_ref)
