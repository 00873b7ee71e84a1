"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

None of these re-types an oracle formula.  Each compares the oracle with something
independent of it: a worked example printed on a page (tests/golden/), a closed form, an
invariant, a textbook or library special case, or brute force on tiny inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from bit_activation_linear_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bf16_bits(values):
    return synth.f32_to_bf16_bits(np.asarray(values, dtype=np.float32))


# ----------------------------------------------------------------------------------------
# Hadamard transform (BitNet v2 write-up: entries +-1, mutually orthogonal rows)
# ----------------------------------------------------------------------------------------

def sylvester_blocks(n):
    """H_n by the block recursion H_2m = [[H_m, H_m], [H_m, -H_m]], H_1 = [1]."""
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def sylvester_bits(n):
    """H_n[i, j] = (-1)^popcount(i & j): an independent closed form of the same matrix."""
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    parity = np.vectorize(lambda v: bin(int(v)).count("1") & 1)(i & j)
    return 1.0 - 2.0 * parity


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_hadamard_entries_and_orthogonality(n):
    H = sylvester_blocks(n)
    assert set(np.unique(H)) <= {-1.0, 1.0}
    np.testing.assert_array_equal(H @ H.T, n * np.eye(n))
    np.testing.assert_array_equal(H, sylvester_bits(n))
    np.testing.assert_array_equal(H, scipy.linalg.hadamard(n))


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_fwht_equals_explicit_matrix_product(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((5, n))
    z = oracle.fwht(x)
    ref = x @ sylvester_blocks(n).T / math.sqrt(n)
    np.testing.assert_allclose(z, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [128, 256, 1024])
def test_fwht_equals_library_hadamard(n):
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, n))
    ref = x @ scipy.linalg.hadamard(n).T.astype(np.float64) / math.sqrt(n)
    np.testing.assert_allclose(oracle.fwht(x), ref, rtol=0, atol=1e-11)


@pytest.mark.parametrize("n", [2, 64, 2048, 8192])
def test_fwht_involution_and_parseval(n):
    rng = np.random.default_rng(n + 1)
    x = rng.laplace(size=(4, n))
    z = oracle.fwht(x)
    np.testing.assert_allclose(np.linalg.norm(z, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(oracle.fwht(z), x, rtol=0, atol=1e-12 * np.abs(x).max())


@pytest.mark.parametrize("n", [16, 256])
def test_fwht_basis_vectors(n):
    H = sylvester_bits(n)
    E = np.eye(n)
    np.testing.assert_allclose(oracle.fwht(E), H.T / math.sqrt(n), atol=1e-14)
    ones = np.ones((1, n))
    e0 = np.zeros((1, n))
    e0[0, 0] = math.sqrt(n)
    np.testing.assert_allclose(oracle.fwht(ones), e0, atol=1e-12)


def test_hadamard_makes_sharp_inputs_gaussian_like():
    """BitNet v2 write-up (Figures 2-3): after the transform the outlier-heavy inputs of
    Wo / Wdown look close to Gaussian, and low-bit quantisation loses less."""
    K = 2048
    x = oracle.bf16_to_f64(synth.sharp_activations(64, K, seed=3))
    z = oracle.fwht(x)

    def excess_kurtosis(a):
        a = a - a.mean(axis=1, keepdims=True)
        return (np.mean(a ** 4, axis=1) / np.mean(a ** 2, axis=1) ** 2 - 3.0).mean()

    assert excess_kurtosis(x) > 20.0
    assert abs(excess_kurtosis(z)) < 0.5

    def int4_rel_mse(v):
        c, d, _, _ = oracle.quant_act(v.astype(np.float32), 4)
        err = c.astype(np.float64) * d[:, None].astype(np.float64) - v
        return np.mean(err ** 2) / np.mean(v ** 2)

    assert int4_rel_mse(z) < 0.5 * int4_rel_mse(x)


# ----------------------------------------------------------------------------------------
# absmean ternarisation (b1.58 summary, 方法论 / 方法详解)
# ----------------------------------------------------------------------------------------

def test_ternarize_hand_example():
    g = golden("ternary_hand_example.json")
    W = bf16_bits(g["W"])
    gamma = oracle.absmean_gamma(W)
    assert gamma == np.float32(g["gamma"])
    np.testing.assert_array_equal(oracle.ternarize(W, gamma), np.array(g["q"], dtype=np.int8))


def test_gamma_is_library_mean_of_abs():
    W = synth.latent_weights(64, 512, seed=5)
    ref = np.float32(np.mean(np.abs(oracle.bf16_to_f64(W))))
    assert oracle.absmean_gamma(W) == ref


def test_ternarize_brute_force_nearest():
    """q is the element of {-1, 0, 1} nearest to w / gamma (fp32 ratio)."""
    W = synth.latent_weights(32, 256, seed=11)
    gamma = oracle.absmean_gamma(W)
    q = oracle.ternarize(W, gamma)
    r = oracle.bf16_to_f64(W).astype(np.float32) / np.float32(gamma)
    cands = np.array([-1.0, 0.0, 1.0])
    dist = np.abs(r.astype(np.float64)[..., None] - cands)
    assert not np.any(np.isclose(np.sort(dist, axis=-1)[..., 0], np.sort(dist, axis=-1)[..., 1]))
    np.testing.assert_array_equal(q, cands[np.argmin(dist, axis=-1)].astype(np.int8))


def test_ternarize_alphabet_and_zero_fraction():
    """Codes lie in {-1, 0, 1}; for W ~ N(0, s), |w| / mean|w| <= 1/2 happens with
    probability 2 Phi(sqrt(2/pi) / 2) - 1 = 0.3101 (half-normal mean s sqrt(2/pi))."""
    W = synth.latent_weights(512, 1024, seed=0)
    q = oracle.ternarize(W, oracle.absmean_gamma(W))
    assert set(np.unique(q)) <= {-1, 0, 1}
    p0 = 2.0 * 0.5 * (1.0 + math.erf(math.sqrt(2.0 / math.pi) / 2.0 / math.sqrt(2.0))) - 1.0
    assert abs(p0 - 0.3101) < 1e-4
    n = q.size
    frac0 = np.mean(q == 0)
    assert abs(frac0 - p0) < 4.0 * math.sqrt(p0 * (1 - p0) / n) + 2e-3  # +bf16 rounding of W
    assert abs(np.mean(q == 1) - np.mean(q == -1)) < 0.01


def test_ternarize_constant_and_zero_weights():
    W = bf16_bits(np.full((4, 16), -0.03125))
    g = oracle.absmean_gamma(W)
    assert g == np.float32(0.03125)
    np.testing.assert_array_equal(oracle.ternarize(W, g), -np.ones((4, 16), np.int8))
    Z = bf16_bits(np.zeros((2, 16)))
    assert oracle.absmean_gamma(Z) == np.float32(1e-5)
    np.testing.assert_array_equal(oracle.ternarize(Z, oracle.absmean_gamma(Z)), 0)


# ---- weight + activation rotation: absmean ternarisation of the rotated fp32 rows ----

def test_ternarize_f32_equals_bf16_path_on_bf16_values():
    # fp32 weights that are exactly bf16 values give the bf16 path's gamma and codes
    W = synth.latent_weights(64, 256, seed=21)
    wf = oracle.bf16_to_f64(W).astype(np.float32)
    g = oracle.absmean_gamma(W)
    assert oracle.absmean_gamma_f32(wf) == g
    np.testing.assert_array_equal(oracle.ternarize_f32(wf, g), oracle.ternarize(W, g))


def test_ternarize_f32_brute_force_and_library_mean():
    rng = np.random.default_rng(22)
    w = (rng.standard_normal((32, 128)) * 0.02).astype(np.float32)
    w[0, :4] = [0.0, -0.0, 1e-9, -1e-9]
    g = oracle.absmean_gamma_f32(w)
    assert g == np.float32(np.abs(w.astype(np.float64)).mean())
    r = (w / g).astype(np.float32)                    # one fp32 division, as the decision takes it
    cand = np.array([-1.0, 0.0, 1.0])
    dist = np.abs(r.astype(np.float64)[..., None] - cand)
    best = dist.min(axis=-1, keepdims=True)
    # nearest of {-1, 0, 1}; a tie at +-0.5 goes to 0 (even)
    pick = np.where(dist == best, np.where(cand == 0, 0, 1), 2)
    q_ref = cand[np.argmin(pick, axis=-1)].astype(np.int8)
    np.testing.assert_array_equal(oracle.ternarize_f32(w, g), q_ref)
    # ties exactly at half of gamma
    half = np.array([[g * np.float32(0.5), -g * np.float32(0.5)]], dtype=np.float32)
    np.testing.assert_array_equal(oracle.ternarize_f32(half, g), [[0, 0]])


@pytest.mark.parametrize("K", [128, 1024])
def test_rotate_weights_is_the_explicit_product_and_preserves_wx(K):
    W = synth.latent_weights(24, K, seed=K)
    Wr = oracle.rotate_weights(W)
    H = scipy.linalg.hadamard(K).astype(np.float64)
    ref = (oracle.bf16_to_f64(W) @ H / math.sqrt(K)).astype(np.float32)
    np.testing.assert_array_equal(Wr, ref)
    # W' (H x / sqrt(K)) = W x: the rotation cancels in the product
    x = np.random.default_rng(K).standard_normal((5, K))
    lhs = Wr.astype(np.float64) @ oracle.fwht(x).T
    rhs = oracle.bf16_to_f64(W) @ x.T
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-6 * np.abs(rhs).max())


def test_ternarize_ties_round_half_to_even():
    """|w / gamma| = 0.5 exactly rounds to 0, 1.5 rounds to 2 and clips to 1."""
    gamma = np.float32(0.25)
    W = bf16_bits([0.125, -0.125, 0.375, -0.375, 0.1250001])
    np.testing.assert_array_equal(oracle.ternarize(W, gamma), [0, 0, 1, -1, 0])


# ----------------------------------------------------------------------------------------
# Storage formats
# ----------------------------------------------------------------------------------------

def test_base3_example_from_the_page():
    g = golden("base3_packing.json")
    b = oracle.pack_base3(np.array(g["digits"], dtype=np.uint8))
    assert b.tolist() == [g["byte"]]
    assert format(int(b[0]), "08b") == g["binary"]
    np.testing.assert_array_equal(oracle.unpack_base3(b, 5), g["digits"])
    assert round(100 * 5 * math.log2(3) / 8, 2) == g["efficiency_percent"]


def test_base3_round_trip_and_range():
    rng = np.random.default_rng(2)
    d = rng.integers(0, 3, size=1003).astype(np.uint8)
    b = oracle.pack_base3(d)
    assert b.size == 201 and int(b.max()) <= 242
    np.testing.assert_array_equal(oracle.unpack_base3(b, d.size), d)


def test_ternary_word_layout_hand_example():
    g = golden("ternary_word_layout.json")
    q = np.array([g["q"]], dtype=np.int8)
    wp = oracle.pack_ternary(q)
    assert wp.shape == (1, 1) and int(wp[0, 0]) == g["word"]
    back, bad = oracle.unpack_ternary(wp, 16)
    assert bad == 0
    np.testing.assert_array_equal(back, q)


def test_ternary_pack_round_trip():
    rng = np.random.default_rng(4)
    q = rng.integers(-1, 2, size=(37, 256)).astype(np.int8)
    wp = oracle.pack_ternary(q)
    assert wp.nbytes == q.size // 4
    back, bad = oracle.unpack_ternary(wp, 256)
    assert bad == 0
    np.testing.assert_array_equal(back, q)


def test_int4_nibble_layout_hand_example():
    g = golden("int4_nibble_layout.json")
    c = np.array([g["codes"]], dtype=np.int8)
    b = oracle.pack_int4(c)
    assert b.ravel().tolist() == g["bytes"]
    np.testing.assert_array_equal(oracle.unpack_int4(b, 8), c)


# ----------------------------------------------------------------------------------------
# Per-token absmax quantisation (2B4T article, 一.2; BitNet v2 write-up)
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits,Q", [(8, 127), (4, 7)])
def test_quant_brute_force_nearest_and_extremes(bits, Q):
    rng = np.random.default_rng(bits)
    z = (rng.laplace(size=(20, 256)) * 0.3).astype(np.float32)
    z[3] = 0.0
    codes, d, pre, rowsum = oracle.quant_act(z, bits)
    # zero row: zero codes, guarded scale
    assert not codes[3].any() and d[3] == np.float32(np.float32(1e-5) / np.float32(Q))
    live = [m for m in range(20) if m != 3]
    # the largest |z| of each row maps to +-Q exactly; all codes lie in range
    for m in live:
        k = int(np.argmax(np.abs(z[m])))
        assert codes[m, k] == Q * np.sign(z[m, k])
    assert codes.min() >= -Q and codes.max() <= Q
    # brute force: each code is the integer nearest to z * s with s = fp32(Q / max|z|)
    s = (np.float32(Q) / np.abs(z).max(axis=1).clip(min=np.float32(1e-5))).astype(np.float32)
    v = (z * s[:, None]).astype(np.float32).astype(np.float64)
    cand = np.stack([np.floor(v), np.ceil(v)], axis=-1)
    best = np.take_along_axis(cand, np.argmin(np.abs(cand - v[..., None]), axis=-1)[..., None],
                              axis=-1)[..., 0]
    np.testing.assert_array_equal(codes[live], best[live].astype(np.int8))
    np.testing.assert_array_equal(rowsum, codes.astype(np.int64).sum(axis=1))
    # d is the dequantisation step: codes * d reproduces z to within half a step
    err = np.abs(codes * d[:, None].astype(np.float64) - z)
    assert np.all(err[live] <= 0.5 * d[live, None] * (1 + 1e-6))


@pytest.mark.parametrize("bits,Q", [(8, 127), (4, 7)])
def test_quant_pre_at_exact_ties(bits, Q):
    """Rows whose max |z| is Q/2 or Q/4 have s = 2 or 4 exactly, so z * s is exact and known:
    ``pre`` must equal those closed-form values and every x.5 must round to the even integer.
    A dropped factor, a wrong scale or a round-half-away rule fails here."""
    z = np.zeros((3, 16), np.float32)
    # s = 2: pre = 2 z
    z[0, :10] = [Q / 2, 0.25, 0.75, -0.25, -0.75, 1.25, -1.75, 0.125, 1.0, -Q / 2]
    # s = 4: pre = 4 z
    z[1, :8] = [Q / 4, 0.125, 0.375, 0.625, -0.875, 0.0625, -Q / 4, 0.25]
    z[2, 0] = -Q / 2                      # one non-zero: pre = -Q at 0, zero elsewhere
    codes, d, pre, rowsum = oracle.quant_act(z, bits)
    exp_pre = np.zeros((3, 16))
    exp_pre[0, :10] = [Q, 0.5, 1.5, -0.5, -1.5, 2.5, -3.5, 0.25, 2.0, -Q]
    exp_pre[1, :8] = [Q, 0.5, 1.5, 2.5, -3.5, 0.25, -Q, 1.0]
    exp_pre[2, 0] = -Q
    np.testing.assert_array_equal(pre, exp_pre)
    exp_codes = np.zeros((3, 16), np.int64)
    exp_codes[0, :10] = [Q, 0, 2, 0, -2, 2, -4, 0, 2, -Q]     # ties to even
    exp_codes[1, :8] = [Q, 0, 2, 2, -4, 0, -Q, 1]
    exp_codes[2, 0] = -Q
    np.testing.assert_array_equal(codes, exp_codes)
    np.testing.assert_array_equal(rowsum, exp_codes.sum(axis=1))
    np.testing.assert_array_equal(d, np.float32([Q / 2, Q / 4, Q / 2]) / np.float32(Q))
    # on random rows pre stays within half a step of its code
    z = np.random.default_rng(bits + 40).laplace(size=(8, 512)).astype(np.float32)
    codes, _, pre, _ = oracle.quant_act(z, bits)
    assert np.all(np.abs(pre - codes) <= 0.5 + 1e-6)


# ---- the INT4 quantiser, with an absmean scale (a reading: the pages give INT8 and INT4 each their
# own strategy without printing either formula; the form is that of the weights' absmean) ----

SQRT7_F32 = np.float32(math.sqrt(7.0))


def _nearest_code_brute(v: np.ndarray, lo: int, hi: int) -> np.ndarray:
    """Nearest integer in [lo, hi] to each value by exhaustive search, ties to the even one."""
    cand = np.arange(lo, hi + 1, dtype=np.float64)
    dist = np.abs(v.astype(np.float64)[..., None] - cand)
    best = dist.min(axis=-1, keepdims=True)
    tie_ok = np.isclose(dist, best, rtol=0, atol=0)
    even = (cand % 2 == 0)
    pick = np.where(tie_ok & even, 0, np.where(tie_ok, 1, 2))  # prefer even among the nearest
    return cand[np.argmin(pick, axis=-1)].astype(np.int64)


def test_absmean4_constant_magnitude_rows():
    # |z| = a everywhere: beta = a, z * s = +-sqrt(7) -> +-3; d = a / sqrt(7)
    a = np.float32(0.37)
    z = np.where(np.arange(64) % 3 == 0, -a, a).astype(np.float32)[None, :].repeat(2, 0)
    codes, d, _, rowsum = oracle.quant_act_absmean4(z)
    np.testing.assert_array_equal(codes, np.where(z > 0, 3, -3))
    assert d[0] == np.float32(a / SQRT7_F32)
    assert rowsum[0] == codes[0].astype(np.int64).sum()


def test_absmean4_brute_force_nearest_with_clipping():
    rng = np.random.default_rng(11)
    z = (rng.laplace(size=(12, 128)) * 0.2).astype(np.float32)
    z[2, 5] = 40.0    # outliers far beyond the clip
    z[4, 9] = -40.0
    codes, d, pre, rowsum = oracle.quant_act_absmean4(z)
    beta = np.abs(z.astype(np.float64)).mean(axis=1)
    g = np.maximum(beta, 1e-5).astype(np.float32)
    s = (SQRT7_F32 / g).astype(np.float32)
    v = (z * s[:, None]).astype(np.float32)          # the fp32 product the decision is taken on
    np.testing.assert_array_equal(codes, _nearest_code_brute(v, -8, 7))
    assert codes[2, 5] == 7 and codes[4, 9] == -8
    assert codes.min() >= -8 and codes.max() <= 7
    np.testing.assert_array_equal(d, (g / SQRT7_F32).astype(np.float32))
    np.testing.assert_array_equal(rowsum, codes.astype(np.int64).sum(axis=1))
    np.testing.assert_allclose(pre, z.astype(np.float64) * s[:, None].astype(np.float64))


def test_absmean4_zero_row_and_scale_invariance():
    rng = np.random.default_rng(5)
    z = rng.standard_normal((6, 256)).astype(np.float32)
    z[1] = 0.0
    codes, d, _, _ = oracle.quant_act_absmean4(z)
    assert not codes[1].any() and d[1] == np.float32(np.float32(1e-5) / SQRT7_F32)
    # a power-of-two scale leaves the codes unchanged and scales d exactly
    codes2, d2, _, _ = oracle.quant_act_absmean4((z * np.float32(8.0)).astype(np.float32))
    np.testing.assert_array_equal(codes2[[0, 2, 3, 4, 5]], codes[[0, 2, 3, 4, 5]])
    np.testing.assert_array_equal(d2[[0, 2, 3, 4, 5]], d[[0, 2, 3, 4, 5]] * np.float32(8.0))


def test_absmean4_gaussian_clip_fraction():
    # a Gaussian row (what the Hadamard produces): beta ~ sigma*sqrt(2/pi), so code 7 needs
    # z > 6.5 beta / sqrt(7) and code -8 needs z < -7.5 beta / sqrt(7): the fractions of the
    # two end codes follow the normal tail at those points
    from scipy.stats import norm
    z = np.random.default_rng(9).standard_normal((16, 16384)).astype(np.float32)
    codes, _, _, _ = oracle.quant_act_absmean4(z)
    r = math.sqrt(2 / math.pi) / math.sqrt(7.0)
    p7, p8 = norm.sf(6.5 * r), norm.cdf(-7.5 * r)
    n = codes.size
    for frac, p in ((np.mean(codes == 7), p7), (np.mean(codes == -8), p8)):
        assert abs(frac - p) < 5 * math.sqrt(p * (1 - p) / n), (frac, p)


# ----------------------------------------------------------------------------------------
# Ternary product (2B4T article, 一.2: +1 adds, -1 subtracts, 0 skips)
# ----------------------------------------------------------------------------------------

def test_gemm_three_ways_agree():
    rng = np.random.default_rng(9)
    c = rng.integers(-128, 128, size=(7, 96)).astype(np.int8)
    q = rng.integers(-1, 2, size=(5, 96)).astype(np.int8)
    a = oracle.gemm_i64(c, q)
    np.testing.assert_array_equal(a, oracle.gemm_addsub(c, q))
    np.testing.assert_array_equal(a, c.astype(np.int64) @ q.astype(np.int64).T)


def test_gemm_all_ones_weights_give_row_sums():
    rng = np.random.default_rng(10)
    c = rng.integers(-128, 128, size=(4, 64)).astype(np.int8)
    q = np.ones((3, 64), np.int8)
    np.testing.assert_array_equal(oracle.gemm_i64(c, q),
                                  np.repeat(c.astype(np.int64).sum(1, keepdims=True), 3, 1))


def test_gemm_tiny_by_hand():
    c = np.array([[1, 2, 3], [-4, 5, -6]], np.int8)
    q = np.array([[1, 0, -1], [-1, -1, 1], [0, 1, 0]], np.int8)
    # row 0: 1-3=-2, -1-2+3=0, 2 ; row 1: -4+6=2, 4-5-6=-7, 5
    np.testing.assert_array_equal(oracle.gemm_i64(c, q), [[-2, 0, 2], [2, -7, 5]])


# ----------------------------------------------------------------------------------------
# bf16 rounding of the output
# ----------------------------------------------------------------------------------------

def test_bf16_rounding_cases():
    f = oracle.f64_to_bf16
    cases = {
        1.0: 0x3F80,
        1.0 + 2 ** -8: 0x3F80,                 # tie -> even (1.0)
        1.0 + 3 * 2 ** -8: 0x3F82,             # tie -> even (1 + 2^-6)
        1.0 + 2 ** -8 + 2 ** -40: 0x3F81,      # above the tie: rounding via fp32 would give 1.0
        -2.5: 0xC020,
        2.0 ** -133: 0x0001,                   # smallest subnormal
        3.0 * 2.0 ** -134: 0x0002,             # subnormal tie -> even
        1e39: 0x7F80,                          # overflow
    }
    for v, bits in cases.items():
        assert int(f(np.array([v]))[0]) == bits, v
    rng = np.random.default_rng(3)
    x = rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000)
    # for values already exact in fp32 (no double rounding possible) torch agrees
    x32 = x.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x32).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(f(x32), ref.view(np.uint16))


def test_dequant_against_exact_products():
    acc = np.array([[0, 1, -127, 2_000_000]], np.int64)
    d = np.array([0.5], np.float32)
    Y = oracle.dequant(acc, d, np.float32(0.25))
    np.testing.assert_array_equal(oracle.bf16_to_f64(Y), [[0.0, 0.125, -15.875, 249856.0]])


# ----------------------------------------------------------------------------------------
# Whole forward: closed forms
# ----------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [8, 4])
def test_forward_hadamard_column_input(bits):
    """x = a * (column j of H): z = a sqrt(K) e_j, one non-zero.  INT8 (absmax): the code is
    +-127 at j only and Y[n] = q[n, j] * a * sqrt(K) * gamma.  INT4 (absmean): mean |z| =
    a / sqrt(K), so z_j * s = +-sqrt(7) K is clipped to 7 or -8, and Y[n] = code * q[n, j] *
    (a / sqrt(K) / sqrt(7)) * gamma (up to bf16 rounding).  A transposed operand, a dropped
    normalisation or a wrong sign fails here."""
    K, N = 256, 64
    H = sylvester_bits(K)
    a = 0.125
    js = [0, 3, 77, 255]
    X = bf16_bits(np.stack([a * H[:, j] * (1 if t % 2 == 0 else -1) for t, j in enumerate(js)]))
    W = synth.latent_weights(N, K, seed=1)
    out = oracle.bitlinear_forward(X, W, hadamard=True, bits=bits)
    gamma = float(out["gamma"])
    for t, j in enumerate(js):
        sgn = 1 if t % 2 == 0 else -1
        if bits == 8:
            code, step = sgn * 127, a * math.sqrt(K) / 127
        else:
            code, step = (7 if sgn > 0 else -8), a / math.sqrt(K) / math.sqrt(7)
        expect_codes = np.zeros(K, np.int8)
        expect_codes[j] = code
        np.testing.assert_array_equal(out["codes"][t], expect_codes)
        np.testing.assert_allclose(out["d"][t], step, rtol=1e-6)
        y = oracle.bf16_to_f64(out["y"][t])
        ref = code * out["q"][:, j] * step * gamma
        np.testing.assert_allclose(y, ref, rtol=2 ** -8, atol=0)


def test_forward_plain_constant_rows():
    """Plain BitLinear with a constant row c: every code is 127 and
    Y[n] = c * gamma * sum_k q[n, k]."""
    K, N = 128, 32
    X = bf16_bits(np.array([[0.5] * K, [-3.0] * K]))
    W = synth.latent_weights(N, K, seed=2)
    out = oracle.bitlinear_forward(X, W, hadamard=False, bits=8)
    assert np.all(np.abs(out["codes"]) == 127)
    rs = out["q"].astype(np.float64).sum(axis=1)
    for m, cval in enumerate([0.5, -3.0]):
        np.testing.assert_allclose(oracle.bf16_to_f64(out["y"][m]), cval * float(out["gamma"]) * rs,
                                   rtol=2 ** -8)


def test_forward_stages_compose():
    """The composite forward equals its own stages called one by one."""
    wl = synth.WORKLOADS["tiny"]
    X = wl.activations()
    W = wl.weights()
    out = oracle.bitlinear_forward(X, W, hadamard=True, bits=8)
    g = oracle.absmean_gamma(W)
    q = oracle.ternarize(W, g)
    z = oracle.fwht(oracle.bf16_to_f64(X))
    c, d, _, _ = oracle.quant_act(z.astype(np.float32), 8)
    acc = oracle.gemm_i64(c, q)
    assert out["gamma"] == g
    np.testing.assert_array_equal(out["q"], q)
    np.testing.assert_array_equal(out["codes"], c)
    np.testing.assert_array_equal(out["acc"], acc)
    np.testing.assert_array_equal(out["y"], oracle.dequant(acc, d, g))


# ----------------------------------------------------------------------------------------
# RMS normalisation before the quantiser (BitNet b1.58 2B4T article, 一.3: subln
# normalisation; BitNet v2 write-up: RMS normalisation)
# ----------------------------------------------------------------------------------------

def test_rmsnorm_matches_library_rms_norm():
    rng = np.random.default_rng(3)
    K = 256
    x = rng.normal(size=(5, K)) * 3.0
    g = bf16_bits(rng.uniform(0.5, 1.5, K))
    for eps in (0.0, 1e-5, 0.1):
        y = oracle.rmsnorm(x, g, eps)
        ref = torch.nn.functional.rms_norm(
            torch.from_numpy(x), (K,), weight=torch.from_numpy(oracle.bf16_to_f64(g)),
            eps=eps).numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-15)
    # no gain = unit gain
    np.testing.assert_allclose(oracle.rmsnorm(x, None, 1e-5),
                               oracle.rmsnorm(x, bf16_bits(np.ones(K)), 1e-5), rtol=0, atol=0)


def test_rmsnorm_invariants_and_closed_forms():
    rng = np.random.default_rng(4)
    x = rng.laplace(size=(4, 128))
    y = oracle.rmsnorm(x, None, 0.0)
    np.testing.assert_allclose((y ** 2).mean(axis=1), 1.0, rtol=1e-14)   # unit RMS
    np.testing.assert_allclose(oracle.rmsnorm(7.5 * x, None, 0.0), y, rtol=1e-14)  # scale
    np.testing.assert_allclose(oracle.rmsnorm(-x, None, 0.0), -y, rtol=0, atol=0)  # odd
    assert np.all(oracle.rmsnorm(np.zeros((2, 128)), None, 1e-5) == 0.0)            # zero row
    c, eps = 0.25, 1e-3
    g = bf16_bits(np.linspace(-2, 2, 128))
    row = oracle.rmsnorm(np.full((1, 128), c), g, eps)[0]
    np.testing.assert_allclose(row, c / math.sqrt(c * c + eps) * oracle.bf16_to_f64(g),
                               rtol=1e-15)


@pytest.mark.parametrize("hadamard", [True, False])
def test_forward_with_norm_composes_from_the_stages(hadamard):
    rng = np.random.default_rng(5)
    M, K, N = 6, 256, 64
    X = synth.sharp_activations(M, K, seed=11)
    W = synth.latent_weights(N, K, seed=12)
    g = bf16_bits(rng.uniform(0.5, 1.5, K))
    ref = oracle.bitlinear_forward(X, W, hadamard, 8, norm_gain=g, norm_eps=1e-5)
    y = oracle.rmsnorm(oracle.bf16_to_f64(X), g, 1e-5)
    z = oracle.fwht(y) if hadamard else y
    np.testing.assert_array_equal(ref["z"], z)
    codes, d, _, _ = oracle.quant_act(z.astype(np.float32), 8)
    np.testing.assert_array_equal(ref["codes"], codes)
    # without norm_eps the forward is the plain one
    plain = oracle.bitlinear_forward(X, W, hadamard, 8)
    np.testing.assert_array_equal(
        plain["z"], oracle.fwht(oracle.bf16_to_f64(X)) if hadamard else oracle.bf16_to_f64(X))


# ----------------------------------------------------------------------------------------
# Activations after the rescale (2B4T article, 一.3: squared ReLU; BitNet v2 write-up:
# SwishGLU), fused into the product's epilogue
# ----------------------------------------------------------------------------------------

def test_squared_relu_closed_forms():
    # d * gamma = 0.5 exactly, so v = acc / 2 and v^2 are exact in bf16
    acc = np.arange(-6, 7, dtype=np.int64).reshape(1, -1)
    y = oracle.bf16_to_f64(oracle.dequant_act(acc, np.array([0.25], np.float32), 2.0,
                                              oracle.RELU2))
    expect = np.where(acc > 0, (acc / 2.0) ** 2, 0.0)
    np.testing.assert_array_equal(y, expect)


def test_swiglu_against_library_silu():
    rng = np.random.default_rng(9)
    M, N = 7, 64
    acc = rng.integers(-3000, 3000, size=(M, N)).astype(np.int64)
    d = rng.uniform(1e-4, 3e-3, size=M).astype(np.float32)
    gamma = np.float32(0.4375)
    y = oracle.bf16_to_f64(oracle.dequant_act(acc, d, gamma, oracle.SWIGLU))
    v = torch.from_numpy(acc.astype(np.float64) * d.astype(np.float64)[:, None] * float(gamma))
    ref = (torch.nn.functional.silu(v[:, 0::2]) * v[:, 1::2]).numpy()
    ref_bf16 = oracle.bf16_to_f64(oracle.f64_to_bf16(ref))
    ulp = np.abs(ref_bf16) * 2.0 ** -7
    assert np.all(np.abs(y - ref_bf16) <= ulp + 1e-30)
    assert y.shape == (M, N // 2)


def test_swiglu_limits():
    acc = np.array([[0, 5, 400, 3, -400, 7]], dtype=np.int64)  # (gate, up) pairs
    y = oracle.bf16_to_f64(oracle.dequant_act(acc, np.array([0.1], np.float32), 1.0,
                                              oracle.SWIGLU))[0]
    s = float(np.float32(0.1))
    assert y[0] == 0.0                                   # silu(0) = 0
    assert y[1] == oracle.bf16_to_f64(oracle.f64_to_bf16(np.array([400 * s * 3 * s])))[0]
    assert abs(y[2]) < 1e-15                             # silu(-40) ~ -1.7e-16


# ----------------------------------------------------------------------------------------
# Base-3 rows for the decode product (2B4T article, 一.1: five ternary weights per byte)
# ----------------------------------------------------------------------------------------

def test_base3_rows_carry_the_page_example():
    # the first five weights of a row with offset codes 2,0,1,2,1 (q = 1,-1,0,1,0): byte 178
    q = np.zeros((2, 40), np.int8)
    q[1, :5] = [1, -1, 0, 1, 0]
    words = oracle.pack_ternary_base3(q)
    assert words.shape == (2, 2)
    assert words[1, 0] & 0xFF == 178
    # all-zero weights are offset code 1 everywhere: 1,1,1,1,1 -> 81+27+9+3+1 = 121 per byte
    assert words[0, 0] == 121 * 0x01010101


@pytest.mark.parametrize("K", [128, 2048, 8192, 384])
def test_base3_rows_round_trip_and_size(K):
    rng = np.random.default_rng(K)
    q = rng.integers(-1, 2, size=(5, K)).astype(np.int8)
    words = oracle.pack_ternary_base3(q)
    assert words.shape == (5, (K + 19) // 20)                 # 1.6 bits per weight, rounded up
    bytes_ = words.view(np.uint8)
    assert bytes_.max() < 243
    back, bad = oracle.unpack_ternary_base3(words, K)
    assert bad == 0
    np.testing.assert_array_equal(back, q)
    # brute force on one row: each byte is sum u_i 3^(4-i) over its five weights
    row = np.concatenate([q[2] + 1, np.ones((-K) % 20, np.int64)])
    expect = (row.reshape(-1, 5) * np.array([81, 27, 9, 3, 1])).sum(axis=1)
    np.testing.assert_array_equal(words[2].view(np.uint8), expect.astype(np.uint8))


# ----------------------------------------------------------------------------------------
# Low-bit Q / K / V states (BitNet v2 write-up, Tables 2 and 3: the QKV states' bit width
# varies; 3 bits match full precision).  The formula is a reading: the activations' absmax
# rule per token or per head, Q = 2^(bits-1) - 1.
# ----------------------------------------------------------------------------------------

def test_state_bitstream_hand_examples():
    g = golden("lowbit_state_bitstream.json")
    for case in g["cases"]:
        c = np.array([case["codes"]], np.int8)
        packed = oracle.pack_bits(c, case["bits"])
        np.testing.assert_array_equal(packed[0], np.array(case["bytes"], np.uint8))
        np.testing.assert_array_equal(oracle.unpack_bits(packed, c.shape[1], case["bits"]), c)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
def test_state_bitstream_round_trip(bits):
    rng = np.random.default_rng(bits)
    c = rng.integers(-(1 << (bits - 1)), 1 << (bits - 1), size=(5, 96)).astype(np.int8)
    packed = oracle.pack_bits(c, bits)
    assert packed.shape == (5, 96 * bits // 8)
    np.testing.assert_array_equal(oracle.unpack_bits(packed, 96, bits), c)


@pytest.mark.parametrize("bits,group", [(3, 64), (3, 512), (4, 128), (8, 512)])
def test_state_quant_brute_force_and_max_rule(bits, group):
    Q = (1 << (bits - 1)) - 1
    rng = np.random.default_rng(bits + group)
    x = bf16_bits(rng.standard_normal((6, 512)) * 0.7)
    x[2, :group] = 0  # one all-zero group: zero codes, guarded scale
    codes, d, pre = oracle.quant_states(x, group, bits)
    xf = oracle.bf16_to_f64(x).astype(np.float32)
    G = 512 // group
    xg = xf.reshape(6, G, group)
    mx = np.abs(xg).max(axis=2)
    gm = np.maximum(mx, np.float32(1e-5)).astype(np.float32)
    s = (np.float32(Q) / gm).astype(np.float32)
    v = (xg * s[..., None]).astype(np.float32)        # the fp32 product the decision uses
    ref = _nearest_code_brute(v.reshape(-1), -Q - 1, Q).reshape(6, 512)
    np.testing.assert_array_equal(codes, ref)
    np.testing.assert_array_equal(d, (gm / np.float32(Q)).astype(np.float32))
    # the largest |x| of each live group maps to +-Q
    cg = codes.reshape(6, G, group)
    for m in range(6):
        for g in range(G):
            if mx[m, g] > 0:
                k = int(np.argmax(np.abs(xg[m, g])))
                assert cg[m, g, k] == Q * np.sign(xg[m, g, k])
    assert not codes[2, :group].any() and d[2, 0] == np.float32(np.float32(1e-5) / np.float32(Q))
    # every code is within half a step of its value
    err = np.abs(codes.reshape(6, G, group) * d[..., None].astype(np.float64) - xg)
    assert np.all(err <= 0.5 * d[..., None] * (1 + 1e-6))


def test_state_quant_exact_ties_and_head_independence():
    # a group with max 1.5: s = 3 / 1.5 = 2 exactly; 0.25, 0.75, 1.25 land on 0.5, 1.5, 2.5
    row = np.zeros(64)
    row[:6] = [1.5, 0.25, 0.75, 1.25, -0.75, -1.25]
    x = bf16_bits(row[None, :])
    codes, d, pre = oracle.quant_states(x, 64, 3)
    np.testing.assert_array_equal(pre[0, :6], [3.0, 0.5, 1.5, 2.5, -1.5, -2.5])
    np.testing.assert_array_equal(codes[0, :6], [3, 0, 2, 2, -2, -2])   # ties to even
    assert d[0, 0] == np.float32(0.5)
    # per-head codes are the per-token rule applied to each head alone
    rng = np.random.default_rng(3)
    x = bf16_bits(rng.laplace(size=(4, 256)))
    c_head, d_head, _ = oracle.quant_states(x, 64, 3)
    for h in range(4):
        c1, d1, _ = oracle.quant_states(x[:, 64 * h:64 * (h + 1)], 64, 3)
        np.testing.assert_array_equal(c_head[:, 64 * h:64 * (h + 1)], c1)
        np.testing.assert_array_equal(d_head[:, h], d1[:, 0])
