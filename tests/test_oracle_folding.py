"""Pins of the oracle's per-input-channel scale folding (SmoothQuant and AWQ) against what the
pages print and what the mathematics fixes (no GPU).

Expected values come from the pages (tests/golden/*.json, with citations), closed forms of
the factor formulas, exact special cases (powers of two), library routines (numpy's float64
to float32 cast, torch's float32 to bfloat16 cast) and brute force in exact rationals; none
comes from the oracle itself or from the CUDA library.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import wq_inputs


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- page-printed values

def test_smoothquant_demo_printed_error(golden_dir):
    """"Granularity and outliers": with alpha = 0.5, per-token INT8 of X/s times
    per-output-channel INT8 of W*s has relative output error 0.0114 (printed), and the
    folded product equals X W^T (the demo's assertion)."""
    g = _load(golden_dir, "granularity_demo.json")
    W, X = wq_inputs.granularity_demo_tensors()
    s = oracle.smoothquant_scales(X, W, 0.5)
    Xs, Ws = oracle.fold_input_scales(X, W, s)
    Y = oracle.matmul_f64(X, W)
    np.testing.assert_allclose(oracle.matmul_f64(Xs, Ws), Y, rtol=1e-10, atol=1e-10)
    Yq = oracle.matmul_f64(oracle.qdq_sym(Xs, 8, axis=1), oracle.qdq_sym(Ws, 8, axis=1))
    assert round(oracle.rel_frobenius(Y, Yq), 4) == g["output_error"]["smoothquant_w8a8_alpha05"]
    # and smoothing is what helps: the naive W8A8 error (also printed) is over 4x larger
    assert g["output_error"]["naive_w8a8"] > 4 * g["output_error"]["smoothquant_w8a8_alpha05"]


def test_calibration_toy_printed_errors(golden_dir):
    """"GPTQ vs AWQ": on the toy's calibration stream, 3-bit per-row RTN has held-out output
    error 0.2684 and weight error 0.268; AWQ's search picks alpha = 0.3 and reaches 0.2128
    (all printed)."""
    g = _load(golden_dir, "calibration_toy.json")
    W, X_cal, X_test = wq_inputs.calibration_toy_tensors()

    def qdq(w):
        return oracle.qdq_sym(w, g["bits"], axis=1)

    def out_err(Q):
        return oracle.rel_frobenius(oracle.matmul_f64(X_test, W), oracle.matmul_f64(X_test, Q))

    Q_rtn = qdq(W)
    assert round(out_err(Q_rtn), 4) == g["output_error"]["rtn"]
    assert round(oracle.rel_frobenius(W, Q_rtn), 3) == g["weight_error"]["rtn"]
    Q_awq, a, s = oracle.awq_search(W, X_cal, np.linspace(0, 1, 11), qdq)
    assert round(a, 1) == g["awq_alpha"]
    assert round(out_err(Q_awq), 4) == g["output_error"]["awq"]
    assert s.shape == (W.shape[1],)


# ------------------------------------------------------------------ closed forms

def _stats_case(seed=5, tokens=9, out=5, K=13):
    """Non-square shapes so that a max over the wrong axis cannot go unnoticed."""
    rng = np.random.default_rng(seed)
    X = rng.normal(0, 1, (tokens, K)) * rng.uniform(0.5, 40, K)
    W = rng.normal(0, 0.05, (out, K)) * rng.uniform(0.5, 4, K)
    return X, W


@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.5, 0.8, 1.0])
def test_smooth_scales_migrate_the_column_maxima(alpha):
    """After folding, max|Xs_j| = xm_j / s_j = (xm_j wm_j)^(1 - alpha) and max|Ws_j| =
    wm_j s_j = (xm_j wm_j)^alpha, so their ratio is (xm_j wm_j)^(1 - 2 alpha) and their
    product xm_j wm_j: alpha = 0.5 balances the two column maxima at sqrt(xm_j wm_j); alpha
    = 1 makes every activation column peak at 1; alpha = 0 every weight column."""
    X, W = _stats_case()
    xm = np.abs(X).max(axis=0)
    wm = np.abs(W).max(axis=0)
    s = oracle.smoothquant_scales(X, W, alpha)
    Xs, Ws = oracle.fold_input_scales(X, W, s)
    mx, mw = np.abs(Xs).max(axis=0), np.abs(Ws).max(axis=0)
    np.testing.assert_allclose(mx / mw, (xm * wm) ** (1 - 2 * alpha), rtol=1e-12)
    np.testing.assert_allclose(mx * mw, xm * wm, rtol=1e-12)  # the product is invariant
    if alpha == 1.0:
        np.testing.assert_allclose(mx, 1.0, rtol=1e-14)
    if alpha == 0.0:
        np.testing.assert_allclose(mw, 1.0, rtol=1e-14)


def test_smooth_scales_dead_channels_and_statistics():
    X, W = _stats_case()
    X[:, 3] = 0.0
    W[:, 7] = 0.0
    s = oracle.smoothquant_scales(X, W, 0.5)
    assert s[3] == 1.0 and s[7] == 1.0
    assert np.all(s[[0, 1, 2, 4]] != 1.0)
    # the statistics by brute force
    for j in range(X.shape[1]):
        assert oracle.channel_absmax(X)[j] == max(abs(v) for v in X[:, j])
        assert oracle.channel_absmax(W)[j] == max(abs(v) for v in W[:, j])


def test_awq_scales_closed_forms():
    """s_i / s_j = (a_i / a_j)^alpha; max s * min s = 1; alpha = 0 gives all ones; a channel
    with zero magnitude gets 1 and does not enter the normalisation."""
    a = np.array([0.5, 2.0, 8.0, 1.0, 0.25, 3.0])
    for alpha in (0.0, 0.3, 0.7, 1.0):
        s = oracle.awq_scales(a, alpha)
        np.testing.assert_allclose(s / s[0], (a / a[0]) ** alpha, rtol=1e-14)
        assert math.isclose(s.max() * s.min(), 1.0, rel_tol=1e-14)
    assert np.all(oracle.awq_scales(a, 0.0) == 1.0)
    # alpha = 1: the extremes 8 and 0.25 normalise to 8/sqrt(2) and 0.25/sqrt(2)
    s1 = oracle.awq_scales(a, 1.0)
    assert math.isclose(s1[2], 8 / math.sqrt(2), rel_tol=1e-15)
    z = np.concatenate([a, [0.0]])
    sz = oracle.awq_scales(z, 0.5)
    assert sz[-1] == 1.0
    np.testing.assert_array_equal(sz[:-1], oracle.awq_scales(a, 0.5))


# ---------------------------------------------------------------- exact folding

def test_fold_identity_exact_with_powers_of_two():
    """(X/s)(W s)^T = X W^T: with integer-valued X, W and power-of-two s every product is
    unchanged and every sum exact, so the identity holds bit for bit; a factor applied on
    the wrong axis (or multiplied on both sides) breaks it."""
    rng = np.random.default_rng(11)
    X = rng.integers(-50, 50, (6, 40)).astype(np.float64)
    W = rng.integers(-50, 50, (7, 40)).astype(np.float64)
    s = 2.0 ** rng.integers(-6, 7, 40)
    Xs, Ws = oracle.fold_input_scales(X, W, s)
    np.testing.assert_array_equal(oracle.matmul_f64(Xs, Ws), oracle.matmul_f64(X, W))
    np.testing.assert_array_equal(Ws[:, 5], W[:, 5] * s[5])
    np.testing.assert_array_equal(Xs[2], X[2] / s)
    # random factors: equal up to float64 rounding
    s2 = np.exp(rng.normal(0, 1, 40))
    Xs2, Ws2 = oracle.fold_input_scales(X, W, s2)
    np.testing.assert_allclose(oracle.matmul_f64(Xs2, Ws2), oracle.matmul_f64(X, W),
                               rtol=1e-12, atol=1e-9)
    for bad in (0.0, -1.0, np.inf, np.nan):
        sb = s.copy()
        sb[3] = bad
        with pytest.raises(ValueError):
            oracle.fold_input_scales(X, W, sb)


def test_f32_round_against_numpy_and_ties():
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.normal(0, 1, 200), rng.normal(0, 1, 50) * 1e-40,
                           rng.normal(0, 1, 50) * 1e30])
    for v in vals:
        assert oracle.f32_round(float(v)) == float(np.float32(v)), v   # numpy's cast
    one = Fraction(1)
    assert oracle.f32_round(one + Fraction(1, 2 ** 24)) == 1.0                 # tie -> even
    assert oracle.f32_round(one + Fraction(3, 2 ** 24)) == 1.0 + 2.0 ** -22    # tie -> even
    assert oracle.f32_round(one + Fraction(1, 2 ** 24) + Fraction(1, 2 ** 80)) == 1.0 + 2.0 ** -23
    assert oracle.f32_round(Fraction(2 ** 128)) == math.inf
    assert oracle.f32_round(Fraction(1, 2 ** 150)) == 0.0                      # half min subnormal
    assert oracle.f32_round(Fraction(3, 2 ** 151)) == 2.0 ** -149


def test_fold_weight_f32_is_one_rounding_of_the_exact_product():
    """Brute force in rationals: fp32(w s) for bf16 w and fp32 s, including products that
    need rounding."""
    rng = np.random.default_rng(4)
    Wb = wq_inputs.bf16_bits_to_f64(wq_inputs.to_bf16_bits(rng.normal(0, 0.02, (3, 16))))
    s = rng.uniform(0.1, 9, 16).astype(np.float32).astype(np.float64)
    F = oracle.fold_weight_f32(Wb, s)
    for n in range(3):
        for k in range(16):
            assert F[n, k] == oracle.f32_round(Fraction(Wb[n, k]) * Fraction(s[k]))
    with pytest.raises(oracle.NonFiniteError):
        oracle.fold_weight_f32(np.array([[3e38, 1.0]]), np.array([4.0, 1.0]))


def test_quantize_rtn_scaled_reductions():
    """s = 1 gives the unscaled quantizer; W = V / s with power-of-two s folds back to V
    exactly, so the codes are V's; a constant power-of-two s keeps the codes and zero-points
    and scales S' by that power (inside binary16's normal range)."""
    rng = np.random.default_rng(6)
    V = wq_inputs.bf16_bits_to_f64(wq_inputs.to_bf16_bits(rng.normal(0, 0.02, (4, 256))))
    c0, S0, Z0 = oracle.quantize_rtn_asym(V, 128)
    c1, S1, Z1 = oracle.quantize_rtn_scaled(V, np.ones(256), 128)
    assert np.array_equal(c0, c1) and np.array_equal(S0, S1) and np.array_equal(Z0, Z1)
    s = 2.0 ** rng.integers(-5, 6, 256)
    c2, S2, Z2 = oracle.quantize_rtn_scaled(V / s, s, 128)
    assert np.array_equal(c0, c2) and np.array_equal(S0, S2) and np.array_equal(Z0, Z2)
    c3, S3, Z3 = oracle.quantize_rtn_scaled(V, np.full(256, 8.0), 128)
    assert np.array_equal(c0, c3) and np.array_equal(Z0, Z3)
    np.testing.assert_array_equal(S3, 8.0 * S0)
    # symmetric storage: Z = 8 everywhere and the same reduction
    q, Ss = oracle.quantize_rtn_sym_int4(V, 128)
    c4, S4, Z4 = oracle.quantize_rtn_scaled(V / s, s, 128, sym=True)
    assert np.array_equal(c4.astype(np.int16) - 8, q) and np.array_equal(S4, Ss)
    assert np.all(Z4 == 8.0)
    with pytest.raises(ValueError):
        oracle.quantize_rtn_scaled(V, np.zeros(256), 128)


def test_scale_activations_bf16_brute_force():
    """bf16 bits of X/s: power-of-two s is an exact exponent shift; s = 1 is the identity;
    in general the correctly rounded float32 quotient (exact rationals) rounded to bf16 by
    torch's cast."""
    import torch

    rng = np.random.default_rng(8)
    Xb = wq_inputs.to_bf16_bits(rng.normal(0, 3, (3, 24)))
    X = wq_inputs.bf16_bits_to_f64(Xb)
    np.testing.assert_array_equal(oracle.scale_activations_bf16(X, np.ones(24)), Xb)
    p2 = 2.0 ** rng.integers(-4, 5, 24)
    np.testing.assert_array_equal(
        wq_inputs.bf16_bits_to_f64(oracle.scale_activations_bf16(X, p2)), X / p2)
    s = rng.uniform(0.05, 20, 24).astype(np.float32).astype(np.float64)
    got = oracle.scale_activations_bf16(X, s)
    for m in range(3):
        for k in range(24):
            q32 = np.float32(oracle.f32_round(Fraction(X[m, k]) / Fraction(s[k])))
            want = torch.tensor(q32).to(torch.bfloat16).view(torch.int16).item() & 0xFFFF
            assert int(got[m, k]) == want


def test_channel_absmean_brute_force():
    """mean |A_ij| per column: the exact rational mean rounded once to float32, on bf16 and
    float32 data (sums that fit 53 bits, so every correct summation order agrees)."""
    rng = np.random.default_rng(9)
    for A in (wq_inputs.bf16_bits_to_f64(wq_inputs.to_bf16_bits(rng.normal(0, 2, (37, 16)))),
              rng.normal(0, 1, (11, 8)).astype(np.float32).astype(np.float64)):
        got = oracle.channel_absmean(A)
        for j in range(A.shape[1]):
            exact = sum(abs(Fraction(v)) for v in A[:, j]) / A.shape[0]
            assert got[j] == oracle.f32_round(exact)
