"""Pins of the oracle's GPTQ column sweep against what the page prints and what the
mathematics fixes (no GPU): the calibration toy's printed output and weight errors, the
reduction to round-to-nearest when the Hessian is diagonal, and the closed form of the
sweep as a constrained least-squares problem, computed independently by linear solves."""
import json
import os

import numpy as np

import oracle
import wq_inputs


def _toy_grid(W, bits=3):
    """The toy's per-row symmetric grid, fixed up front: scale max|row| / (2^(bits-1) - 1)."""
    qmax = 2 ** (bits - 1) - 1
    scale = np.abs(W).max(axis=1) / qmax

    def qdq(i, w):
        return np.clip(np.rint(w / scale), -qmax - 1, qmax) * scale

    return qdq


def test_gptq_toy_printed_errors(golden_dir):
    """"GPTQ vs AWQ": on the toy's stream GPTQ reaches held-out output error 0.2272 while its
    weights move further from the originals (weight error 0.409 against RTN's 0.268)."""
    with open(os.path.join(golden_dir, "calibration_toy.json")) as f:
        g = json.load(f)
    W, X_cal, X_test = wq_inputs.calibration_toy_tensors()
    Q = oracle.gptq_sweep(W, oracle.gptq_hessian(X_cal, 0.01), _toy_grid(W, g["bits"]))
    Y = oracle.matmul_f64(X_test, W)
    assert round(oracle.rel_frobenius(Y, oracle.matmul_f64(X_test, Q)), 4) == g["output_error"]["gptq"]
    assert round(oracle.rel_frobenius(W, Q), 3) == g["weight_error"]["gptq"]


def test_gptq_with_diagonal_hessian_is_rtn():
    """Uncorrelated input channels (H diagonal): no error can be moved, so GPTQ returns the
    round-to-nearest result exactly, in the library's INT4 format too."""
    rng = np.random.default_rng(2)
    K = 256
    X = np.diag(rng.uniform(0.5, 3.0, K))            # orthogonal columns: H = X^T X diagonal
    W = rng.normal(0, 0.02, (6, K))
    c_rtn, S, Z = oracle.quantize_rtn_asym(W, 128)
    c_gptq, S2, Z2 = oracle.gptq_quantize_asym(W, X, 128)
    assert np.array_equal(c_rtn, c_gptq) and np.array_equal(S, S2) and np.array_equal(Z, Z2)
    q, Ss = oracle.quantize_rtn_sym_int4(W, 128)
    c_sym, S3, Z3 = oracle.gptq_quantize_asym(W, X, 128, sym=True)
    assert np.array_equal(c_sym.astype(np.int16) - 8, q) and np.array_equal(S3, Ss)
    assert np.all(Z3 == 8.0)
    Q = oracle.gptq_sweep(W, oracle.gptq_hessian(X), _toy_grid(W))
    scale = np.abs(W).max(axis=1, keepdims=True) / 3
    np.testing.assert_array_equal(Q, np.clip(np.rint(W / scale), -4, 3) * scale)


def test_gptq_sweep_is_constrained_least_squares():
    """After columns F = {0..i-1} are fixed at Q_F, the sweep's remaining weights minimise
    (w - W)^T H (w - W) with w_F = Q_F, i.e. w_R = W_R + H_RR^-1 H_RF (W_F - Q_F). The value
    each column has when its turn comes is checked against that formula, solved directly."""
    rng = np.random.default_rng(3)
    K, N = 12, 4
    X = rng.normal(0, 1, (40, K)) @ rng.normal(0, 1, (K, K))   # correlated channels
    W = rng.normal(0, 1, (N, K))
    H = oracle.gptq_hessian(X, 0.01)
    seen = {}
    grid = _toy_grid(W, 3)

    def qdq(i, w):
        seen[i] = w.copy()
        return grid(i, w)

    Q = oracle.gptq_sweep(W, H, qdq)
    for i in range(K):
        F, R = np.arange(i), np.arange(i, K)
        d = np.linalg.solve(H[np.ix_(R, R)], H[np.ix_(R, F)] @ (W[:, F] - Q[:, F]).T)
        expect = W[:, i] + d[0]
        np.testing.assert_allclose(seen[i], expect, rtol=1e-9, atol=1e-12)


def test_gptq_int4_lowers_calibration_error():
    """In the library's INT4 g128 format on the toy's correlated activations, GPTQ's output
    error on the calibration set is below round-to-nearest's (what the sweep minimises),
    with the same S' and Z."""
    W, X_cal, _ = wq_inputs.calibration_toy_tensors()
    c0, S, Z = oracle.quantize_rtn_asym(W, 128)
    c1, S1, Z1 = oracle.gptq_quantize_asym(W, X_cal, 128)
    assert np.array_equal(S, S1) and np.array_equal(Z, Z1)
    Y = oracle.matmul_f64(X_cal, W)
    e0 = oracle.rel_frobenius(Y, oracle.w4a16_matmul(X_cal, c0, S, Z, 128))
    e1 = oracle.rel_frobenius(Y, oracle.w4a16_matmul(X_cal, c1, S1, Z1, 128))
    assert e1 < 0.9 * e0
