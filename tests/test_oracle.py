"""Pins of the CPU oracle against what the pages and mathematics fix (no GPU).

Each test names what it pins. Expected values come from the pages (tests/golden/*.json,
each with its citation), from hand derivations, from library routines for special
cases (numpy's float64->float16 cast, torch's float32->bfloat16 cast), or from brute
force on tiny inputs; none come from the oracle itself or from the CUDA library.
"""
import bisect
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

def test_int8_worked_example_full_precision_scale(golden_dir):
    """DL S067 section 1 numeric example: q, x_hat and the infinity-norm error."""
    g = _load(golden_dir, "int8_worked_example.json")
    x = np.array(g["x"])
    x_hat = oracle.qdq_sym(x, 8)
    s = np.abs(x).max() / 127
    assert round(s, 5) == g["scale_printed"]
    assert np.array_equal(np.rint(x / s), g["q"])
    assert np.array_equal(np.round(x_hat, 3), g["x_hat_3dp"])
    assert round(float(np.abs(x - x_hat).max()), 3) == g["err_inf_3dp"]


def test_int8_worked_example_fp16_scale(golden_dir):
    """Same example through the stored-scale quantizer: codes identical to the page;
    the binary16 scale moves x_hat by less than half a printed digit's step + 1e-3."""
    g = _load(golden_dir, "int8_worked_example.json")
    x = np.array(g["x"], dtype=np.float32).astype(np.float64)[None, :]
    q, s = oracle.quantize_sym_int8_per_channel(x)
    assert s[0] == float(np.float16(1.2 / 127))
    assert q.tolist() == [g["q"]]
    x_hat = oracle.dequant_sym_per_channel(q, s)[0]
    assert np.max(np.abs(x_hat - np.array(g["x_hat_3dp"]))) < 1e-3


def test_granularity_demo_values(golden_dir):
    """Study-docs granularity demo: symmetric qdq errors at four granularities and the
    W8A8 / W8A16 output errors, to every printed digit."""
    g = _load(golden_dir, "granularity_demo.json")
    W, X = wq_inputs.granularity_demo_tensors()
    we = g["weight_error"]
    assert round(oracle.rel_frobenius(W, oracle.qdq_sym(W, 8)), 4) == we["int8_per_tensor"]
    assert round(oracle.rel_frobenius(W, oracle.qdq_sym(W, 8, axis=1)), 4) == we["int8_per_channel"]
    assert round(oracle.rel_frobenius(W, oracle.qdq_sym(W, 4, axis=1)), 4) == we["int4_per_channel"]
    assert round(oracle.rel_frobenius(W, oracle.qdq_sym(W, 4, group=128)), 4) == we["int4_group128"]
    Y = oracle.matmul_f64(X, W)
    oe = g["output_error"]
    Yq = oracle.matmul_f64(oracle.qdq_sym(X, 8, axis=1), oracle.qdq_sym(W, 8, axis=1))
    assert round(oracle.rel_frobenius(Y, Yq), 4) == oe["naive_w8a8"]
    Yw = oracle.matmul_f64(X, oracle.qdq_sym(W, 8, axis=1))
    assert round(oracle.rel_frobenius(Y, Yw), 4) == oe["weight_only_w8a16"]


def test_format_math(golden_dir):
    """Bits per weight 4 + 16/128 and the batch-1 decode ceilings printed by the
    format-math snippet (these pin the byte model the benchmark uses)."""
    g = _load(golden_dir, "format_math.json")
    assert oracle.bits_per_weight(4, 128) == g["bits_per_weight"]["INT4_g128"]
    assert oracle.bits_per_weight(4, 128, zero_bits=16) == 4.25
    for row in g["ceilings_tok_s"]:
        bpw = g["bits_per_weight"][row["format"]]
        v = oracle.decode_ceiling_tok_s(row["params"], bpw, g["bandwidth_bytes_s"], row["gpus"])
        assert round(v) == row["value"], row


# --------------------------------------------------------------- hand-derived values

def test_asym_int4_hand_examples(golden_dir):
    """Hand-worked asymmetric INT4 groups: S', Z, codes, packing, dequant; a 4x8 matrix
    with g=4, so a transposed grouping or a swapped nibble order fails."""
    g = _load(golden_dir, "asym_int4_hand.json")
    W = np.array(g["W"], dtype=np.float64)
    assert np.array_equal(W.astype(np.float32).astype(np.float64), W)
    codes, S, Z = oracle.quantize_rtn_asym(W, g["group"])
    assert S.tolist() == g["S"]
    assert Z.tolist() == g["Z"]
    assert codes.tolist() == g["q"]
    assert oracle.pack_int4(codes)[0].tolist() == g["packed_row0"]
    W_hat = oracle.dequant_asym(codes, S, Z, g["group"])
    assert W_hat[0, :4].tolist() == [-0.375, 1.5, 0.0, 0.5]


def test_pack_roundtrip_and_order():
    codes = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    p = oracle.pack_int4(codes)
    assert p.tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(oracle.unpack_int4(p), codes)
    rng = np.random.default_rng(5)
    c = rng.integers(0, 16, (7, 40), dtype=np.uint8)
    assert np.array_equal(oracle.unpack_int4(oracle.pack_int4(c)), c)


# ---------------------------------------------------------------- roundings vs library

def test_fp16_round_matches_numpy_on_floats():
    """For float64 inputs, exact binary16 rounding equals numpy's float64->float16 cast."""
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.normal(0, 1, 2000) * 10.0 ** rng.integers(-9, 5, 2000),
        [1 + 2 ** -11, 1 + 3 * 2 ** -11, 65504.0, 65519.99, 65520.0, 2 ** -25,
         3 * 2 ** -26, 2 ** -24, 2 ** -14, 2 ** -14 - 2 ** -25, 1e-30, -0.2],
    ])
    for v in vals:
        assert oracle.fp16_round(Fraction(float(v))) == float(np.float16(v)), v


def test_fp16_round_exact_rational_tie():
    """A value just above a binary16 tie by less than a float64 ulp rounds up; the
    tie itself rounds to even."""
    t = Fraction(1) + Fraction(1, 2 ** 11)
    assert oracle.fp16_round(t) == 1.0
    assert oracle.fp16_round(t + Fraction(1, 2 ** 100)) == 1.0009765625
    assert oracle.fp16_round(t - Fraction(1, 2 ** 100)) == 1.0


def test_fp16_round_brute_force():
    """Nearest finite binary16 value by search over all of them, ties to even code."""
    allv = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    rng = np.random.default_rng(3)
    for _ in range(300):
        r = Fraction(int(rng.integers(1, 10 ** 9)), int(rng.integers(1, 10 ** 9))) \
            * Fraction(2) ** int(rng.integers(-26, 14))
        i = bisect.bisect_left(allv.tolist(), float(r))
        cands = [j for j in (i - 1, i, i + 1) if 0 <= j < len(allv)]
        best = min(cands, key=lambda j: (abs(Fraction(float(allv[j])) - r), j % 2))
        assert oracle.fp16_round(r) == float(allv[best])


def test_bf16_round_matches_torch():
    import torch
    rng = np.random.default_rng(4)
    x = (rng.normal(0, 1, 5000) * 10.0 ** rng.integers(-6, 6, 5000)).astype(np.float32)
    # exact ties: low 16 bits = 0x8000
    ties = (rng.integers(0, 2 ** 31, 200, dtype=np.uint32) & 0xFFFF0000 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties[np.isfinite(ties)]])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_round_bits(x.astype(np.float64)), ref)


# ------------------------------------------------------------- brute force / invariants

def _brute_scale(alpha, beta):
    """S' by exhaustive nearest search over binary16 values, Z by nearest integer."""
    allv = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    target = (Fraction(beta) - Fraction(alpha)) / 15
    best = min(range(len(allv)), key=lambda j: (abs(Fraction(float(allv[j])) - target), j % 2))
    s = float(allv[best]) or 1.0
    zt = -Fraction(alpha) / Fraction(s)
    z = min((abs(zt - k), k % 2, k) for k in range(0, 40))[2]
    return s, float(min(max(z, 0), 15))


def _brute_codes(w, s, z):
    """Nearest of the 16 levels s*(q - z); on a tie, the level with (q - z) even."""
    out = []
    for x in w:
        fx = Fraction(float(x))
        out.append(min(range(16), key=lambda q: (abs(fx - Fraction(s) * (q - int(z))),
                                                 (q - int(z)) % 2)))
    return out


def test_rtn_brute_force_tiny():
    rng = np.random.default_rng(8)
    cases = [rng.normal(0, 0.02, 16), rng.normal(0.3, 0.01, 16), -np.abs(rng.normal(0, 1, 16)),
             rng.normal(0, 1e-6, 16), rng.normal(0, 300.0, 16)]
    # exact half-integer ties w = (k + 1/2) S' with S' a power of two
    tie = np.array([-0.5, 0.0, 7.5, -6.5, 2.5, 1.5, 0.5, -3.5]) * 0.5
    tie = np.concatenate([tie, [-8.0 * 0.5 * 15 / 15, 7.5 * 0.5]])
    cases.append(tie)
    for w in cases:
        w = w.astype(np.float32).astype(np.float64)
        codes, S, Z = oracle.quantize_rtn_asym(w[None, :], len(w))
        a, b = min(0.0, w.min()), max(0.0, w.max())
        s_bf, z_bf = _brute_scale(a, b)
        assert (S[0, 0], Z[0, 0]) == (s_bf, z_bf)
        assert codes[0].tolist() == _brute_codes(w, s_bf, z_bf)


def test_rtn_invariants_tiny_config():
    """On the tiny config: Z integral in [0, 15]; scales positive binary16; the error
    bound |w - w_hat| <= S'/2 + 15 max(0, S - S'); zero maps to zero exactly."""
    W, _ = wq_inputs.tiny_config()
    W = W.astype(np.float64)
    W[3, 5] = 0.0
    codes, S, Z = oracle.quantize_rtn_asym(W, 128)
    assert S.shape == (256, 4) and codes.shape == (256, 512)
    assert np.all(Z == np.rint(Z)) and Z.min() >= 0 and Z.max() <= 15
    assert np.all(S > 0) and np.array_equal(S.astype(np.float16).astype(np.float64), S)
    W_hat = oracle.dequant_asym(codes, S, Z, 128)
    assert oracle.error_bound_ok(W, W_hat, S, 128)
    assert W_hat[3, 5] == 0.0
    # each group's minimum lands on code 0 (RNE is odd-symmetric, so RNE(alpha/S') + Z
    # = 0); its maximum on 15, or 14 when S' rounded up or -alpha/S' was a tie
    g = codes.reshape(256, 4, 128)
    Wg = W.reshape(256, 4, 128)
    ix = (np.arange(256)[:, None], np.arange(4)[None, :])
    assert np.all(g[ix + (Wg.argmin(-1),)] == 0)
    top = g[ix + (Wg.argmax(-1),)]
    assert np.all((top == 15) | (top == 14)) and np.mean(top == 15) > 0.5


def test_rtn_per_channel_and_per_tensor():
    rng = np.random.default_rng(9)
    W = rng.normal(0, 0.05, (6, 64)).astype(np.float32).astype(np.float64)
    for group in (64, 0):
        codes, S, Z = oracle.quantize_rtn_asym(W, group)
        flat = W.reshape(-1, 64) if group else W.reshape(1, -1)
        for r in range(flat.shape[0]):
            s_bf, z_bf = _brute_scale(min(0.0, flat[r].min()), max(0.0, flat[r].max()))
            assert (S[r, 0], Z[r, 0]) == (s_bf, z_bf)
        W_hat = oracle.dequant_asym(codes, S, Z, group)
        assert oracle.error_bound_ok(W, W_hat, S, group)


def test_rtn_subnormal_scale_clips_zero_point():
    """A group whose scale is a binary16 subnormal far below S: Z is clipped to 15 and
    the widened error bound still holds."""
    w = np.array([-1.35 * 15 * 2 ** -24 * 0.999, 1e-12, 0.0, 0.0]).astype(np.float32).astype(np.float64)
    codes, S, Z = oracle.quantize_rtn_asym(w[None, :], 4)
    assert S[0, 0] == 2.0 ** -24
    assert Z[0, 0] == 15.0
    W_hat = oracle.dequant_asym(codes, S, Z, 4)
    assert oracle.error_bound_ok(w[None, :], W_hat, S, 4)


def test_rtn_errors():
    with pytest.raises(oracle.NonFiniteError):
        oracle.quantize_rtn_asym(np.array([[0.0, np.nan, 1.0, 2.0]]), 4)
    with pytest.raises(oracle.NonFiniteError):
        oracle.quantize_rtn_asym(np.array([[0.0, 1e6, 1.0, 2.0]]), 4)
    with pytest.raises(ValueError):
        oracle.quantize_rtn_asym(np.zeros((2, 12)), 8)


def test_int8_per_channel_invariants():
    rng = np.random.default_rng(10)
    W = rng.normal(0, 0.02, (16, 256)).astype(np.float32).astype(np.float64)
    q, s = oracle.quantize_sym_int8_per_channel(W)
    assert q.dtype == np.int8 and q.min() >= -127 and q.max() <= 127
    for r in range(16):
        amax = np.abs(W[r]).max()
        assert s[r] == float(np.float16(amax / 127))
        assert abs(int(q[r, np.abs(W[r]).argmax()])) == 127
        err = np.abs(W[r] - q[r] * s[r]).max()
        assert err <= s[r] / 2 + 127 * max(0.0, amax / 127 - s[r]) + 1e-15


# ---------------------------------------------------------------------------- matmul

def test_matmul_brute_force():
    """Y = X W^T against pure-Python exactly rounded sums on a non-square case."""
    rng = np.random.default_rng(12)
    X = rng.normal(0, 1, (3, 8))
    W = rng.normal(0, 1, (5, 8))
    Y = oracle.matmul_f64(X, W)
    assert Y.shape == (3, 5)
    for m in range(3):
        for n in range(5):
            ref = math.fsum(X[m, k] * W[n, k] for k in range(8))
            assert abs(Y[m, n] - ref) <= 1e-14 * (1 + abs(ref))


def test_w4a16_matmul_modes():
    """exact mode = X (S'(q-Z))^T; bf16 mode rounds each S'(q-Z) to bfloat16 first,
    checked against a per-element loop with torch's cast."""
    import torch
    rng = np.random.default_rng(13)
    W = rng.normal(0, 0.02, (4, 256)).astype(np.float32).astype(np.float64)
    X = rng.normal(0, 1, (2, 256))
    codes, S, Z = oracle.quantize_rtn_asym(W, 128)
    Y = oracle.w4a16_matmul(X, codes, S, Z, 128, "exact")
    Yb = oracle.w4a16_matmul(X, codes, S, Z, 128, "bf16")
    for m in range(2):
        for n in range(4):
            wh = [S[n, k // 128] * (int(codes[n, k]) - Z[n, k // 128]) for k in range(256)]
            assert abs(Y[m, n] - math.fsum(X[m, k] * wh[k] for k in range(256))) < 1e-12
            whb = torch.tensor(wh, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).tolist()
            assert abs(Yb[m, n] - math.fsum(X[m, k] * whb[k] for k in range(256))) < 1e-12


def test_gemm_gate():
    ref = np.array([1.0, -2.0, 0.0, 4.0])
    assert oracle.gemm_gate(ref, ref) == 0.0
    rms = math.sqrt(np.mean(ref ** 2))
    assert math.isclose(oracle.gemm_gate(ref + [0, 0, 1e-3, 0], ref), 1e-3 / (1e-3 * rms))
    assert math.isclose(oracle.gemm_gate(ref * 1.01, ref), 0.01)
    # with K, the floor is 100 x (K/16) fp32 ulps of rms: 100 * 2048 * 2^-23 = 0.0244 at
    # K = 32768, and never below 1e-3
    assert math.isclose(oracle.gemm_gate(ref + [0, 0, 1e-3, 0], ref, 32768),
                        1e-3 / (100 * 2048 * 2.0 ** -23 * rms))
    assert oracle.gemm_gate(ref + [0, 0, 1e-3, 0], ref, 16) == oracle.gemm_gate(
        ref + [0, 0, 1e-3, 0], ref)
    assert math.isclose(oracle.gemm_gate(ref * 1.01, ref, 32768), 0.01)  # large outputs: relative


def test_outlier_quality_ordering():
    """Finer groups quantize outlier-heavy weights better: g=128 < per-channel < per-tensor
    (ordering stated by both DL S067 section 2 and the study-docs granularity section)."""
    Wb, Xb, cols = wq_inputs.outlier_config(N=64, K=1024, M=8)
    W = wq_inputs.bf16_bits_to_f64(Wb)
    X = wq_inputs.bf16_bits_to_f64(Xb)
    assert len(cols) == 1
    e = {g: oracle.outlier_quality(W, X, g) for g in (128, 1024, 0)}
    assert e[128][0] < e[1024][0] < e[0][0]
    # output errors are reported, not ordered: with one outlier column they are dominated
    # by that column's rounding at any granularity
    assert all(0 < e[g][1] < 1 for g in e)


# --------------------------------------------------- symmetric INT4 per group [GR]

def _brute_sym_scale(w):
    """s' by exhaustive nearest search over binary16 values of max|w| / 7 (ties to even)."""
    allv = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    target = Fraction(float(np.abs(w).max())) / 7
    j = bisect.bisect_left(allv.tolist(), float(target))
    cands = [k for k in (j - 1, j, j + 1) if 0 <= k < len(allv)]
    best = min(cands, key=lambda k: (abs(Fraction(float(allv[k])) - target), k % 2))
    return float(allv[best]) or 1.0


def _brute_sym_codes(w, s):
    """Nearest of the 16 levels s*q, q in [-8, 7]; on a tie the even q."""
    return [min(range(-8, 8), key=lambda q: (abs(Fraction(float(x)) - Fraction(s) * q), q % 2))
            for x in w]


def test_sym_int4_brute_force_tiny():
    """Scale and codes against exhaustive searches: the nearest binary16 to max|w|/7, and
    the nearest of the 16 levels s'q, ties to even q."""
    rng = np.random.default_rng(21)
    cases = [rng.normal(0, 0.02, 16), rng.normal(0.3, 0.01, 16), -np.abs(rng.normal(0, 1, 16)),
             rng.normal(0, 1e-6, 16), rng.normal(0, 300.0, 16), np.zeros(16),
             np.full(16, 0.37), np.full(16, -2.5)]
    tie = np.array([0.5, -0.5, 1.5, -2.5, 3.5, 6.5, -6.5, 7.0]) * 0.25  # s' = 0.25 exactly
    cases.append(tie)
    for w in cases:
        w = w.astype(np.float32).astype(np.float64)
        q, S = oracle.quantize_rtn_sym_int4(w[None, :], len(w))
        s_bf = _brute_sym_scale(w)
        assert S[0, 0] == s_bf
        assert q[0].tolist() == _brute_sym_codes(w, s_bf)


def test_sym_int4_special_cases():
    """All-zero group: s' = 1, q = 0. A constant group c maps to 7 (or -7): c/s' lies
    within one binary16 step of 7. The ties of the exact grid go to even q."""
    q, S = oracle.quantize_rtn_sym_int4(np.zeros((1, 32)), 32)
    assert S[0, 0] == 1.0 and not q.any()
    for c in (0.37, -2.5, 1e-3, 123.0):
        q, _ = oracle.quantize_rtn_sym_int4(np.full((2, 64), c, dtype=np.float32).astype(np.float64), 32)
        assert (q == (7 if c > 0 else -7)).all()
    # group max 1.75 -> s' = 0.25 exactly; 0.125 * (2k + 1) are ties between k and k + 1
    w = np.array([1.75] + [0.125 * (2 * k + 1) for k in range(-7, 7)] + [0.0])
    q, S = oracle.quantize_rtn_sym_int4(w[None, :], len(w))
    assert S[0, 0] == 0.25
    expect = [7] + [k if k % 2 == 0 else k + 1 for k in range(-7, 7)] + [0]
    assert q[0].tolist() == expect


def test_sym_int4_equals_pinned_qdq_when_scale_exact():
    """Where every group's max|w| / 7 is a binary16 value (so storing the scale changes
    nothing), s'q equals qdq_sym(W, 4, group=g), which the printed granularity demo pins."""
    rng = np.random.default_rng(22)
    N, K, g = 8, 512, 128
    W = rng.normal(0, 0.02, (N, K))
    for r in range(N):
        for j in range(K // g):
            blk = W[r, j * g:(j + 1) * g]
            m = float(np.float16(np.abs(blk).max() / 7)) * 7  # a group max that is 7 x binary16
            blk *= m / np.abs(blk).max()
    W = W.astype(np.float32).astype(np.float64)
    q, S = oracle.quantize_rtn_sym_int4(W, g)
    assert np.all(np.abs(W).reshape(N, -1, g).max(axis=-1) / 7 == S)  # scales exact
    What = (q.reshape(N, -1, g) * S[:, :, None]).reshape(N, K)
    assert np.array_equal(What, oracle.qdq_sym(W, 4, group=g))


def test_sym_int4_storage_roundtrip():
    """Stored as code q + 8 with Z = 8, the asymmetric dequant gives s'q exactly."""
    W, _ = wq_inputs.tiny_config()
    q, S = oracle.quantize_rtn_sym_int4(W.astype(np.float64), 128)
    codes, S2, Z = oracle.sym_int4_storage(q, S)
    assert codes.min() >= 0 and codes.max() <= 15 and (Z == 8).all()
    assert np.array_equal(oracle.dequant_asym(codes, S2, Z, 128),
                          (q.reshape(q.shape[0], -1, 128) * S[:, :, None]).reshape(q.shape))


def test_sym_int4_hand_examples(golden_dir):
    """Hand-worked symmetric INT4 groups (g = 4 on a 3 x 8 matrix, so a transposed grouping
    fails): s', codes, the stored form (q + 8, Z = 8) and its packing."""
    g = _load(golden_dir, "sym_int4_hand.json")
    W = np.array(g["W"], dtype=np.float64)
    q, S = oracle.quantize_rtn_sym_int4(W, g["group"])
    assert S.tolist() == g["S"]
    assert q.tolist() == g["q"]
    codes, _, Z = oracle.sym_int4_storage(q, S)
    assert (Z == 8).all()
    assert oracle.pack_int4(codes)[0].tolist() == g["packed_row0"]


# ------------------------------------------- pins of the remaining checker functions

def test_w8a16_matmul_modes():
    """W8A16 on the same dequantized weights: exact mode = X (s' q)^T, bf16 mode rounds each
    s' q to bfloat16 first; both against a per-element math.fsum loop, the bf16 weights
    through torch's float32 -> bfloat16 cast (not the oracle's own rounding)."""
    import torch
    rng = np.random.default_rng(31)
    W = rng.normal(0, 0.02, (5, 96)).astype(np.float32).astype(np.float64)
    X = rng.normal(0, 1, (3, 96))
    q, s = oracle.quantize_sym_int8_per_channel(W)
    Y = oracle.w8a16_matmul(X, q, s, "exact")
    Yb = oracle.w8a16_matmul(X, q, s, "bf16")
    assert Y.shape == Yb.shape == (3, 5)
    for n in range(5):
        wh = [float(s[n]) * int(q[n, k]) for k in range(96)]
        whb = torch.tensor(wh, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).tolist()
        # the bf16 rounding really moves some weights here, so the two modes differ
        assert any(a != b for a, b in zip(wh, whb))
        for m in range(3):
            assert abs(Y[m, n] - math.fsum(X[m, k] * wh[k] for k in range(96))) < 1e-12
            assert abs(Yb[m, n] - math.fsum(X[m, k] * whb[k] for k in range(96))) < 1e-12
    with pytest.raises(ValueError):
        oracle.w8a16_matmul(X, q, s, "fp8")


def test_error_bound_ok_rejects_violations():
    """error_bound_ok is a checker, so it must also say no: a dequantized weight moved to
    just beyond S'/2 (+ 15 max(0, S - S')) from w is rejected, one exactly on the bound is
    accepted. Two groups: one where binary16 rounded S up (bound S'/2) and one where it
    rounded S down (bound widened by 15 (S - S'))."""
    # group A: range 4.5 -> S = 0.3, S' = fp16(0.3) = 0.300048828125 > S
    # group B: range 1.5 -> S = 0.1, S' = fp16(0.1) = 0.0999755859375 < S
    wa = np.array([0.0, 4.5, 1.3, 2.2])
    wb = np.array([0.0, 1.5, 0.7, 0.2])
    W = np.stack([np.concatenate([wa, wb])]).astype(np.float32).astype(np.float64)
    S = np.array([[0.300048828125, 0.0999755859375]])
    assert S.tolist() == [[float(np.float16(0.3)), float(np.float16(0.1))]]
    s_exact = [Fraction(9, 2) / 15, Fraction(3, 2) / 15]
    assert Fraction(S[0, 0]) > s_exact[0] and Fraction(S[0, 1]) < s_exact[1]
    bounds = [Fraction(S[0, 0]) / 2,
              Fraction(S[0, 1]) / 2 + 15 * (s_exact[1] - Fraction(S[0, 1]))]
    for g, elem in ((0, 2), (1, 6)):
        for sign in (1, -1):
            on = W.copy()
            on[0, elem] = float(Fraction(float(W[0, elem])) + sign * bounds[g])
            # the sum is exact in float64 here (a few bits each), so `on` sits on the bound
            assert Fraction(on[0, elem]) - Fraction(float(W[0, elem])) == sign * bounds[g]
            assert oracle.error_bound_ok(W, on, S, 4)
            off = on.copy()
            off[0, elem] = float(np.nextafter(on[0, elem], sign * np.inf))
            assert not oracle.error_bound_ok(W, off, S, 4)
    # an all-zero group has bound 0: any nonzero W_hat there is rejected
    Wz = np.zeros((1, 4))
    assert oracle.error_bound_ok(Wz, Wz, np.ones((1, 1)), 4)
    assert not oracle.error_bound_ok(Wz, Wz + [[0, 0, 2.0 ** -30, 0]], np.ones((1, 1)), 4)


def _brute_group_dequant(w):
    """One group's dequantized weights from the brute-force searches alone: S' as the
    nearest binary16 to the exact range / 15, Z and codes as the nearest levels."""
    a, b = min(0.0, float(np.min(w))), max(0.0, float(np.max(w)))
    s, z = _brute_scale(a, b)
    return [s * (q - int(z)) for q in _brute_codes(w, s, z)]


def _fsum_frobenius_rel(A, B):
    """||A - B||_F / ||A||_F with exactly rounded sums of squares."""
    num = math.fsum((float(x) - float(y)) ** 2 for x, y in zip(np.ravel(A), np.ravel(B)))
    den = math.fsum(float(x) ** 2 for x in np.ravel(A))
    return math.sqrt(num / den)


def test_outlier_quality_brute_force():
    """outlier_quality recomputed on a tiny outlier case (4 x 256, two outlier input
    columns x 20-100, as "DL S067 - Quantization", "The origin story") from the brute-force
    searches and fsum norms, at g = 128, per channel (g = K) and per tensor: both the
    weight and the output error, so a wrong group axis, a per-tensor reshape bug or a
    transposed product fails."""
    rng = np.random.default_rng(41)
    N, K, M = 4, 256, 3
    W = rng.normal(0, 0.02, (N, K))
    X = rng.normal(0, 1, (M, K))
    cols = [17, 200]
    W[:, cols] *= [37.0, 81.0]
    X[:, cols] *= [55.0, 23.0]
    W = W.astype(np.float32).astype(np.float64)
    Y = [[math.fsum(X[m, k] * W[n, k] for k in range(K)) for n in range(N)] for m in range(M)]
    results = {}
    for group in (128, K, 0):
        if group == 0:
            flat = _brute_group_dequant(W.ravel())
            What = np.array(flat).reshape(N, K)
        else:
            What = np.array([sum((_brute_group_dequant(W[n, j:j + group])
                                  for j in range(0, K, group)), []) for n in range(N)])
        Yq = [[math.fsum(X[m, k] * What[n, k] for k in range(K)) for n in range(N)]
              for m in range(M)]
        ref = (_fsum_frobenius_rel(W, What), _fsum_frobenius_rel(Y, Yq))
        got = oracle.outlier_quality(W, X, group)
        assert got[0] == pytest.approx(ref[0], rel=1e-12), group
        assert got[1] == pytest.approx(ref[1], rel=1e-12), group
        results[group] = got
    # the three granularities really differ on this case
    assert results[128][0] < results[K][0] < results[0][0]
    assert len({round(v[1], 9) for v in results.values()}) == 3
