"""Plain, slow CPU oracle for round-to-nearest group-wise affine quantization and the
W4A16 matmul, in float64 / exact rationals.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py``; never by the CUDA library, with which it shares no
code. Inputs come from ``wq_inputs`` (random draws and dtype casts only).

Sources (page title, section):
  [AQ]  "Model Quantization", section 1 "Mathematical Mechanics of Quantization":
        affine quantize/dequantize with a scale S and zero-point Z; group-wise S, Z over
        blocks of g = 128 weights.
  [CM]  "DL S067 - Quantization", section 1 "The core math": asymmetric
        scale = (beta - alpha)/(q_max - q_min), z = round(q_min - alpha/scale),
        q = clip(round(x/scale) + z, q_min, q_max), x_hat = scale*(q - z); symmetric
        scale = max|x|/q_max; the INT8 worked example.
  [GR]  same page, section 2 "Per-tensor vs per-channel vs per-group": groups are g
        consecutive weights along the input dimension of a (out, in) weight; 4 + 16/128
        bits per weight; symmetric clip range [-q_max-1, q_max].
  [VO]  "LLM Weight Quantization - GPTQ, AWQ, SmoothQuant, FP8 & INT4/INT8 Trade-offs",
        section "The vocabulary": W4A16 dequantizes 4-bit weights to 16 bits inside the
        kernel and runs a 16-bit matmul, Y = X W^T; section "Granularity and outliers":
        the symmetric quantize-dequantize demo and its relative Frobenius errors.
  [SQ]  same page, "Granularity and outliers": SmoothQuant's per-input-channel factor
        s_j = max|X_j|^alpha / max|W_j|^(1 - alpha) (alpha = 0.5), with X/s and W*s
        giving the same product X W^T.
  [AW]  same page, "GPTQ vs AWQ: two ways to choose what error to keep": AWQ scales the
        weight columns of large-activation channels up by s (activations down by s)
        before rounding; s = mean|X_j|^a normalised so that sqrt(max s * min s) = 1, the
        exponent a chosen on calibration data by the output error. Also "DL S067 -
        Quantization", section 5 "AWQ intuition" (y = (W diag(s)) (diag(1/s) x), 1/s
        pushed into the previous layer), and "Model Quantization", section 2.2.
  [GQ]  same page, "GPTQ vs AWQ": GPTQ quantizes one input column at a time and moves each
        column's rounding error onto the columns not yet quantized through the inverse of
        the dampened layer-input Hessian H = X^T X + damp * mean(diag) * I, dropping the
        finished column from the inverse after each step (the Optimal Brain Surgeon
        update); the quantization grid is fixed before the sweep. Also "DL S067 -
        Quantization", section 4, and "Model Quantization", section 2.1.

Readings where the pages are silent (each is pinned by a test in tests/test_oracle.py):
  * range includes zero: alpha = min(0, min w), beta = max(0, max w);
  * S is the exact (beta - alpha)/15 rounded once to binary16 (round half to even); all
    later steps use that stored S'; S' = 0 (range below half the smallest binary16
    subnormal, e.g. an all-zero group) is replaced by 1.0; S' overflow or a non-finite
    weight is an error;
  * Z = RNE(-alpha/S') on the exact quotient, clipped to [0, 15] (the clip only acts when
    S' is a binary16 subnormal far below S), stored as binary16;
  * codes use the exact quotient w/S', rounded half to even;
  * packed layout: row-major [N, K/2], byte j = q[2j] | q[2j+1] << 4;
  * symmetric INT4 per group [GR]: s = max|w|/7 rounded once to binary16 (0 -> 1.0),
    q = clip(RNE(w/s'), -8, 7) on the exact quotient, stored as q + 8 with Z = 8;
  * a matmul "on the same dequantized weights" uses either the exact S'(q - Z)
    ("exact" mode) or its bfloat16 rounding ("bf16" mode);
  * scale folding [SQ][AW]: the folded weight W*s is rounded once to float32 (the
    precision in which a kernel forms it) before the RTN steps above; the folded
    activation X/s is the float32 quotient rounded to bfloat16 (the activations' storage
    type); every s_j must be finite and > 0;
  * a channel whose statistic is zero (max|X_j| or max|W_j| for SmoothQuant, mean|X_j|
    for AWQ) gets s_j = 1 and is left out of AWQ's normalisation (the pages' formulas
    give 0/0 or 0 there);
  * GPTQ [GQ]: the grid of each group (S', Z, or the per-row symmetric scale of the
    page's toy) is computed from the original weights before the sweep, as the toy fixes
    its per-row scale up front; columns are taken in their natural order;
  * the per-channel mean |X_j| is the column's exact sum (math.fsum, exact whenever the
    sum fits binary64's 53 bits) divided by the row count and rounded once to float32.

Parity status: every function below is pinned by tests/test_oracle.py. The pages print
no values for the outlier-stress construction, so ``outlier_quality`` is pinned by
recomputing it from brute-force scale and level searches with exactly rounded norms on a
small outlier case (all three granularities, weight and output errors), and the ordering
g128 < per-channel < per-tensor is asserted as the pages state it.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

__all__ = [
    "Q4_MIN", "Q4_MAX", "Q8_MAX", "NonFiniteError",
    "fp16_round", "bf16_round_bits", "bf16_bits_to_f64",
    "group_range", "asym_scale_zero", "quantize_rtn_asym", "pack_int4", "unpack_int4",
    "dequant_asym", "sym_scale", "quantize_sym_int8_per_channel", "dequant_sym_per_channel",
    "Q4S_MIN", "Q4S_MAX", "quantize_rtn_sym_int4", "sym_int4_storage",
    "matmul_f64", "w4a16_matmul", "w8a16_matmul", "qdq_sym", "rel_frobenius",
    "gemm_gate", "bits_per_weight", "decode_ceiling_tok_s", "error_bound_ok",
    "outlier_quality", "f32_round", "channel_absmax", "channel_absmean", "smooth_scales",
    "smoothquant_scales", "awq_scales", "fold_input_scales", "fold_weight_f32",
    "quantize_rtn_scaled", "scale_activations_bf16", "awq_search",
    "gptq_hessian", "gptq_sweep", "gptq_quantize_asym",
]

Q4_MIN, Q4_MAX = 0, 15       # asymmetric INT4 integer range [CM]
Q8_MAX = 127                  # symmetric INT8 integer range [CM]
Q4S_MIN, Q4S_MAX = -8, 7      # symmetric INT4 range [-q_max - 1, q_max] [GR]
FP16_MAX = 65504.0


class NonFiniteError(ValueError):
    """A weight is NaN/inf, or the scale overflows binary16."""


# --------------------------------------------------------------------------- roundings

def fp16_round(r) -> float:
    """Round an exact rational (or float) to the nearest binary16 value, ties to even.

    Returns the value as a Python float (exact), +-inf on overflow."""
    r = Fraction(r)
    if r == 0:
        return 0.0
    sign = -1.0 if r < 0 else 1.0
    a = abs(r)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if a < Fraction(2) ** e:
        e -= 1                      # now 2**e <= a < 2**(e+1)
    e = max(e, -14)                 # below 2**-14 the spacing stays 2**-24 (subnormals)
    ulp = Fraction(2) ** (e - 10)   # 10 fraction bits
    n = round(a / ulp)              # Python rounds a Fraction half to even
    v = n * ulp
    if v > FP16_MAX:
        return sign * math.inf
    return sign * float(v)


def f32_round(r) -> float:
    """Round an exact rational (or float) to the nearest binary32 value, ties to even
    (subnormals included); +-inf on overflow. Returned as an exact Python float."""
    r = Fraction(r)
    if r == 0:
        return 0.0
    sign = -1.0 if r < 0 else 1.0
    a = abs(r)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if a < Fraction(2) ** e:
        e -= 1                      # 2**e <= a < 2**(e+1)
    e = max(e, -126)                # subnormal spacing 2**-149
    ulp = Fraction(2) ** (e - 23)   # 23 fraction bits
    v = round(a / ulp) * ulp
    if v > Fraction(float(np.finfo(np.float32).max)):
        return sign * math.inf
    return sign * float(v)


def bf16_round_bits(x) -> np.ndarray:
    """bfloat16 bit patterns of values that are exactly representable in float32,
    rounded to nearest, ties to even (finite inputs only)."""
    u = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f64(bits) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ------------------------------------------------------------- asymmetric INT4 RTN [CM]

def group_range(w) -> tuple[float, float]:
    """alpha = min(0, min w), beta = max(0, max w) over one group."""
    w = np.asarray(w, dtype=np.float64)
    return min(0.0, float(w.min())), max(0.0, float(w.max()))


def asym_scale_zero(alpha: float, beta: float, qmin: int = Q4_MIN, qmax: int = Q4_MAX):
    """Stored scale S' = fp16(RNE((beta - alpha)/(qmax - qmin))) and zero-point
    Z = clip(RNE(qmin - alpha/S'), qmin, qmax), both exact."""
    if not (math.isfinite(alpha) and math.isfinite(beta)):
        raise NonFiniteError("non-finite weight")
    s = fp16_round((Fraction(beta) - Fraction(alpha)) / (qmax - qmin))
    if math.isinf(s):
        raise NonFiniteError("scale overflows binary16")
    if s == 0.0:
        s = 1.0
    z = round(Fraction(qmin) - Fraction(alpha) / Fraction(s))   # half to even
    z = min(max(z, qmin), qmax)
    return s, float(z)


def _groups(W, group):
    """View W [N, K] as [N, G, g]: g consecutive weights along the input dim [GR].
    group = K gives one group per output row; group in (0, None) gives one group for
    the whole tensor (returned as [1, 1, N*K])."""
    N, K = W.shape
    if not group:
        return W.reshape(1, 1, N * K)
    if K % group:
        raise ValueError(f"K={K} is not a multiple of the group size {group}")
    return W.reshape(N, K // group, group)


def quantize_rtn_asym(W, group=128, qmin: int = Q4_MIN, qmax: int = Q4_MAX):
    """Round-to-nearest asymmetric quantization [CM], group-wise [AQ][GR].

    W: float array [N, K] whose values are exactly representable in float32.
    Returns (codes uint8 [N, K], S float64 [N, G], Z float64 [N, G]); S and Z hold
    binary16 values. Per-tensor (group 0/None) returns S, Z of shape [1, 1]."""
    W = np.asarray(W, dtype=np.float64)
    if not np.all(np.isfinite(W)):
        raise NonFiniteError("non-finite weight")
    Wg = _groups(W, group)
    R, G, _ = Wg.shape
    S = np.empty((R, G))
    Z = np.empty((R, G))
    for r in range(R):
        for g in range(G):
            S[r, g], Z[r, g] = asym_scale_zero(*group_range(Wg[r, g]), qmin, qmax)
    # float64 division of a float32 weight by a binary16 scale is exact enough that
    # rint() of it equals the round-half-even of the exact quotient (|w/S'| < 64).
    q = np.rint(Wg / S[:, :, None]) + Z[:, :, None]
    codes = np.clip(q, qmin, qmax).astype(np.uint8).reshape(W.shape)
    return codes, S, Z


def pack_int4(codes) -> np.ndarray:
    """Two 4-bit codes per byte, row-major: byte j of a row = q[2j] | q[2j+1] << 4."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.shape[-1] % 2:
        raise ValueError("K must be even to pack two codes per byte")
    if np.any(c > 15):
        raise ValueError("codes must lie in [0, 15]")
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def dequant_asym(codes, S, Z, group=128) -> np.ndarray:
    """W_hat = S' * (q - Z) in float64 (exact: an 11-bit scale times a 5-bit integer)."""
    c = np.asarray(codes, dtype=np.float64)
    cg = _groups(c, group)
    return (np.asarray(S)[:, :, None] * (cg - np.asarray(Z)[:, :, None])).reshape(c.shape)


def error_bound_ok(W, What, S, group=128, qmax_minus_qmin: int = 15) -> bool:
    """Per element |w - w_hat| <= S'/2 + (qmax - qmin)*max(0, S - S'), with S the exact
    unrounded scale: the "half a step" bound of round-to-nearest, widened by what the
    binary16 rounding of S can lose at the clipped ends. Checked in exact rationals."""
    W = np.asarray(W, dtype=np.float64)
    Wg = _groups(W, group)
    Hg = _groups(np.asarray(What, dtype=np.float64), group)
    R, G, _ = Wg.shape
    for r in range(R):
        for g in range(G):
            a, b = group_range(Wg[r, g])
            s_exact = (Fraction(b) - Fraction(a)) / qmax_minus_qmin
            s16 = Fraction(float(S[r, g]))
            bound = s16 / 2 + qmax_minus_qmin * max(Fraction(0), s_exact - s16)
            if s_exact == 0:
                bound = Fraction(0)
            err = max(abs(Fraction(float(x)) - Fraction(float(y)))
                      for x, y in zip(Wg[r, g], Hg[r, g]))
            if err > bound:
                return False
    return True


# ----------------------------------------------------- symmetric INT8 per channel [CM]

def sym_scale(amax: float, qmax: int = Q8_MAX) -> float:
    """Stored symmetric scale fp16(RNE(max|w| / qmax)); 0 -> 1.0."""
    if not math.isfinite(amax):
        raise NonFiniteError("non-finite weight")
    s = fp16_round(Fraction(amax) / qmax)
    if math.isinf(s):
        raise NonFiniteError("scale overflows binary16")
    return 1.0 if s == 0.0 else s


def quantize_sym_int8_per_channel(W):
    """Symmetric INT8 with one scale per output row: s = max|w|/127 stored as binary16,
    q = clip(RNE(w/s'), -127, 127). Returns (codes int8 [N, K], s float64 [N])."""
    W = np.asarray(W, dtype=np.float64)
    if not np.all(np.isfinite(W)):
        raise NonFiniteError("non-finite weight")
    s = np.array([sym_scale(float(np.abs(row).max())) for row in W])
    q = np.clip(np.rint(W / s[:, None]), -Q8_MAX, Q8_MAX).astype(np.int8)
    return q, s


def dequant_sym_per_channel(codes, s) -> np.ndarray:
    return np.asarray(codes, dtype=np.float64) * np.asarray(s, dtype=np.float64)[:, None]


# ------------------------------------------------------ symmetric INT4 per group [GR]

def quantize_rtn_sym_int4(W, group=128):
    """Symmetric INT4 per group of g consecutive input weights [GR] ("quantize_per_group"):
    s = max|w| / 7 over the group, stored as binary16 (RNE of the exact value; 0 -> 1.0),
    q = clip(RNE(w/s'), -8, 7) on the exact quotient.

    W: float array [N, K] of float32-representable values. Returns (q int8 [N, K],
    S float64 [N, G] holding binary16 values)."""
    W = np.asarray(W, dtype=np.float64)
    if not np.all(np.isfinite(W)):
        raise NonFiniteError("non-finite weight")
    if not group:
        raise ValueError("symmetric INT4 is defined per group here")
    Wg = _groups(W, group)
    R, G, _ = Wg.shape
    S = np.empty((R, G))
    for r in range(R):
        for g in range(G):
            S[r, g] = sym_scale(float(np.abs(Wg[r, g]).max()), Q4S_MAX)
    # as in quantize_rtn_asym: rint of the float64 quotient is the RNE of the exact one
    q = np.clip(np.rint(Wg / S[:, :, None]), Q4S_MIN, Q4S_MAX).astype(np.int8)
    return q.reshape(W.shape), S


def sym_int4_storage(q, S):
    """The symmetric codes in the asymmetric INT4 storage (stored code q + 8, Z = 8), in
    which S'(code - Z) = S' q: the format the library stores for zero_point = 0."""
    codes = (np.asarray(q, dtype=np.int16) - Q4S_MIN).astype(np.uint8)
    return codes, np.asarray(S, dtype=np.float64), np.full(np.shape(S), float(-Q4S_MIN))


# -------------------------------------------------------------------- matmul [VO]

def matmul_f64(X, W_hat) -> np.ndarray:
    """Y = X W_hat^T in float64. X [M, K], W_hat [N, K] -> Y [M, N]."""
    X = np.asarray(X, dtype=np.float64)
    W_hat = np.asarray(W_hat, dtype=np.float64)
    if X.shape[1] != W_hat.shape[1]:
        raise ValueError("inner dimensions differ")
    return X @ W_hat.T


def w4a16_matmul(X, codes, S, Z, group=128, mode="exact") -> np.ndarray:
    """W4A16 matmul on the same dequantized weights as a kernel: mode "exact" uses
    S'(q - Z) as is, mode "bf16" rounds it to bfloat16 first (a kernel that feeds
    16-bit tensor cores)."""
    W_hat = dequant_asym(codes, S, Z, group)
    if mode == "bf16":
        W_hat = bf16_bits_to_f64(bf16_round_bits(W_hat))
    elif mode != "exact":
        raise ValueError(mode)
    return matmul_f64(X, W_hat)


def w8a16_matmul(X, codes, s, mode="exact") -> np.ndarray:
    W_hat = dequant_sym_per_channel(codes, s)
    if mode == "bf16":
        W_hat = bf16_bits_to_f64(bf16_round_bits(W_hat))
    elif mode != "exact":
        raise ValueError(mode)
    return matmul_f64(X, W_hat)


def gemm_gate(y, y_ref, K=None) -> float:
    """max_i |y_i - y_ref_i| / max(|y_ref_i|, floor): relative error with a floor, so that
    outputs that cross zero do not make the ratio unbounded.

    floor = 1e-3 * rms(y_ref), or, given the contraction length K, at least 100 times the
    worst-case error of fp32 accumulation in K/16 steps (a tensor core adds one 16-term dot
    product to its fp32 accumulator per step, losing up to one fp32 ulp, 2^-23 relative, of
    partial sums of about rms(y_ref) size): floor = max(1e-3, 100 (K/16) 2^-23) rms(y_ref).
    With the tolerance 1e-2, an output below the floor is then held to that absolute
    accumulation error rather than to 1 % of itself."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    rel = 1e-3 if K is None else max(1e-3, 100.0 * (K / 16.0) * 2.0 ** -23)
    floor = rel * math.sqrt(float(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    den = np.maximum(np.abs(y_ref), floor)
    if y.size == 0:
        return 0.0
    return float(np.max(np.abs(y - y_ref) / den))


# ------------------------------------------------- symmetric quantize-dequantize [VO][GR]

def qdq_sym(x, bits, axis=None, group=None) -> np.ndarray:
    """Symmetric round-to-nearest quantize then dequantize in float64 with a
    full-precision scale max|x|/qmax taken over the whole tensor (axis None), along
    ``axis`` (keepdims), or per group of ``group`` consecutive entries of each row;
    codes clipped to [-qmax-1, qmax]."""
    x = np.asarray(x, dtype=np.float64)
    qmax = 2 ** (bits - 1) - 1
    if group:
        rows = x.shape[0]
        xg = x.reshape(rows, -1, group)
        s = np.abs(xg).max(axis=-1, keepdims=True) / qmax
        return (np.clip(np.rint(xg / s), -qmax - 1, qmax) * s).reshape(x.shape)
    if axis is None:
        s = np.abs(x).max() / qmax
    else:
        s = np.abs(x).max(axis=axis, keepdims=True) / qmax
    return np.clip(np.rint(x / s), -qmax - 1, qmax) * s


def rel_frobenius(a, b) -> float:
    """||a - b||_F / ||a||_F."""
    a = np.asarray(a, dtype=np.float64)
    return float(np.linalg.norm(a - np.asarray(b, dtype=np.float64)) / np.linalg.norm(a))


# --------------------------------------------------------------- storage model [GR][VO]

def bits_per_weight(bits=4, group=128, scale_bits=16, zero_bits=0) -> float:
    """Storage bits per weight: the code plus one scale (and zero-point) per group."""
    return bits + (scale_bits + zero_bits) / group


def decode_ceiling_tok_s(params, bits_per_w, bandwidth_bytes_s, gpus=1) -> float:
    """Batch-1 decode ceiling when every token streams every weight once."""
    return bandwidth_bytes_s * gpus / (params * bits_per_w / 8)


# --------------------------------------------------------------- outlier stress quality

def outlier_quality(W, X, group):
    """Relative Frobenius weight and output errors of asymmetric INT4 RTN at one
    granularity (group = 128, K, or 0 for per-tensor): ||W - W_hat|| / ||W|| and
    ||X W^T - X W_hat^T|| / ||X W^T|| ("LLM Weight Quantization ...", "Granularity and
    outliers", the error measure of its demo)."""
    codes, S, Z = quantize_rtn_asym(W, group)
    W_hat = dequant_asym(codes, S, Z, group)
    W64 = np.asarray(W, dtype=np.float64)
    return rel_frobenius(W64, W_hat), rel_frobenius(matmul_f64(X, W64), matmul_f64(X, W_hat))


# ------------------------------------------------ per-input-channel scale folding [SQ][AW]

def channel_absmax(A) -> np.ndarray:
    """max_i |A_ij| for every column j of A [rows, cols] (exact)."""
    return np.abs(np.asarray(A, dtype=np.float64)).max(axis=0)


def channel_absmean(A) -> np.ndarray:
    """mean_i |A_ij| per column j, rounded once to float32 (returned as float64):
    the column sum by math.fsum (correctly rounded, so exact when it fits 53 bits),
    then the exact quotient by the row count rounded to float32."""
    A = np.abs(np.asarray(A, dtype=np.float64))
    rows = A.shape[0]
    return np.array([f32_round(Fraction(math.fsum(A[:, j])) / rows)
                     for j in range(A.shape[1])])


def smooth_scales(xmax, wmax, alpha=0.5) -> np.ndarray:
    """SmoothQuant migration factors [SQ] from per-channel statistics:
    s_j = xmax_j^alpha / wmax_j^(1 - alpha); s_j = 1 where either statistic is zero."""
    xmax = np.asarray(xmax, dtype=np.float64)
    wmax = np.asarray(wmax, dtype=np.float64)
    s = np.ones_like(xmax)
    live = (xmax > 0) & (wmax > 0)
    s[live] = xmax[live] ** alpha / wmax[live] ** (1.0 - alpha)
    return s


def smoothquant_scales(X, W, alpha=0.5) -> np.ndarray:
    """s for activations X [tokens, K] and weights W [out, K]: the column maxima of |X|
    (over tokens) and of |W| (over output rows) fed to ``smooth_scales`` [SQ]."""
    return smooth_scales(channel_absmax(X), channel_absmax(W), alpha)


def awq_scales(a_mag, alpha) -> np.ndarray:
    """AWQ factors [AW]: s_j = a_j^alpha divided by sqrt(max_j s_j * min_j s_j), so that
    the factors are centred on 1 in log scale; a channel with a_j = 0 gets s_j = 1 and is
    left out of the max and min."""
    a = np.asarray(a_mag, dtype=np.float64)
    s = np.ones_like(a)
    live = a > 0
    if np.any(live):
        p = a[live] ** alpha
        s[live] = p / math.sqrt(float(p.max()) * float(p.min()))
    return s


def _check_factors(s):
    s = np.asarray(s, dtype=np.float64)
    if not np.all(np.isfinite(s)) or np.any(s <= 0):
        raise ValueError("scale factors must be finite and positive")
    return s


def fold_input_scales(X, W, s):
    """(X / s, W * s) in float64 [SQ][AW]: activations divided and weight columns
    multiplied by the same per-input-channel factor, so (X/s)(W s)^T = X W^T."""
    s = _check_factors(s)
    return np.asarray(X, dtype=np.float64) / s, np.asarray(W, dtype=np.float64) * s


def fold_weight_f32(W, s) -> np.ndarray:
    """W * s per input channel, rounded once to float32 (returned as float64). W and s
    hold float32 values, whose product (at most 48 significant bits) float64 holds
    exactly, so the cast below is the only rounding."""
    s = _check_factors(s)
    P = np.asarray(W, dtype=np.float64) * s
    with np.errstate(over="ignore"):
        P32 = P.astype(np.float32)
    if not np.all(np.isfinite(P32)):
        raise NonFiniteError("folded weight is not finite in float32")
    return P32.astype(np.float64)


def quantize_rtn_scaled(W, s, group=128, sym=False):
    """RTN INT4 of the folded weight W * s (``fold_weight_f32``) [AW]: asymmetric (codes,
    S, Z) as ``quantize_rtn_asym``, or symmetric in the stored form of
    ``sym_int4_storage``."""
    Wf = fold_weight_f32(W, s)
    if sym:
        return sym_int4_storage(*quantize_rtn_sym_int4(Wf, group))
    return quantize_rtn_asym(Wf, group)


def scale_activations_bf16(X, s) -> np.ndarray:
    """bfloat16 bits of X / s [SQ][AW]: the float32 quotient (float64 division of two
    float32 values rounded to float32 equals the correctly rounded float32 quotient,
    since 53 >= 2*24 + 2), then rounded to bfloat16, ties to even."""
    s = _check_factors(s)
    q = (np.asarray(X, dtype=np.float64) / s).astype(np.float32)
    return bf16_round_bits(q)


def awq_search(W, X, alphas, qdq):
    """AWQ's exponent search [AW]: a_j = mean_i |X_ij| on the calibration set X; for each
    candidate exponent a (in the given order) fold s = ``awq_scales``(a_mag, a) into the
    weight columns, quantize-dequantize with ``qdq``, fold 1/s back, and score
    ||X W^T - X Q^T||_F. Returns (Q, a, s) of the first candidate with the smallest
    score."""
    W = np.asarray(W, dtype=np.float64)
    X = np.asarray(X, dtype=np.float64)
    a_mag = np.abs(X).mean(axis=0)
    Y = X @ W.T
    best = None
    for a in alphas:
        s = awq_scales(a_mag, a)
        Q = qdq(W * s) / s
        err = np.linalg.norm(Y - X @ Q.T)
        if best is None or err < best[0]:
            best = (err, a, Q, s)
    return best[2], best[1], best[3]


# -------------------------------------------------------------------------- GPTQ [GQ]

def gptq_hessian(X, damp=0.01) -> np.ndarray:
    """H = X^T X of the calibration activations X [tokens, K], plus damp times the mean of
    its diagonal on the diagonal (numerical stability) [GQ]."""
    X = np.asarray(X, dtype=np.float64)
    H = X.T @ X
    return H + damp * float(np.mean(np.diag(H))) * np.eye(H.shape[0])


def gptq_sweep(W, H, qdq_column):
    """GPTQ's column sweep [GQ]. W [N, K]; H [K, K] dampened; qdq_column(i, w) returns the
    quantize-dequantized values of column i for the current values w [N] of that column on
    a grid fixed before the sweep. Every row sees the same sequence of inverse Hessians, so
    the rows are swept together: for column i, Q_i = qdq(w_i), the error e = (w_i - Q_i) /
    Hinv_ii moves onto the later columns as w_j -= e Hinv_ij (j > i), and column i leaves
    the inverse: Hinv -= Hinv_{:,i} Hinv_{i,:} / Hinv_ii. Returns Q [N, K] (float64)."""
    Wc = np.array(W, dtype=np.float64, copy=True)
    Hinv = np.linalg.inv(np.asarray(H, dtype=np.float64))
    N, K = Wc.shape
    Q = np.zeros_like(Wc)
    for i in range(K):
        Q[:, i] = qdq_column(i, Wc[:, i])
        err = (Wc[:, i] - Q[:, i]) / Hinv[i, i]
        Wc[:, i + 1:] -= np.outer(err, Hinv[i, i + 1:])
        Hinv -= np.outer(Hinv[:, i], Hinv[i, :]) / Hinv[i, i]
    return Q


def gptq_quantize_asym(W, X, group=128, damp=0.01, sym=False):
    """GPTQ into the library's INT4 format [GQ][CM]: S' and Z of every group from the
    original weights (``quantize_rtn_asym``, or with ``sym`` the symmetric grid in its stored
    form, Z = 8), then the sweep with codes clip(RNE(w/S') + Z, 0, 15) of the updated
    weights. Returns (codes uint8 [N, K], S, Z) for the unchanged W4A16 kernels."""
    W = np.asarray(W, dtype=np.float64)
    if sym:
        _, S, Z = sym_int4_storage(*quantize_rtn_sym_int4(W, group))
    else:
        _, S, Z = quantize_rtn_asym(W, group)
    g = group or W.shape[1]
    codes = np.zeros(W.shape, dtype=np.uint8)

    def qdq(i, w):
        s, z = S[:, i // g], Z[:, i // g]
        q = np.clip(np.rint(w / s) + z, Q4_MIN, Q4_MAX)
        codes[:, i] = q.astype(np.uint8)
        return s * (q - z)

    gptq_sweep(W, gptq_hessian(X, damp), qdq)
    return codes, S, Z
