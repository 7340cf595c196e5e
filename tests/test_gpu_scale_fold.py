"""Parity of the per-input-channel scale folding kernels (SmoothQuant / AWQ factors, the
folded quantizer, activation division) with the CPU oracle, through the C ABI.

Bit-exact: column max, column mean (on data whose column sums fit 53 bits), the folded
codes, S' and Z, and X / s. Factor formulas (float64 pow on both sides, rounded to float32):
within one float32 ulp. The folded W4A16 product: within the GEMM gate of the other
matmul tests.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import w4a16_dequant_matmul_b200 as wq  # noqa: E402
import wq_inputs  # noqa: E402
from tests import gpu_util as gu  # noqa: E402

GATE = 1e-2
ULP32 = 2.0 ** -23


def _f32_close(got, want):
    """Within one float32 ulp, relatively (the two sides' float64 pow may differ by an ulp
    of float64, which moves the float32 rounding only near a float32 midpoint)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert np.all(np.abs(got - want) <= ULP32 * np.abs(want)), np.max(np.abs(got - want) / want)
    assert np.mean(got == want) > 0.99


def _salient_acts(M, K, seed, n_salient=None, factor=30.0):
    """Activations with a few large channels (the pattern both methods target)."""
    rng = np.random.default_rng(seed)
    X = rng.normal(0, 1, (M, K))
    n_salient = n_salient or max(1, K // 100)
    ch = rng.choice(K, n_salient, replace=False)
    X[:, ch] *= factor
    return wq_inputs.to_bf16_bits(X)


@pytest.mark.parametrize("rows,cols,pad", [(1, 64, 0), (300, 1032, 8), (2048, 4096, 0)])
def test_channel_stat_bf16_bit_exact(rows, cols, pad):
    Xb = _salient_acts(rows, cols + pad, 3)
    X = gu.bf16_from_bits(Xb)[:, :cols]                      # row stride cols + pad
    Xf = wq_inputs.bf16_bits_to_f64(Xb)[:, :cols]
    mx = wq.wq_channel_stat(X, wq.WQ_STAT_ABSMAX)
    mean = wq.wq_channel_stat(X, wq.WQ_STAT_ABSMEAN)
    assert wq.wq_get_status() == 0
    np.testing.assert_array_equal(gu.to_np(mx).astype(np.float64), oracle.channel_absmax(Xf))
    np.testing.assert_array_equal(gu.to_np(mean).astype(np.float64), oracle.channel_absmean(Xf))


def test_channel_stat_fp32_weights():
    """Weights W [N, K] fp32: the max is exact; the mean within one float32 ulp (float32
    data can need more than 53 bits for an exact column sum)."""
    W = np.random.default_rng(4).normal(0, 0.02, (1500, 512)).astype(np.float32)
    mx = wq.wq_channel_stat(gu.f32(W), wq.WQ_STAT_ABSMAX)
    mean = wq.wq_channel_stat(gu.f32(W), wq.WQ_STAT_ABSMEAN)
    np.testing.assert_array_equal(gu.to_np(mx).astype(np.float64), oracle.channel_absmax(W))
    _f32_close(gu.to_np(mean), oracle.channel_absmean(W))


def test_channel_stat_propagates_nan():
    X = np.random.default_rng(5).normal(0, 1, (64, 128)).astype(np.float32)
    X[17, 9] = np.nan
    mx = gu.to_np(wq.wq_channel_stat(gu.f32(X), wq.WQ_STAT_ABSMAX))
    assert np.isnan(mx[9]) and np.all(np.isfinite(np.delete(mx, 9)))


@pytest.mark.parametrize("alpha", [0.0, 0.5, 0.85, 1.0])
def test_smooth_scales_match_oracle(alpha):
    xm = np.abs(np.random.default_rng(6).normal(0, 10, 1024)).astype(np.float32)
    wm = np.abs(np.random.default_rng(7).normal(0, 0.05, 1024)).astype(np.float32)
    xm[5] = 0.0
    wm[9] = 0.0
    a32 = float(np.float32(alpha))
    s = gu.to_np(wq.wq_smooth_scales(gu.f32(xm), gu.f32(wm), a32))
    want = oracle.smooth_scales(xm, wm, a32).astype(np.float32).astype(np.float64)
    _f32_close(s, want)
    assert s[5] == 1.0 and s[9] == 1.0


@pytest.mark.parametrize("alpha", [0.0, 0.3, 0.5, 1.0])
def test_awq_scales_match_oracle(alpha):
    a = np.abs(np.random.default_rng(8).normal(0, 1, 11008)).astype(np.float32) + 1e-3
    a[::997] *= 40.0
    a[123] = 0.0
    a32 = float(np.float32(alpha))
    s = gu.to_np(wq.wq_awq_scales(gu.f32(a), a32))
    want = oracle.awq_scales(a, a32).astype(np.float32).astype(np.float64)
    _f32_close(s, want)
    assert s[123] == 1.0


def _quant_case(dtype, N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.normal(0, 0.02, (N, K))
    if dtype == "bf16":
        Wb = wq_inputs.to_bf16_bits(W)
        return gu.bf16_from_bits(Wb), wq_inputs.bf16_bits_to_f64(Wb)
    W32 = W.astype(np.float32)
    return gu.f32(W32), W32.astype(np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("group", [32, 64, 128, 256, 1024])
@pytest.mark.parametrize("sym", [False, True])
def test_quantize_rtn_scaled_bit_exact(dtype, group, sym):
    N, K = 67, 1024  # ragged row count
    Wt, W = _quant_case(dtype, N, K, 10 + group)
    rng = np.random.default_rng(20)
    s = np.exp(rng.normal(0, 1.2, K)).astype(np.float32)     # factors over ~3 decades
    s[rng.choice(K, 8, replace=False)] = 40.0                # a few salient channels
    packed, S, Z = wq.wq_quantize_rtn_scaled(Wt, gu.f32(s), group=group, zero_point=not sym)
    assert wq.wq_get_status() == 0
    codes, So, Zo = oracle.quantize_rtn_scaled(W, s.astype(np.float64), group, sym=sym)
    np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))
    np.testing.assert_array_equal(gu.bits16(S), gu.f16_bits_of(So))
    np.testing.assert_array_equal(gu.bits16(Z), gu.f16_bits_of(Zo))


def test_quantize_rtn_scaled_full_size_sampled_rows():
    """4096 x 11008 bf16 weights folded with SmoothQuant factors from synthetic activations
    (the statistics and factors computed by the library): every code, S' and Z of 64 sampled
    rows equals the oracle's on the same factors."""
    N, K = 4096, 11008
    Wb = wq_inputs.weight_bf16(N, K)
    W = gu.bf16_from_bits(Wb)
    X = gu.bf16_from_bits(_salient_acts(64, K, 9))
    xm = wq.wq_channel_stat(X, wq.WQ_STAT_ABSMAX)
    wm = wq.wq_channel_stat(W, wq.WQ_STAT_ABSMAX)
    s = wq.wq_smooth_scales(xm, wm, 0.5)
    packed, S, Z = wq.wq_quantize_rtn_scaled(W, s)
    assert wq.wq_get_status() == 0
    rows = np.sort(np.random.default_rng(1).choice(N, 64, replace=False))
    s64 = gu.to_np(s).astype(np.float64)
    codes, So, Zo = oracle.quantize_rtn_scaled(
        wq_inputs.bf16_bits_to_f64(Wb[rows]), s64, 128)
    np.testing.assert_array_equal(gu.to_np(packed)[rows], oracle.pack_int4(codes))
    np.testing.assert_array_equal(gu.bits16(S)[rows], gu.f16_bits_of(So))
    np.testing.assert_array_equal(gu.bits16(Z)[rows], gu.f16_bits_of(Zo))


def test_quantize_rtn_scaled_reports_bad_factors_and_overflow():
    W = gu.bf16_from_bits(wq_inputs.weight_bf16(8, 256))
    for bad in (0.0, -2.0, np.inf, np.nan):
        s = np.ones(256, np.float32)
        s[77] = bad
        wq.wq_quantize_rtn_scaled(W, gu.f32(s))
        assert wq.wq_get_status() == 9  # WQ_ERR_RANGE
    Wbig = np.full((2, 128), 3e38, np.float32)
    wq.wq_quantize_rtn_scaled(gu.f32(Wbig), gu.f32(np.full(128, 4.0, np.float32)))
    assert wq.wq_get_status() == 7      # WQ_ERR_NONFINITE: the folded weight overflows
    wq.wq_quantize_rtn_scaled(W, gu.f32(np.ones(256, np.float32)))
    assert wq.wq_get_status() == 0      # the status word was cleared


@pytest.mark.parametrize("M,K,pad", [(1, 4096, 0), (33, 1032, 16), (2048, 4096, 0)])
def test_scale_activations_bit_exact(M, K, pad):
    Xb = _salient_acts(M, K + pad, 12)
    X = gu.bf16_from_bits(Xb)[:, :K]
    s = np.exp(np.random.default_rng(13).normal(0, 1, K)).astype(np.float32)
    Xs = wq.wq_scale_activations(X, gu.f32(s))
    want = oracle.scale_activations_bf16(wq_inputs.bf16_bits_to_f64(Xb)[:, :K], s)
    np.testing.assert_array_equal(gu.bits16(Xs), want)
    # in place, row for row
    Xc = X.clone()
    wq.wq_scale_activations(Xc, gu.f32(s), out=Xc)
    np.testing.assert_array_equal(gu.bits16(Xc), want)


@pytest.mark.parametrize("method", ["smoothquant", "awq"])
@pytest.mark.parametrize("M", [1, 16, 256])
def test_folded_w4a16_matmul_matches_oracle(method, M):
    """The whole folded path on the GPU: statistics, factors, folded quantization, X / s,
    then the unchanged W4A16 GEMM; Y within the gate of the oracle's (X/s) W_hat^T on the
    oracle's own codes and activations (computed from the same factors)."""
    N, K = 1536, 2048
    Wb = wq_inputs.weight_bf16(N, K, seed=21)
    W = gu.bf16_from_bits(Wb)
    Xcal = gu.bf16_from_bits(_salient_acts(128, K, 22))
    Xb = _salient_acts(M, K, 23)
    X = gu.bf16_from_bits(Xb)
    if method == "smoothquant":
        s = wq.wq_smooth_scales(wq.wq_channel_stat(Xcal, wq.WQ_STAT_ABSMAX),
                                wq.wq_channel_stat(W, wq.WQ_STAT_ABSMAX), 0.5)
    else:
        s = wq.wq_awq_scales(wq.wq_channel_stat(Xcal, wq.WQ_STAT_ABSMEAN), 0.5)
    packed, S, Z = wq.wq_quantize_rtn_scaled(W, s)
    Xs = wq.wq_scale_activations(X, s)
    Y = wq.wq_w4a16_gemm(Xs, packed, S, Z)
    assert wq.wq_get_status() == 0
    s64 = gu.to_np(s).astype(np.float64)
    codes, So, Zo = oracle.quantize_rtn_scaled(wq_inputs.bf16_bits_to_f64(Wb), s64, 128)
    Xs_o = wq_inputs.bf16_bits_to_f64(
        oracle.scale_activations_bf16(wq_inputs.bf16_bits_to_f64(Xb), s64))
    mode = "bf16" if M > 32 else "exact"
    Yref = oracle.w4a16_matmul(Xs_o, codes, So, Zo, 128, mode=mode)
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE


def test_awq_exponent_search_composes_from_gpu_calls():
    """AWQ's search on the page's calibration toy, in the library's INT4 g128 format, from
    the GPU calls: mean |X_j| (wq_channel_stat), the factors for each exponent
    (wq_awq_scales), the folded codes (wq_quantize_rtn_scaled). Each step matches the oracle
    (factors within a float32 ulp, codes bit for bit on the same factors), and every exponent's
    calibration output error is the oracle's, so the exponent chosen is the oracle's best."""
    W, X_cal, _ = wq_inputs.calibration_toy_tensors()
    W32 = W.astype(np.float32)
    Xb = wq_inputs.to_bf16_bits(X_cal)
    X = wq_inputs.bf16_bits_to_f64(Xb)
    a_gpu = wq.wq_channel_stat(gu.bf16_from_bits(Xb), wq.WQ_STAT_ABSMEAN)
    np.testing.assert_array_equal(gu.to_np(a_gpu).astype(np.float64), oracle.channel_absmean(X))
    Y = oracle.matmul_f64(X, W32.astype(np.float64))
    errs = []
    for a in np.linspace(0, 1, 11):
        a32 = float(np.float32(a))
        s = wq.wq_awq_scales(a_gpu, a32)
        s64 = gu.to_np(s).astype(np.float64)
        _f32_close(s64, oracle.awq_scales(oracle.channel_absmean(X), a32)
                   .astype(np.float32).astype(np.float64))
        packed, S, Z = wq.wq_quantize_rtn_scaled(gu.f32(W32), s)
        assert wq.wq_get_status() == 0
        codes, So, Zo = oracle.quantize_rtn_scaled(W32.astype(np.float64), s64, 128)
        np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))
        Q = oracle.dequant_asym(codes, So, Zo, 128) / s64          # fold 1/s back
        errs.append(oracle.rel_frobenius(Y, oracle.matmul_f64(X, Q)))
    # the oracle's own search (float64 factors) scores every exponent alike, within 1e-3
    # relative: the two agree on the best exponent up to near ties
    qdq = lambda Ws: oracle.dequant_asym(*oracle.quantize_rtn_asym(
        Ws.astype(np.float32).astype(np.float64), 128), 128)
    errs_or = []
    for a in np.linspace(0, 1, 11):
        Qo, _, _ = oracle.awq_search(W32.astype(np.float64), X, [a], qdq)
        errs_or.append(oracle.rel_frobenius(Y, oracle.matmul_f64(X, Qo)))
    np.testing.assert_allclose(errs, errs_or, rtol=1e-3)
    best = int(np.argmin(errs))
    assert errs_or[best] <= min(errs_or) * (1 + 1e-3)
    assert errs[best] < 0.95 * errs[0]  # scaling helps against round-to-nearest (exponent 0)
