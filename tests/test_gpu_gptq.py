"""Parity of the GPU GPTQ quantizer (float64 Hessian, Gauss-Jordan inverse, downdates and
column sweep) with the oracle's sweep on the same inputs, through the C ABI: codes, S' and Z
equal, on the page's calibration toy and on larger correlated activations; the diagonal
Hessian reduces to round-to-nearest; a singular Hessian without damping is reported."""
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


def _correlated(T, K, seed, salient=4):
    rng = np.random.default_rng(seed)
    mix = rng.normal(0, 1, (K, K)) / np.sqrt(K)
    chan = np.ones(K)
    chan[rng.choice(K, salient, replace=False)] = 8.0
    return (rng.normal(0, 1, (T, K)) @ mix + 0.3 * rng.normal(0, 1, (T, K))) * chan


def _compare(W32, Xb, group, sym=False, damp=0.01):
    packed, S, Z = wq.wq_quantize_gptq(gu.f32(W32), gu.bf16_from_bits(Xb), group,
                                       zero_point=not sym, damp=damp)
    assert wq.wq_get_status() == 0
    codes, So, Zo = oracle.gptq_quantize_asym(W32.astype(np.float64),
                                              wq_inputs.bf16_bits_to_f64(Xb), group, damp, sym)
    np.testing.assert_array_equal(gu.bits16(S), gu.f16_bits_of(So))
    np.testing.assert_array_equal(gu.bits16(Z), gu.f16_bits_of(Zo))
    got = oracle.unpack_int4(gu.to_np(packed))
    return got, codes, So, Zo


def test_gptq_calibration_toy_matches_oracle():
    """The page's toy layer (64 x 128) and calibration set, in the library's INT4 g128."""
    W, X_cal, _ = wq_inputs.calibration_toy_tensors()
    W32 = W.astype(np.float32)
    got, codes, _, _ = _compare(W32, wq_inputs.to_bf16_bits(X_cal), 128)
    np.testing.assert_array_equal(got, codes)


@pytest.mark.parametrize("group,sym", [(128, False), (64, False), (128, True)])
def test_gptq_larger_matches_oracle(group, sym):
    N, K, T = 192, 512, 300
    W32 = np.random.default_rng(3).normal(0, 0.02, (N, K)).astype(np.float32)
    Xb = wq_inputs.to_bf16_bits(_correlated(T, K, 4))
    got, codes, So, Zo = _compare(W32, Xb, group, sym)
    np.testing.assert_array_equal(got, codes)
    # and it does what it is for: lower calibration output error than round-to-nearest
    X = wq_inputs.bf16_bits_to_f64(Xb)
    Y = oracle.matmul_f64(X, W32.astype(np.float64))
    c0, S0, Z0 = (oracle.sym_int4_storage(*oracle.quantize_rtn_sym_int4(W32, group)) if sym
                  else oracle.quantize_rtn_asym(W32, group))
    e_rtn = oracle.rel_frobenius(Y, oracle.w4a16_matmul(X, c0, S0, Z0, group))
    e_gptq = oracle.rel_frobenius(Y, oracle.w4a16_matmul(X, got, So, Zo, group))
    assert e_gptq < 0.9 * e_rtn


def test_gptq_diagonal_hessian_is_rtn():
    """Uncorrelated channels: nothing moves, the codes are round-to-nearest's, bf16 W."""
    N, K = 64, 256
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=6)
    X = np.diag(np.random.default_rng(7).uniform(0.5, 3.0, K))
    Xb = wq_inputs.to_bf16_bits(X)
    packed, S, Z = wq.wq_quantize_gptq(gu.bf16_from_bits(Wb), gu.bf16_from_bits(Xb), 128)
    assert wq.wq_get_status() == 0
    p0, S0, Z0 = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    assert torch.equal(packed, p0) and torch.equal(S.view(torch.int16), S0.view(torch.int16))


def test_gptq_singular_hessian_is_reported():
    """A calibration channel that is always zero and no damping: H is singular, the pivot of
    that channel is zero, and the call reports WQ_ERR_NONFINITE (7)."""
    N, K, T = 16, 128, 256
    W32 = np.random.default_rng(8).normal(0, 0.02, (N, K)).astype(np.float32)
    X = _correlated(T, K, 9)
    X[:, 5] = 0.0
    wq.wq_quantize_gptq(gu.f32(W32), gu.bf16_from_bits(wq_inputs.to_bf16_bits(X)), 128,
                        damp=0.0)
    assert wq.wq_get_status() == 7
    wq.wq_quantize_rtn_g128(gu.f32(W32))
    assert wq.wq_get_status() == 0
