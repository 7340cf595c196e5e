"""Parity of the skinny tensor-core kernel (split-K over a cluster) with the float64 oracle,
through the C ABI: W4A16 (9 to 64 tokens, g = 128; kind::f16 on the centred codes q - Z as
bf16 and the activations as stored) on the exact dequantized weights S'(q - Z), and W8A16
(3 to 64 tokens; kind::i8 on the s8 codes copied as they are and exact activation digits)
on the exact s' q. The W8A16 cases also cover one
token, which runs on the row kernel, against the same exact product.

Cases span one group (K = 128, no split), ragged row counts (a partial 128-row tile), every
token-count class (16, 32, 64 token columns) with ragged M, long K (70B-class), and
outlier activations (a token's group scale set by one large channel)."""
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


def _case(M, N, K, seed, x_outliers=False):
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=seed)
    X = wq_inputs.normal_f64((M, K), 1.0, seed + 1)
    if x_outliers:
        cols = np.random.default_rng(seed + 2).choice(K, max(1, K // 1000), replace=False)
        X[:, cols] *= 80.0
    Xb = wq_inputs.to_bf16_bits(X)
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb), 128)
    packed = gu.u8(oracle.pack_int4(codes))
    S = gu.f16_from_values(So.ravel()).reshape(So.shape)
    Z = gu.f16_from_values(Zo.ravel()).reshape(Zo.shape)
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    return gu.bf16_to_f64(Y), Yref


@pytest.mark.parametrize("M", [9, 12, 16, 17, 31, 32, 33, 48, 64])
@pytest.mark.parametrize("N,K", [(300, 512), (128, 128), (1024, 2048)])
def test_skinny_parity(M, N, K):
    y, yref = _case(M, N, K, seed=M + N)
    assert oracle.gemm_gate(y, yref, K) <= GATE
    assert oracle.rel_frobenius(yref, y) < 4e-3


@pytest.mark.parametrize("M", [12, 32])
def test_skinny_outlier_activations(M):
    """A channel 80x larger sets its token's group scale: the other 127 values of the group
    keep 14 bits below it exactly, which the fp32 products would keep too."""
    y, yref = _case(M, 512, 4096, seed=40 + M, x_outliers=True)
    assert oracle.gemm_gate(y, yref, 4096) <= GATE


def test_skinny_long_k_sampled():
    """70B-class K = 28672 at M = 16 (a long split-K range per cluster): sampled rows."""
    M, N, K = 16, 1024, 28672
    Wb = wq_inputs.weight_bf16(N, K, 0.015, seed=3)
    Xb = wq_inputs.act_bf16(M, K, seed=4)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    rows = np.sort(np.random.default_rng(5).choice(N, 40, replace=False))
    rows[0], rows[-1] = 0, N - 1
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb[rows]), 128)
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y)[:, rows], Yref, K) <= GATE


def test_skinny_deterministic_and_strided():
    """Bitwise repeatable (fixed-order cluster reduction), and X / Y with row strides."""
    M, N, K = 24, 640, 1024
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=9)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Xbig = gu.bf16_from_bits(wq_inputs.act_bf16(M, K + 64, seed=10))
    X = Xbig[:, :K]
    Ybig = torch.zeros((M, N + 8), dtype=torch.bfloat16, device="cuda")
    Y1 = wq.wq_w4a16_gemm(X, packed, S, Z, 128, Y=Ybig[:, :N])
    Y2 = wq.wq_w4a16_gemm(X.contiguous(), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    assert Y1.data_ptr() == Ybig.data_ptr()
    assert torch.equal(Ybig[:, :N].contiguous().view(torch.int16), Y2.view(torch.int16))
    assert torch.count_nonzero(Ybig[:, N:]) == 0  # nothing written past N
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb), 128)
    Yref = oracle.w4a16_matmul(gu.bf16_to_f64(X), codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y2), Yref, K) <= GATE


def test_skinny_nonfinite_activation_propagates():
    """An inf activation makes its token's outputs non-finite (as the fp32 products would)
    and leaves the other tokens exact."""
    M, N, K = 10, 256, 512
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=11)
    X = wq_inputs.normal_f64((M, K), 1.0, 12)
    X[3, 100] = np.inf
    Xb = wq_inputs.to_bf16_bits(X)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y = gu.bf16_to_f64(wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128))
    assert wq.wq_get_status() == 0
    assert not np.any(np.isfinite(Y[3]))
    keep = [m for m in range(M) if m != 3]
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb), 128)
    Xk = wq_inputs.bf16_bits_to_f64(Xb[keep])
    Yref = oracle.w4a16_matmul(Xk, codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(Y[keep], Yref, K) <= GATE


@pytest.mark.parametrize("M", [1, 3, 8, 16, 17, 40, 64])
@pytest.mark.parametrize("N,K", [(300, 512), (1024, 2048)])
def test_skinny_w8a16_parity(M, N, K):
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=50 + N)
    Xb = wq_inputs.act_bf16(M, K, seed=51 + M)
    q, S, _ = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb), 8, K, False)
    Y = wq.wq_w8a16_gemm(gu.bf16_from_bits(Xb), q, S)
    assert wq.wq_get_status() == 0
    qo, so = oracle.quantize_sym_int8_per_channel(wq_inputs.bf16_bits_to_f64(Wb))
    np.testing.assert_array_equal(gu.to_np(q), qo)
    Yref = oracle.w8a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), qo, so, "exact")
    y = gu.bf16_to_f64(Y)
    assert oracle.gemm_gate(y, Yref, K) <= GATE
    assert oracle.rel_frobenius(Yref, y) < 4e-3


@pytest.mark.parametrize("M", [1, 4])
def test_skinny_w8a16_7b_shapes_sampled(M):
    """W8A16 decode on the 7B-class shapes (sampled rows): M = 1 on the row kernel, M = 4
    on the skinny kernel."""
    for (N, K) in wq_inputs.SHAPES_7B:
        Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N + 1)
        Xb = wq_inputs.act_bf16(M, K, seed=K + 1)
        q, S, _ = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb), 8, K, False)
        Y = wq.wq_w8a16_gemm(gu.bf16_from_bits(Xb), q, S)
        assert wq.wq_get_status() == 0
        rows = np.sort(np.random.default_rng(N).choice(N, 48, replace=False))
        rows[0], rows[-1] = 0, N - 1
        qo, so = oracle.quantize_sym_int8_per_channel(wq_inputs.bf16_bits_to_f64(Wb[rows]))
        Yref = oracle.w8a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), qo, so, "exact")
        assert oracle.gemm_gate(gu.bf16_to_f64(Y)[:, rows], Yref, K) <= GATE
