"""GPU parity of the tensor-core (tcgen05/TMEM) W4A16 / W8A16 GEMM (M > 8) against the
float64 oracle on the same dequantized weights: the kernel rounds S'(q - Z) to bfloat16
before the tensor core, so the oracle runs in "bf16" mode. Gate as in test_gpu_gemm."""
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


def _run(M, N, K, group=128, seed=0):
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=seed + N)
    Xb = wq_inputs.act_bf16(M, K, seed=seed + M)
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb), group)
    packed = gu.u8(oracle.pack_int4(codes))
    S = gu.f16_from_values(So.ravel()).reshape(So.shape)
    Z = gu.f16_from_values(Zo.ravel()).reshape(Zo.shape)
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, group)
    assert wq.wq_get_status() == 0
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, group, "bf16")
    return gu.bf16_to_f64(Y), Yref


# shapes that reach the tensor-core kernel: M > 64, or M > 8 with g != 128 (the skinny
# kernel and the fast decode kernels take g = 128 only)
@pytest.mark.parametrize("M,N,K,group", [(16, 128, 64, 64), (9, 136, 128, 64), (65, 256, 256, 128),
                                         (300, 200, 512, 128), (257, 384, 1024, 128),
                                         (40, 4096, 4096, 256), (72, 4096, 4096, 128)])
def test_tc_gemm_parity(M, N, K, group):
    y, yref = _run(M, N, K, group=group)
    assert oracle.gemm_gate(y, yref) <= GATE
    assert oracle.rel_frobenius(yref, y) < 4e-3


@pytest.mark.parametrize("group", [32, 64, 256, 0])
def test_tc_gemm_groups(group):
    y, yref = _run(40, 160, 512, group=group)
    assert oracle.gemm_gate(y, yref) <= GATE


def test_tc_gemm_prefill_shape_sampled():
    """The prefill workload: X 2048x4096, W 11008x4096 g128, checked on sampled rows."""
    M, N, K = 2048, 11008, 4096
    Wb = wq_inputs.weight_bf16(N, K, 0.02)
    Xb = wq_inputs.act_bf16(M, K)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(N, 48, replace=False))
    toks = np.sort(rng.choice(M, 64, replace=False))
    rows[-1], toks[-1] = N - 1, M - 1
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb[rows]), 128)
    Xs = wq_inputs.bf16_bits_to_f64(Xb[toks])
    Yref = oracle.w4a16_matmul(Xs, codes, So, Zo, 128, "bf16")
    y = gu.bf16_to_f64(Y)[np.ix_(toks, rows)]
    assert oracle.gemm_gate(y, Yref) <= GATE


@pytest.mark.parametrize("M,N,K", [(96, 128, 256), (2048, 1024, 4096)])
def test_tc_w8a16(M, N, K):
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=3)
    Xb = wq_inputs.act_bf16(M, K, seed=4)
    q, S, _ = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb), 8, K, False)
    Y = wq.wq_w8a16_gemm(gu.bf16_from_bits(Xb), q, S)
    assert wq.wq_get_status() == 0
    qo, so = oracle.quantize_sym_int8_per_channel(wq_inputs.bf16_bits_to_f64(Wb))
    Yref = oracle.w8a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), qo, so, "bf16")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE


def test_tc_gemm_deterministic():
    M, N, K = 300, 512, 1024
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=8)
    X = gu.bf16_from_bits(wq_inputs.act_bf16(M, K, seed=9))
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y1 = wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    Y2 = wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("M,N,K", [(512, 4096, 11008), (96, 1024, 28672)])
def test_tc_gemm_long_k_sampled(M, N, K):
    """Long contractions (the 7B down projection in prefill, a 70B-class K): the tensor core's
    fp32 accumulation error grows with K, so the gate's floor is the one derived from K."""
    Wb = wq_inputs.weight_bf16(N, K, 0.015, seed=7)
    Xb = wq_inputs.act_bf16(M, K, seed=8)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    rows = np.sort(np.random.default_rng(6).choice(N, 48, replace=False))
    rows[0], rows[-1] = 0, N - 1
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb[rows]), 128)
    np.testing.assert_array_equal(gu.to_np(packed)[rows], oracle.pack_int4(codes))
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "bf16")
    y = gu.bf16_to_f64(Y)[:, rows]
    assert oracle.gemm_gate(y, Yref, K) <= GATE
    assert oracle.rel_frobenius(Yref, y) < 4e-3


def test_tc_w8a16_long_k_sampled():
    M, N, K = 256, 2048, 11008
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=9)
    Xb = wq_inputs.act_bf16(M, K, seed=10)
    q, S, _ = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb), 8, K, False)
    Y = wq.wq_w8a16_gemm(gu.bf16_from_bits(Xb), q, S)
    assert wq.wq_get_status() == 0
    rows = np.sort(np.random.default_rng(11).choice(N, 48, replace=False))
    qo, so = oracle.quantize_sym_int8_per_channel(wq_inputs.bf16_bits_to_f64(Wb[rows]))
    np.testing.assert_array_equal(gu.to_np(q)[rows], qo)
    Yref = oracle.w8a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), qo, so, "bf16")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y)[:, rows], Yref, K) <= GATE
