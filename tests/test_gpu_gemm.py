"""GPU parity of the W4A16 / W8A16 matmul against the float64 oracle on the same
dequantized weights. Gate: max |y - y_ref| / max(|y_ref|, 1e-3 rms(y_ref)) <= 1e-2
(bf16 output rounding is 2^-9 relative; fp32 accumulation adds ~1e-6)."""
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


def _quantize_both(Wb, group):
    """GPU quantization of bf16 W and the oracle's; asserts they agree bit for bit."""
    Wt = gu.bf16_from_bits(Wb)
    if group == 0:
        packed, S, Z = wq.wq_quantize_rtn_per_tensor(Wt)
    else:
        packed, S, Z = wq.wq_quantize_rtn_g128(Wt, 4, group, True)
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb), group)
    np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))
    np.testing.assert_array_equal(gu.bits16(S).ravel(), gu.f16_bits_of(So).ravel())
    return packed, S, Z, codes, So, Zo


def test_tiny_config():
    """W fp32 256x512, X bf16 1x512: Y 1x256 against the oracle."""
    W, Xb = wq_inputs.tiny_config()
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.f32(W))
    codes, So, Zo = oracle.quantize_rtn_asym(W.astype(np.float64), 128)
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    assert Y.shape == (1, 256)
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE


SHAPES = [(256, 512), (300, 1152), (1000, 4096), (77, 2304), (129, 11008)]


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 8])
def test_small_m_parity(N, K, M):
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N + K)
    Xb = wq_inputs.act_bf16(M, K, seed=M)
    packed, S, Z, codes, So, Zo = _quantize_both(Wb, 128)
    X = gu.bf16_from_bits(Xb)
    Y = wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    y = gu.bf16_to_f64(Y)
    assert oracle.gemm_gate(y, Yref) <= GATE
    assert oracle.rel_frobenius(Yref, y) < 4e-3
    Y2 = wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    assert torch.equal(Y, Y2), "fixed reduction order: repeated runs are bitwise identical"


@pytest.mark.parametrize("group", [32, 256, 2304, 0])
@pytest.mark.parametrize("M", [1, 4])
def test_granularities(group, M):
    Wb, Xb, _ = wq_inputs.outlier_config(N=96, K=2304, M=M)
    packed, S, Z, codes, So, Zo = _quantize_both(Wb, group)
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, group)
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, group, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE


def test_strided_x_and_y():
    N, K, M = 200, 1024, 3
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=9)
    Xwide = gu.bf16_from_bits(wq_inputs.act_bf16(M, K + 64, seed=2))
    X = Xwide[:, 64:]
    packed, S, Z, codes, So, Zo = _quantize_both(Wb, 128)
    Ybig = torch.full((M, N + 40), float("nan"), dtype=torch.bfloat16, device="cuda")
    Y = Ybig[:, 8:8 + N]
    wq.wq_w4a16_gemm(X, packed, S, Z, 128, Y=Y)
    Yref = oracle.w4a16_matmul(gu.bf16_to_f64(X), codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE
    assert torch.isnan(Ybig[:, :8]).all() and torch.isnan(Ybig[:, 8 + N:]).all()


@pytest.mark.parametrize("N,K", [(4096, 4096), (11008, 4096), (4096, 11008)])
def test_full_size_decode_sampled(N, K):
    """7B-class layer shapes at M = 1 in the benchmark's configuration: GPU quantization
    of the whole W, GEMV over all N rows; the oracle quantizes and multiplies 64 sampled
    rows on its own."""
    Wb = wq_inputs.weight_bf16(N, K, 0.02)
    Xb = wq_inputs.act_bf16(1, K)
    Wt = gu.bf16_from_bits(Wb)
    packed, S, Z = wq.wq_quantize_rtn_g128(Wt)
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    rows = np.sort(np.random.default_rng(N + K).choice(N, 64, replace=False))
    rows[0], rows[-1] = 0, N - 1
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb[rows]), 128)
    np.testing.assert_array_equal(gu.to_np(packed)[rows], oracle.pack_int4(codes))
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y)[:, rows], Yref) <= GATE


# N a multiple of 16, short and long rows: for M = 2..4 the streaming kernel on 16-row tiles
# (short rows) and the TMA-fed kernel on 32-row tiles (K = 11008), for M = 1 the bulk-copy
# kernel (short rows) and the TMA-fed one (K = 11008)
STREAM_SHAPES = [(16, 128), (48, 384), (160, 1152), (32, 11008), (256, 4096)]


@pytest.mark.parametrize("N,K", STREAM_SHAPES)
@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_stream_tiles_and_chunks(N, K, M):
    """One tile, ragged last chunks (G = 3, 9, 86 groups), every M of the kernel, X with a
    row stride above K; bitwise repeatable."""
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N * 7 + K)
    Xwide = gu.bf16_from_bits(wq_inputs.act_bf16(M, K + 128, seed=M + 40))
    X = Xwide[:, 128:]
    packed, S, Z, codes, So, Zo = _quantize_both(Wb, 128)
    Y = wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    Yref = oracle.w4a16_matmul(gu.bf16_to_f64(X), codes, So, Zo, 128, "exact")
    y = gu.bf16_to_f64(Y)
    assert oracle.gemm_gate(y, Yref) <= GATE
    assert oracle.rel_frobenius(Yref, y) < 4e-3
    assert torch.equal(Y, wq.wq_w4a16_gemm(X, packed, S, Z, 128))


@pytest.mark.parametrize("N,K,M", [(16576, 4096, 1), (11888, 1024, 4), (14208, 256, 2)])
def test_stream_many_tiles_sampled(N, K, M):
    """CTAs that own more tiles than there are S'/Z slots and more chunks than ring stages
    (16576 x 4096: 7 tiles, 56 chunks per CTA on 148 SMs), and a last CTA with fewer tiles;
    the oracle checks sampled rows, including the first and last."""
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N)
    Xb = wq_inputs.act_bf16(M, K, seed=N + 1)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    rows = np.sort(np.random.default_rng(N).choice(N, 96, replace=False))
    rows[0], rows[-1] = 0, N - 1
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb[rows]), 128)
    np.testing.assert_array_equal(gu.to_np(packed)[rows], oracle.pack_int4(codes))
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y)[:, rows], Yref) <= GATE


@pytest.mark.parametrize("N,K", [(8, 256), (100, 768), (1000, 4096), (4104, 4096), (96, 11008),
                                 (300, 8192), (48, 28672), (32, 40960)])
def test_m1_decode_shapes(N, K):
    """M = 1 at assorted sizes: one row block, ragged row blocks, a row count just past a
    multiple of the tile, K up to 11008, and K whose rows do not fit in shared memory whole:
    28672 (the 70B down projection's K) with N = 48 on the register-fed MMA kernel, and
    40960 with N = 32 on the TMA-fed kernel in chunks of 8 groups; bitwise repeatable."""
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N + 5 * K)
    Xb = wq_inputs.act_bf16(1, K, seed=K)
    packed, S, Z, codes, So, Zo = _quantize_both(Wb, 128)
    X = gu.bf16_from_bits(Xb)
    Y = wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    y = gu.bf16_to_f64(Y)
    assert oracle.gemm_gate(y, Yref) <= GATE
    assert oracle.rel_frobenius(Yref, y) < 4e-3
    assert torch.equal(Y, wq.wq_w4a16_gemm(X, packed, S, Z, 128))


@pytest.mark.parametrize("M", [8, 9, 16, 24, 32])
@pytest.mark.parametrize("N,K", [(256, 4096), (32, 11008)])
def test_token_block_passes(N, K, M):
    """M with no single fast decode kernel (M = 8 at K = 11008, and 9..32) runs as passes
    over blocks of tokens; each pass is an exact-mode decode."""
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N + 3 * K)
    Xb = wq_inputs.act_bf16(M, K, seed=M + 77)
    packed, S, Z, codes, So, Zo = _quantize_both(Wb, 128)
    X = gu.bf16_from_bits(Xb)
    Y = wq.wq_w4a16_gemm(X, packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    y = gu.bf16_to_f64(Y)
    assert oracle.gemm_gate(y, Yref) <= GATE
    assert oracle.rel_frobenius(Yref, y) < 4e-3


@pytest.mark.parametrize("M", [16, 32])
def test_skinny_full_size_sampled(M):
    """11008 x 4096 at M = 16 and 32 (the skinny decode sizes), sampled rows."""
    N, K = 11008, 4096
    Wb = wq_inputs.weight_bf16(N, K, 0.02)
    Xb = wq_inputs.act_bf16(M, K, seed=5)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    rows = np.sort(np.random.default_rng(M).choice(N, 48, replace=False))
    rows[0], rows[-1] = 0, N - 1
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb[rows]), 128)
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y)[:, rows], Yref) <= GATE


@pytest.mark.parametrize("M", [1, 3, 8])
def test_w8a16_small_m(M):
    N, K = 130, 2048
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=11)
    Xb = wq_inputs.act_bf16(M, K, seed=12)
    q, S, _ = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb), 8, K, False)
    qo, so = oracle.quantize_sym_int8_per_channel(wq_inputs.bf16_bits_to_f64(Wb))
    np.testing.assert_array_equal(gu.to_np(q), qo)
    Y = wq.wq_w8a16_gemm(gu.bf16_from_bits(Xb), q, S)
    Yref = oracle.w8a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), qo, so, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE


@pytest.mark.parametrize("M,N,K", [(1, 256, 4096), (1, 64, 11008), (3, 160, 4096), (8, 128, 2048),
                                   (64, 136, 1024), (96, 136, 1024)])
def test_symmetric_int4_matmul(M, N, K):
    """Symmetric INT4 weights (codes q + 8, Z = 8) through the same matmul kernels: the
    decode and skinny kernels (M <= 64) against the exact product, the tensor-core GEMM
    (M = 96) against the bf16-rounded weights."""
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N + K)
    Xb = wq_inputs.act_bf16(M, K, seed=M + 9)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb), 4, 128, False)
    q, So = oracle.quantize_rtn_sym_int4(wq_inputs.bf16_bits_to_f64(Wb), 128)
    codes, So, Zo = oracle.sym_int4_storage(q, So)
    np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    mode = "exact" if M <= 64 else "bf16"
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, mode)
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE


def test_host_memory_is_rejected_before_launch():
    """Pointers that are not memory of the current device are refused with WQ_ERR_DEVICE
    before anything is launched (pinned host memory here: even a launch would only have
    read it through unified addressing, so the check itself is what the test observes)."""
    N, K = 64, 1024
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=5)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Xh = torch.zeros((1, K), dtype=torch.bfloat16).pin_memory()
    Y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_w4a16_gemm(Xh, packed, S, Z, 128, Y=Y)
    assert e.value.status == 11
    Ph = packed.cpu().pin_memory()
    with pytest.raises(wq.WQError) as e:
        wq.wq_dequant(Ph, S, Z, 128)
    assert e.value.status == 11
    assert wq.wq_get_status() == 0


def _sampled_rows(N, k, seed):
    rows = np.sort(np.random.default_rng(seed).choice(N, k, replace=False))
    rows[0], rows[-1] = 0, N - 1
    return rows


@pytest.mark.parametrize("N,K", [(28672, 8192), (8192, 28672)])
@pytest.mark.parametrize("M", [8, 32])
def test_70b_skinny_sampled(N, K, M):
    """70B-class decode layers at M = 8 and 32 in the benchmark's configuration (the whole W
    quantized and multiplied on the GPU); the oracle quantizes and multiplies 64 sampled rows,
    the first and last among them. Both run on the skinny tensor-core kernel, whose
    exact bf16 products of the centred codes and the activations, summed in fp32 per group,
    are scaled by S' per group: the product is with the exact S'(q - Z)."""
    Wb = wq_inputs.weight_bf16(N, K, 0.015)
    Xb = wq_inputs.act_bf16(M, K)
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.bf16_from_bits(Wb))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    rows = _sampled_rows(N, 64, N + M)
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb[rows]), 128)
    np.testing.assert_array_equal(gu.to_np(packed)[rows], oracle.pack_int4(codes))
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    y = gu.bf16_to_f64(Y)[:, rows]
    assert oracle.gemm_gate(y, Yref, K) <= GATE
    assert oracle.rel_frobenius(Yref, y) < 4e-3


@pytest.mark.parametrize("group", [4096, 0])
def test_outlier_config_m8_channel_and_tensor(group):
    """The outlier-stress configuration itself (W 4096 x 4096 with 0.1% of the input columns
    scaled x20-100, X 8 x 4096 with the same channels scaled) at per-channel and per-tensor
    scales: codes, S' and Z bit-exact against the oracle (all rows per tensor, sampled rows
    per channel), and Y on sampled rows within the gate."""
    Wb, Xb, _ = wq_inputs.outlier_config(N=4096, K=4096, M=8)
    Wt = gu.bf16_from_bits(Wb)
    if group:
        packed, S, Z = wq.wq_quantize_rtn_g128(Wt, 4, group, True)
    else:
        packed, S, Z = wq.wq_quantize_rtn_per_tensor(Wt)
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, group)
    assert wq.wq_get_status() == 0
    W64 = wq_inputs.bf16_bits_to_f64(Wb)
    rows = _sampled_rows(4096, 128, 11 + group)
    if group:
        codes, So, Zo = oracle.quantize_rtn_asym(W64[rows], group)
        np.testing.assert_array_equal(gu.to_np(packed)[rows], oracle.pack_int4(codes))
        np.testing.assert_array_equal(gu.bits16(S)[rows].ravel(), gu.f16_bits_of(So).ravel())
        np.testing.assert_array_equal(gu.bits16(Z)[rows].ravel(), gu.f16_bits_of(Zo).ravel())
    else:
        codes_all, So, Zo = oracle.quantize_rtn_asym(W64, 0)
        np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes_all))
        np.testing.assert_array_equal(gu.bits16(S).ravel(), gu.f16_bits_of(So).ravel())
        np.testing.assert_array_equal(gu.bits16(Z).ravel(), gu.f16_bits_of(Zo).ravel())
        codes = codes_all[rows]
    What = oracle.dequant_asym(codes, So, Zo, group)
    Yref = oracle.matmul_f64(wq_inputs.bf16_bits_to_f64(Xb), What)
    assert oracle.gemm_gate(gu.bf16_to_f64(Y)[:, rows], Yref) <= GATE


@pytest.mark.parametrize("N,K,group", [(77, 1120, 32), (80, 1120, 32), (77, 1120, 0)])
def test_m1_fallback_kernels(N, K, group):
    """M = 1 shapes that none of the tiled decode kernels take (K not a multiple of 128, N not
    a multiple of 16): the register-fed kernels, by rows of 8 (N = 80) or not (N = 77)."""
    Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=N + K + group)
    Xb = wq_inputs.act_bf16(1, K, seed=3)
    packed, S, Z, codes, So, Zo = _quantize_both(Wb, group)
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, group)
    assert wq.wq_get_status() == 0
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, group, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= GATE
