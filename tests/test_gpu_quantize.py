"""GPU parity of the quantizer, packer and dequantizer against the CPU oracle: codes, packed
bytes, scales and zero-points bit for bit; dequantized weights bit for bit."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import w4a16_dequant_matmul_b200 as wq  # noqa: E402
import wq_inputs  # noqa: E402
from tests import gpu_util as gu  # noqa: E402


def _check_int4(W64, Wt, group):
    """Quantize Wt (torch, on device) and compare with the oracle on W64 (its exact values)."""
    packed, S, Z = wq.wq_quantize_rtn_g128(Wt, 4, group, True)
    assert wq.wq_get_status() == 0
    codes, So, Zo = oracle.quantize_rtn_asym(W64, group)
    np.testing.assert_array_equal(gu.bits16(S), gu.f16_bits_of(So))
    np.testing.assert_array_equal(gu.bits16(Z), gu.f16_bits_of(Zo))
    np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))
    return packed, S, Z, codes, So, Zo


def test_tiny_config_bitexact():
    W, _ = wq_inputs.tiny_config()
    _check_int4(W.astype(np.float64), gu.f32(W), 128)


@pytest.mark.parametrize("group", [32, 64, 128, 256, 384, 1152])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_random_shapes_and_groups(group, dtype):
    N, K = 37, 1152  # ragged N; K not a multiple of 256 or 1024
    if K % group:
        pytest.skip("group does not divide K")
    sigma = 0.02
    if dtype == "f32":
        W = wq_inputs.to_f32(wq_inputs.normal_f64((N, K), sigma, 3))
        _check_int4(W.astype(np.float64), gu.f32(W), group)
    else:
        Wb = wq_inputs.weight_bf16(N, K, sigma, seed=3)
        _check_int4(wq_inputs.bf16_bits_to_f64(Wb), gu.bf16_from_bits(Wb), group)


def _adversarial_rows(K=256):
    """Rows of two 128-groups each exercising one special case."""
    rows = []
    # exact half-integer ties: S' = 2^-4 exactly, Z = 5, w = (k + 1/2) S'
    ties = [(k + 0.5) * 0.0625 for k in range(-5, 10)]
    g = np.resize(np.array(ties + [-0.3125, 0.625]), 128)
    g[:2] = [-0.3125, 0.625]
    rows.append(np.concatenate([g, g[::-1]]))
    rows.append(np.concatenate([np.full(128, 0.37), np.full(128, -0.37)]))         # constant
    rows.append(np.zeros(K))                                                         # all zero
    rng = np.random.default_rng(21)
    o = rng.normal(0, 0.01, K)
    o[7], o[200] = 5.0, -3.0
    rows.append(o)                                                                   # outlier
    rows.append(rng.normal(0, 1e-9, K))                                              # S' -> 1
    rows.append(rng.normal(0, 1e-6, K))                                              # subnormal S'
    r = np.zeros(K)
    r[0], r[1] = 15.00732421875, -2.0 ** -100                                        # rational tie
    r[128] = 15.00732421875                                                          # exact tie
    rows.append(r)
    rows.append(np.concatenate([np.full(128, 0.0), np.linspace(-1e-3, 2e-3, 128)]))
    big = rng.normal(0, 1, K)
    big[3], big[130] = 449500.0, -449500.0                                           # S~6e4 at g=256
    rows.append(big)
    mags = 10.0 ** rng.uniform(-20, 4, (6, 1))
    rows.extend(list(rng.normal(0, 1, (6, K)) * mags))                               # magnitudes
    one = np.abs(rng.normal(0, 0.1, K))
    rows.append(one)                                                                 # one-signed +
    rows.append(-one)                                                                # one-signed -
    return np.array(rows)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_adversarial_groups(dtype):
    A = _adversarial_rows()
    if dtype == "f32":
        W = wq_inputs.to_f32(A)
        _check_int4(W.astype(np.float64), gu.f32(W), 128)
    else:
        Wb = wq_inputs.to_bf16_bits(A)
        _check_int4(wq_inputs.bf16_bits_to_f64(Wb), gu.bf16_from_bits(Wb), 128)
    for g in (32, 256):
        W = wq_inputs.to_f32(A)
        _check_int4(W.astype(np.float64), gu.f32(W), g)


def _tie_lattice_bits():
    """bf16 groups rich in exact and near half-integer quotients w/S'.

    Each 128-group is built around S0 = m 2^e (m odd, up to 8 bits) and Z0 in 0..15: its
    ends -Z0 S0 and (15 - Z0) S0, every (k + 1/2) S0 in between, and uniform fill. After the
    cast to bf16 many values are exact ties of the group's S' and the rest lie within a few
    ulps of one; a second copy moves half the weights one bf16 ulp up or down."""
    rng = np.random.default_rng(99)
    groups = []
    for m in (1, 3, 5, 7, 9, 11, 13, 15, 17, 25, 31, 63, 127, 255):
        for e in (-22, -12, -5, 0, 4):
            for z in range(16):
                s0 = m * 2.0 ** e
                vals = [-z * s0, (15 - z) * s0] + [(k + 0.5) * s0 for k in range(-z, 15 - z)]
                g = np.resize(np.array(vals), 128)
                g[len(vals):] = rng.uniform(-z * s0, (15 - z) * s0, 128 - len(vals))
                groups.append(g)
    bits = wq_inputs.to_bf16_bits(np.array(groups).reshape(-1, 256)).astype(np.int32)
    move = (rng.random(bits.shape) < 0.5) & ((bits & 0x7FFF) != 0)
    step = np.where(rng.random(bits.shape) < 0.5, 1, -1)
    return np.concatenate([bits, np.where(move, bits + step, bits)]).astype(np.uint16)


def test_tie_lattice_bf16():
    """Round-half-even decisions on exact ties and their bf16 neighbours, every Z parity,
    clipped and unclipped groups."""
    Wb = _tie_lattice_bits()
    _check_int4(wq_inputs.bf16_bits_to_f64(Wb), gu.bf16_from_bits(Wb), 128)


def test_strided_rows():
    """ldw > K: W is a column slice of a wider matrix."""
    big = wq_inputs.to_f32(wq_inputs.normal_f64((20, 640), 0.02, 4))
    Wt = gu.f32(big)[:, 128:640]
    assert Wt.stride(0) == 640
    _check_int4(big[:, 128:640].astype(np.float64), Wt, 128)


def test_per_tensor():
    Wb, _, _ = wq_inputs.outlier_config(N=64, K=512)
    packed, S, Z = wq.wq_quantize_rtn_per_tensor(gu.bf16_from_bits(Wb))
    assert wq.wq_get_status() == 0
    codes, So, Zo = oracle.quantize_rtn_asym(wq_inputs.bf16_bits_to_f64(Wb), 0)
    np.testing.assert_array_equal(gu.bits16(S), gu.f16_bits_of(So.ravel()))
    np.testing.assert_array_equal(gu.bits16(Z), gu.f16_bits_of(Zo.ravel()))
    np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_int8_per_channel(dtype):
    A = np.concatenate([_adversarial_rows(), wq_inputs.normal_f64((20, 256), 0.02, 5)])
    if dtype == "f32":
        W = wq_inputs.to_f32(A)
        W64, Wt = W.astype(np.float64), gu.f32(W)
    else:
        Wb = wq_inputs.to_bf16_bits(A)
        W64, Wt = wq_inputs.bf16_bits_to_f64(Wb), gu.bf16_from_bits(Wb)
    q, S, _ = wq.wq_quantize_rtn_g128(Wt, 8, 256, False)
    assert wq.wq_get_status() == 0
    qo, so = oracle.quantize_sym_int8_per_channel(W64)
    np.testing.assert_array_equal(gu.to_np(q), qo)
    np.testing.assert_array_equal(gu.bits16(S), gu.f16_bits_of(so))


def test_int8_worked_example():
    """The page's INT8 example row (padded with zeros to 32): codes -95, -11, 5, 74, 127."""
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, :5] = [-0.9, -0.1, 0.05, 0.7, 1.2]
    q, S, _ = wq.wq_quantize_rtn_g128(gu.f32(x), 8, 32, False)
    assert gu.to_np(q)[0, :5].tolist() == [-95, -11, 5, 74, 127]


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf, 1.0e6])
def test_nonfinite_and_overflow_status(bad):
    W = np.full((4, 128), 0.01, dtype=np.float32)
    W[2, 77] = bad
    wq.wq_quantize_rtn_g128(gu.f32(W), 4, 128, True)
    assert wq.wq_get_status() == 7          # WQ_ERR_NONFINITE
    assert wq.wq_get_status() == 0          # cleared


def test_pack_bitexact_and_range_status():
    rng = np.random.default_rng(6)
    c = rng.integers(0, 16, (19, 320), dtype=np.uint8)
    p = wq.wq_pack_int4(gu.u8(c))
    assert wq.wq_get_status() == 0
    np.testing.assert_array_equal(gu.to_np(p), oracle.pack_int4(c))
    c[3, 5] = 16
    wq.wq_pack_int4(gu.u8(c))
    assert wq.wq_get_status() == 9          # WQ_ERR_RANGE


@pytest.mark.parametrize("group", [32, 128, 1024, 0])
def test_dequant_bitexact(group):
    Wb = wq_inputs.weight_bf16(29, 1024, 0.02, seed=7)
    W64 = wq_inputs.bf16_bits_to_f64(Wb)
    codes, So, Zo = oracle.quantize_rtn_asym(W64, group)
    packed = gu.u8(oracle.pack_int4(codes))
    S, Z = gu.f16_from_values(So.ravel()), gu.f16_from_values(Zo.ravel())
    ref = oracle.dequant_asym(codes, So, Zo, group)
    out32 = wq.wq_dequant(packed, S, Z, group, torch.float32)
    np.testing.assert_array_equal(gu.to_np(out32).astype(np.float64), ref)
    out16 = wq.wq_dequant(packed, S, Z, group, torch.bfloat16)
    np.testing.assert_array_equal(gu.bits16(out16), oracle.bf16_round_bits(ref))


def test_empty_inputs():
    W = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    packed, S, Z = wq.wq_quantize_rtn_g128(W)
    assert packed.shape == (0, 64)
    X = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    Y = wq.wq_w4a16_gemm(X, torch.empty((5, 64), dtype=torch.uint8, device="cuda"),
                         torch.ones((5, 1), dtype=torch.float16, device="cuda"),
                         torch.zeros((5, 1), dtype=torch.float16, device="cuda"))
    assert Y.shape == (0, 5)


# ------------------------------------------ symmetric INT4 per group (codes q + 8, Z = 8)

def _check_sym4(W64, Wt, group):
    packed, S, Z = wq.wq_quantize_rtn_g128(Wt, 4, group, False)
    assert wq.wq_get_status() == 0
    q, So = oracle.quantize_rtn_sym_int4(W64, group)
    codes, So, Zo = oracle.sym_int4_storage(q, So)
    np.testing.assert_array_equal(gu.bits16(S), gu.f16_bits_of(So))
    np.testing.assert_array_equal(gu.bits16(Z), gu.f16_bits_of(Zo))
    np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))
    return packed, S, Z, codes, So, Zo


@pytest.mark.parametrize("group", [32, 128, 256, 384, 1152])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sym4_random_shapes_and_groups(group, dtype):
    N, K = 37, (1152 if 1152 % group == 0 else 1024)  # ragged N; K a multiple of g
    if dtype == "f32":
        W = wq_inputs.to_f32(wq_inputs.normal_f64((N, K), 0.02, 4))
        _check_sym4(W.astype(np.float64), gu.f32(W), group)
    else:
        Wb = wq_inputs.weight_bf16(N, K, 0.02, seed=4)
        _check_sym4(wq_inputs.bf16_bits_to_f64(Wb), gu.bf16_from_bits(Wb), group)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_sym4_adversarial_groups(dtype):
    A = _adversarial_rows()
    if dtype == "f32":
        W = wq_inputs.to_f32(A)
        _check_sym4(W.astype(np.float64), gu.f32(W), 128)
    else:
        Wb = wq_inputs.to_bf16_bits(A)
        _check_sym4(wq_inputs.bf16_bits_to_f64(Wb), gu.bf16_from_bits(Wb), 128)


def _sym_tie_lattice_bits():
    """bf16 groups whose max|w| is 7 S0 with S0 = m 2^e a binary16 value, so s' = S0, holding
    every exact tie (k + 1/2) S0 of the symmetric grid (k = -8..6) and fill; a second copy
    moves half of the weights one bf16 ulp."""
    rng = np.random.default_rng(98)
    groups = []
    for m in (1, 3, 5, 7, 9, 11, 13, 15, 17):
        for e in (-20, -9, -3, 0, 5):
            s0 = m * 2.0 ** e
            for sign in (1.0, -1.0):
                vals = [sign * 7 * s0] + [(k + 0.5) * s0 for k in range(-8, 7)]
                g = np.resize(np.array(vals), 128)
                g[len(vals):] = rng.uniform(-7 * s0, 7 * s0, 128 - len(vals))
                groups.append(g)
    bits = wq_inputs.to_bf16_bits(np.array(groups).reshape(-1, 256)).astype(np.int32)
    move = (rng.random(bits.shape) < 0.5) & ((bits & 0x7FFF) != 0)
    step = np.where(rng.random(bits.shape) < 0.5, 1, -1)
    return np.concatenate([bits, np.where(move, bits + step, bits)]).astype(np.uint16)


def test_sym4_tie_lattice_bf16():
    Wb = _sym_tie_lattice_bits()
    _check_sym4(wq_inputs.bf16_bits_to_f64(Wb), gu.bf16_from_bits(Wb), 128)


def test_sym4_dequant_bitexact():
    Wb = wq_inputs.weight_bf16(64, 1024, 0.02, seed=6)
    packed, S, Z, codes, So, Zo = _check_sym4(wq_inputs.bf16_bits_to_f64(Wb),
                                              gu.bf16_from_bits(Wb), 128)
    W_hat = wq.wq_dequant(packed, S, Z, 128, torch.float32)
    np.testing.assert_array_equal(gu.to_np(W_hat).astype(np.float64),
                                  oracle.dequant_asym(codes, So, Zo, 128))
