"""The C-ABI library builds, loads and exports every function include/wq.h declares, and its
host-side argument checks reject bad calls before touching a device (CPU only: no kernel
runs, and the fake pointers passed here are never dereferenced)."""
import ctypes
import os
import re

import pytest

import w4a16_dequant_matmul_b200 as wq
from w4a16_dequant_matmul_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wq.h")

OK, NULL, SHAPE, ALIGN, DTYPE, UNSUP, NODEV = 0, 1, 2, 3, 4, 5, 10
FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced
ODD = ctypes.c_void_p(0x10008)       # 8-byte but not 16-byte aligned


@pytest.fixture(scope="module")
def lib():
    _build.build_library()
    return wq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("wq_quantize_rtn_g128", "wq_pack_int4", "wq_dequant", "wq_w4a16_gemm"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(wq._SIGNATURES), "binding must wrap every C entry point"


def test_version_and_status_strings(lib):
    assert wq.wq_version() == 100
    for code in range(12):
        s = wq.wq_status_string(code)
        assert s and s != "unknown status"
    assert wq.wq_status_string(99) == "unknown status"


def _qp(w_bit=4, group=128, zp=1):
    return ctypes.byref(wq._QParams(w_bit, group, zp))


def test_quantize_argument_checks(lib):
    f = lib.wq_quantize_rtn_g128
    # empty problems are a no-op
    assert f(None, wq.WQ_BF16, 0, 128, 128, None, None, None, None, None) == OK
    assert f(FAKE, wq.WQ_BF16, -1, 128, 128, None, FAKE, FAKE, FAKE, None) == SHAPE
    assert f(FAKE, wq.WQ_F16, 4, 128, 128, None, FAKE, FAKE, FAKE, None) == DTYPE
    assert f(None, wq.WQ_BF16, 4, 128, 128, None, FAKE, FAKE, FAKE, None) == NULL
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, None, FAKE, FAKE, None, None) == NULL
    assert f(FAKE, wq.WQ_BF16, 4, 100, 128, None, FAKE, FAKE, FAKE, None) == SHAPE   # K % 32
    assert f(FAKE, wq.WQ_BF16, 4, 192, 192, None, FAKE, FAKE, FAKE, None) == SHAPE   # K % g
    assert f(FAKE, wq.WQ_BF16, 4, 128, 64, None, FAKE, FAKE, FAKE, None) == SHAPE    # ldw < K
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, _qp(4, 48), FAKE, FAKE, FAKE, None) == SHAPE
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, _qp(3, 128), FAKE, FAKE, FAKE, None) == UNSUP
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, _qp(8, 128, 0), FAKE, FAKE, FAKE, None) == UNSUP
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, _qp(8, 64, 0), FAKE, FAKE, None, None) == UNSUP
    # symmetric INT4 ({4, g, 0}) takes the INT4 checks: Z required, g a multiple of 32 dividing K
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, _qp(4, 128, 0), FAKE, FAKE, None, None) == NULL
    assert f(FAKE, wq.WQ_BF16, 4, 192, 192, _qp(4, 128, 0), FAKE, FAKE, FAKE, None) == SHAPE
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, _qp(4, 128, 2), FAKE, FAKE, FAKE, None) == UNSUP
    assert f(ODD, wq.WQ_BF16, 4, 128, 128, None, FAKE, FAKE, FAKE, None) == ALIGN
    assert f(FAKE, wq.WQ_BF16, 4, 128, 132, None, FAKE, FAKE, FAKE, None) == ALIGN   # row stride
    assert f(FAKE, wq.WQ_BF16, 4, 128, 128, None, ODD, FAKE, FAKE, None) == ALIGN


def test_gemm_argument_checks(lib):
    g = lib.wq_w4a16_gemm
    assert g(FAKE, 0, 128, FAKE, FAKE, FAKE, 64, 128, 128, FAKE, 64, None) == OK    # M = 0
    assert g(FAKE, 1, 128, FAKE, FAKE, FAKE, 0, 128, 128, FAKE, 64, None) == OK     # N = 0
    assert g(FAKE, 1, 128, FAKE, FAKE, FAKE, 64, 0, 128, FAKE, 64, None) == SHAPE   # K = 0
    assert g(None, 1, 128, FAKE, FAKE, FAKE, 64, 128, 128, FAKE, 64, None) == NULL
    assert g(FAKE, 1, 128, FAKE, FAKE, None, 64, 128, 128, FAKE, 64, None) == NULL
    assert g(FAKE, 1, 96, FAKE, FAKE, FAKE, 64, 128, 128, FAKE, 64, None) == SHAPE  # ldx < K
    assert g(FAKE, 2, 128, FAKE, FAKE, FAKE, 64, 128, 128, FAKE, 32, None) == SHAPE # ldy < N
    assert g(FAKE, 1, 128, FAKE, FAKE, FAKE, 64, 128, 96, FAKE, 64, None) == SHAPE  # K % g
    assert g(FAKE, 1, 132, FAKE, FAKE, FAKE, 64, 128, 128, FAKE, 64, None) == ALIGN # ldx % 8
    assert g(ODD, 1, 128, FAKE, FAKE, FAKE, 64, 128, 128, FAKE, 64, None) == ALIGN
    h = lib.wq_w8a16_gemm
    assert h(FAKE, 1, 128, None, FAKE, 64, 128, FAKE, 64, None) == NULL
    assert h(FAKE, 1, 128, FAKE, FAKE, 64, 100, FAKE, 64, None) == SHAPE


def test_selftest_argument_checks(lib):
    f = lib.wq_selftest_bounded_wait
    assert f(0, 1, None) == SHAPE
    assert f(2_000_000_000, 0, None) == SHAPE


def test_pack_dequant_argument_checks(lib):
    assert lib.wq_pack_int4(FAKE, 4, 100, FAKE, None) == SHAPE
    assert lib.wq_pack_int4(None, 4, 128, FAKE, None) == NULL
    assert lib.wq_pack_int4(ODD, 4, 128, FAKE, None) == ALIGN
    d = lib.wq_dequant
    assert d(FAKE, FAKE, FAKE, 4, 128, 128, FAKE, wq.WQ_F16, None) == DTYPE
    assert d(FAKE, FAKE, FAKE, 4, 128, 48, FAKE, wq.WQ_F32, None) == SHAPE
    assert d(FAKE, None, FAKE, 4, 128, 128, FAKE, wq.WQ_F32, None) == NULL
    p = lib.wq_quantize_rtn_per_tensor
    assert p(FAKE, wq.WQ_BF16, 4, 128, 128, FAKE, FAKE, FAKE, None, 0, None) == NULL


def test_scale_folding_argument_checks(lib):
    RANGE_ALPHA = (-0.1, 1.5, float("nan"))
    c = lib.wq_channel_stat
    assert c(FAKE, wq.WQ_BF16, 8, 0, 0, 0, FAKE, None) == OK          # no columns: no-op
    assert c(FAKE, wq.WQ_BF16, 0, 64, 64, 0, FAKE, None) == SHAPE     # statistic over no rows
    assert c(FAKE, wq.WQ_F16, 8, 64, 64, 0, FAKE, None) == DTYPE
    assert c(FAKE, wq.WQ_BF16, 8, 64, 64, 2, FAKE, None) == UNSUP     # unknown statistic
    assert c(None, wq.WQ_BF16, 8, 64, 64, 1, FAKE, None) == NULL
    assert c(FAKE, wq.WQ_BF16, 8, 60, 64, 0, FAKE, None) == SHAPE     # cols % 8
    assert c(FAKE, wq.WQ_BF16, 8, 64, 32, 0, FAKE, None) == SHAPE     # lda < cols
    assert c(ODD, wq.WQ_BF16, 8, 64, 64, 0, FAKE, None) == ALIGN
    assert c(FAKE, wq.WQ_BF16, 8, 64, 68, 0, FAKE, None) == ALIGN     # row stride 136 B
    for f, args in ((lib.wq_smooth_scales, lambda a: (FAKE, FAKE, 64, a, FAKE, None)),
                    (lib.wq_awq_scales, lambda a: (FAKE, 64, a, FAKE, None))):
        for a in RANGE_ALPHA:
            assert f(*args(a)) == SHAPE
    assert lib.wq_smooth_scales(FAKE, None, 64, 0.5, FAKE, None) == NULL
    assert lib.wq_smooth_scales(FAKE, FAKE, 0, 0.5, None, None) == OK
    assert lib.wq_awq_scales(None, 64, 0.5, FAKE, None) == NULL
    q = lib.wq_quantize_rtn_scaled
    assert q(FAKE, wq.WQ_BF16, 4, 128, 128, None, None, FAKE, FAKE, FAKE, None) == NULL  # no s
    assert q(FAKE, wq.WQ_BF16, 4, 128, 128, FAKE, _qp(8, 128, 0), FAKE, FAKE, FAKE,
             None) == UNSUP
    assert q(FAKE, wq.WQ_BF16, 4, 192, 192, FAKE, None, FAKE, FAKE, FAKE, None) == SHAPE
    assert q(FAKE, wq.WQ_BF16, 4, 128, 128, ODD, None, FAKE, FAKE, FAKE, None) == ALIGN
    assert q(FAKE, wq.WQ_I8, 4, 128, 128, FAKE, None, FAKE, FAKE, FAKE, None) == DTYPE
    a = lib.wq_scale_activations
    assert a(FAKE, 0, 64, 64, FAKE, FAKE, 64, None) == OK
    assert a(FAKE, 2, 60, 64, FAKE, FAKE, 64, None) == SHAPE             # K % 8
    assert a(FAKE, 2, 64, 64, FAKE, FAKE, 32, None) == SHAPE             # ldxs < K
    assert a(FAKE, 2, 64, 64, ODD, FAKE, 64, None) == ALIGN              # s alignment
    assert a(FAKE, 2, 64, 64, FAKE, FAKE, 72, None) == UNSUP             # in place, other ld


def test_gptq_argument_checks(lib):
    g = lib.wq_quantize_gptq
    ws = lib.wq_gptq_workspace_bytes(64, 256)
    assert ws == 8 * 256 * 256 + 32 * 256
    args = lambda **kw: (kw.get("W", FAKE), kw.get("dt", wq.WQ_BF16), kw.get("N", 64),
                         kw.get("K", 256), kw.get("ldw", 256), kw.get("X", FAKE), kw.get("T", 32),
                         kw.get("ldx", 256), kw.get("damp", 0.01), kw.get("qp", None), FAKE, FAKE,
                         FAKE, kw.get("ws", FAKE), kw.get("wsb", ws), None)
    assert g(*args(N=0)) == OK
    assert g(*args(X=None)) == NULL
    assert g(*args(T=0)) == SHAPE
    assert g(*args(K=96, ldw=96, ldx=96)) == SHAPE         # K % 64
    assert g(*args(damp=-1.0)) == SHAPE
    assert g(*args(wsb=ws - 8)) == SHAPE                  # workspace too small
    assert g(*args(qp=_qp(8, 256, 0))) == UNSUP
    assert g(*args(K=16384, ldw=16384, ldx=16384, wsb=1 << 40)) == UNSUP  # K > 8192
    assert g(*args(ws=ODD)) == ALIGN


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="host without a GPU only")
def test_valid_call_without_device_reports_nodevice(lib):
    """A call that passes every host check but finds no sm_100 device fails loudly
    (WQ_ERR_NODEVICE), and the Python binding raises: there is no CPU fallback."""
    assert lib.wq_w4a16_gemm(FAKE, 1, 128, FAKE, FAKE, FAKE, 64, 128, 128, FAKE, 64, None) == NODEV
    assert lib.wq_selftest_bounded_wait(20_000_000, 1, None) == NODEV
    sym = ctypes.byref(wq._QParams(4, 128, 0))
    assert lib.wq_quantize_rtn_g128(FAKE, wq.WQ_BF16, 4, 128, 128, sym, FAKE, FAKE, FAKE,
                                    None) == NODEV
    assert lib.wq_get_status(None) in (NODEV, 6)


class _FakeCudaTensor:
    """Stands in for a CUDA tensor on device `dev` (nothing is ever dereferenced)."""

    def __init__(self, shape, dev, addr=0x10000):
        self.shape = shape
        self._dev = dev
        self._addr = addr

    def get_device(self):
        return self._dev

    def dim(self):
        return len(self.shape)

    def stride(self, i=None):
        st = (self.shape[1], 1)
        return st if i is None else st[i]

    def data_ptr(self):
        return self._addr


def test_binding_makes_the_tensors_device_current(monkeypatch):
    """The C library works on the current device and rejects other devices' memory, so the
    binding switches to the device that holds the tensors for the call (host-side mock: a
    tensor "on cuda:1" while cuda:0 is current; no GPU is touched)."""
    import torch

    current = [0]
    seen = []

    class _Dev:
        def __init__(self, d):
            self.d = d

        def __enter__(self):
            self.prev, current[0] = current[0], self.d

        def __exit__(self, *exc):
            current[0] = self.prev

    monkeypatch.setattr(torch.cuda, "device", _Dev)
    monkeypatch.setattr(wq, "_GET_DEVICE", lambda: current[0])

    def fake_gemm(*args):
        seen.append(current[0])
        return 0

    monkeypatch.setattr(wq, "_GEMM", fake_gemm)

    class _Stream:
        cuda_stream = 0

    M, N, K = 1, 64, 128
    X = _FakeCudaTensor((M, K), 1)
    P = _FakeCudaTensor((N, K // 2), 1)
    S = _FakeCudaTensor((N, 1), 1)
    Y = _FakeCudaTensor((M, N), 1)
    wq.wq_w4a16_gemm(X, P, S, S, 128, Y=Y, stream=_Stream())
    assert seen == [1] and current[0] == 0, "called on the tensors' device, then restored"
    # tensors already on the current device: no switch
    X0, P0, S0, Y0 = (_FakeCudaTensor(t.shape, 0) for t in (X, P, S, Y))
    wq.wq_w4a16_gemm(X0, P0, S0, S0, 128, Y=Y0, stream=_Stream())
    assert seen == [1, 0]
