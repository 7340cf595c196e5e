"""Failure detection on the GPU without a fault: a bounded mbarrier wait that nothing
satisfies gives up after its limit, the kernel records WQ_ERR_TIMEOUT and returns, the
status read reports and clears it, and the context keeps running kernels."""
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

TIMEOUT = 8  # WQ_ERR_TIMEOUT


@pytest.mark.parametrize("spin", [True, False])
def test_bounded_wait_times_out_and_context_survives(spin):
    assert wq.wq_get_status() == 0
    limit_ns = 20_000_000
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    wq.wq_selftest_bounded_wait(limit_ns, spin)
    e1.record()
    assert wq.wq_get_status() == TIMEOUT
    assert e0.elapsed_time(e1) >= 0.8 * limit_ns / 1e6   # it waited (about) its limit
    assert wq.wq_get_status() == 0                      # the read cleared the word
    # the context still runs the library's kernels correctly
    W, Xb = wq_inputs.tiny_config()
    packed, S, Z = wq.wq_quantize_rtn_g128(gu.f32(W))
    Y = wq.wq_w4a16_gemm(gu.bf16_from_bits(Xb), packed, S, Z, 128)
    assert wq.wq_get_status() == 0
    codes, So, Zo = oracle.quantize_rtn_asym(W.astype(np.float64), 128)
    np.testing.assert_array_equal(gu.to_np(packed), oracle.pack_int4(codes))
    Yref = oracle.w4a16_matmul(wq_inputs.bf16_bits_to_f64(Xb), codes, So, Zo, 128, "exact")
    assert oracle.gemm_gate(gu.bf16_to_f64(Y), Yref) <= 1e-2
