"""The allocation-free per-tensor quantizer (for callers that may not allocate device
memory, such as engine plugins or code under a framework's caching allocator) gives the
same packed codes, scale and zero-point as the workspace-taking entry point.

Called through the C ABI directly, twice in a row with different weights, so a second
call that reused stale contents of the library's shared scratch array would show up.
This file sorts last so that a run stopping at the first failure has run everything
else; it also passes on its own in a fresh process (the first call sets the array up).
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import oracle  # noqa: E402
import w4a16_dequant_matmul_b200 as wq  # noqa: E402
import wq_inputs  # noqa: E402


def _noalloc_via_c_abi(W):
    N, K = W.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    S = torch.empty((1,), dtype=torch.float16, device=W.device)
    Z = torch.empty((1,), dtype=torch.float16, device=W.device)
    dt = wq.WQ_F32 if W.dtype == torch.float32 else wq.WQ_BF16
    st = wq.lib().wq_quantize_rtn_per_tensor_noalloc(
        ctypes.c_void_p(W.data_ptr()), dt, N, K, W.stride(0),
        ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(S.data_ptr()),
        ctypes.c_void_p(Z.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, wq.status_name(st)
    return packed, S, Z


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [wq_inputs.outlier_config(N=96, K=1024)[0],              # outlier columns
             wq_inputs.weight_bf16(300, 2048, 0.05, seed=17)]         # different range
    for Wb in cases:
        W = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
        p0, s0, z0 = _noalloc_via_c_abi(W)
        p1, s1, z1 = wq.wq_quantize_rtn_per_tensor(W)
        assert wq.wq_get_status() == 0
        assert torch.equal(p0, p1)
        assert torch.equal(s0.view(torch.int16), s1.view(torch.int16))
        assert torch.equal(z0.view(torch.int16), z1.view(torch.int16))


def test_noalloc_fp32_weights_match_the_oracle():
    """fp32 weights through the library's scratch array: codes, S and Z equal the oracle's
    per-tensor quantization bit for bit, on two calls in a row."""
    for seed, sigma in ((31, 0.02), (32, 3.0)):
        W = np.random.default_rng(seed).normal(0, sigma, (200, 1024)).astype(np.float32)
        W[7, 100] *= 40.0  # one outlier sets the tensor-wide range
        p, s_, z = _noalloc_via_c_abi(torch.from_numpy(W).cuda())
        assert wq.wq_get_status() == 0
        codes, So, Zo = oracle.quantize_rtn_asym(W.astype(np.float64), 0)
        np.testing.assert_array_equal(p.cpu().numpy(), oracle.pack_int4(codes))
        assert float(s_.float().item()) == So[0, 0] and float(z.float().item()) == Zo[0, 0]
