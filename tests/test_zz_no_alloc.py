"""The allocation-free W4A16 entry point (qspec_gemm_w4a16_noalloc).

It serves callers that cannot allocate device memory where they call (for
example code running inside a host function enqueued on a stream, or a
plugin whose host application owns all device memory), so its scratch lives
in a fixed device array inside the library.  These tests call it through the
C ABI and check it against qspec_gemm_w4a16 on the same inputs, twice in a
row (the array keeps the previous call's contents), and that sizes beyond the
array are refused, against the oracle on one shape, and that its status
query (which allocates nothing either) reports no fault after normal calls.
The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import assert_close_1e3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def _call_noalloc(qs, x, wq, ws, n, group, y):
    P = ctypes.c_void_p
    return qs.LIB.qspec_gemm_w4a16_noalloc(P(x.data_ptr()), x.shape[0], x.shape[1], P(wq.data_ptr()),
                                           P(ws.data_ptr()), n, group, P(y.data_ptr()), 0,
                                           P(torch.cuda.current_stream().cuda_stream))


def _rel(a, b):
    a = a.double()
    b = b.double()
    return float((a - b).norm() / b.norm())


@pytest.mark.parametrize("m,n,k,group", [(80, 4096, 4096, 128), (16, 12288, 4096, 128),
                                         (5, 384, 512, 64)])
def test_matches_workspace_entry_point_twice(qs, m, n, k, group):
    gi = synth.gemm_inputs("llama2_7b", m, n, k, group, stream=77)
    w = torch.from_numpy(gi.w).cuda()
    x = torch.from_numpy(gi.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    wq, ws = qs.quantize_weights(w, group)
    y_ref = qs.gemm_w4a16(x, wq, ws, group)
    torch.cuda.synchronize()
    for _ in range(2):
        y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
        assert _call_noalloc(qs, x, wq, ws, n, group, y) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(y).all()
        assert _rel(y, y_ref) <= 1e-3                 # the W4A16 output bar of the other tests
        assert torch.equal(y, y_ref)                  # same kernel, same schedule: identical bits


def test_allocates_nothing_after_setup(qs):
    m, n, k = 16, 4096, 4096
    gi = synth.gemm_inputs("llama2_7b", m, n, k, 128, stream=78)
    wq, ws = qs.quantize_weights(torch.from_numpy(gi.w).cuda(), 128)
    x = torch.from_numpy(gi.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    y = torch.empty((m, n), dtype=torch.float32, device="cuda")
    assert _call_noalloc(qs, x, wq, ws, n, 128, y) == 0      # first call: one-time set-up
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch_alloc0 = torch.cuda.memory_allocated()
    for _ in range(3):
        assert _call_noalloc(qs, x, wq, ws, n, 128, y) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0 and torch.cuda.memory_allocated() == torch_alloc0


def test_refuses_shapes_beyond_the_builtin_scratch(qs):
    m, n, k = 200, 4096, 4096          # token tile 128: split-K slots exceed 16 MiB on a 148-SM part
    x = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((n, k // 2), dtype=torch.uint8, device="cuda")
    ws = torch.zeros((n, qs.scale_row_stride(k, 128)), dtype=torch.float16, device="cuda")
    y = torch.zeros((m, n), dtype=torch.float32, device="cuda")
    assert _call_noalloc(qs, x, wq, ws, n, 128, y) == 4    # QSPEC_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert not y.any()                                       # nothing was launched


def test_matches_oracle_and_reports_clean_status(qs):
    m, n, k, group = 80, 4096, 4096, 128
    gi = synth.gemm_inputs("llama2_7b", m, n, k, group, stream=79)
    wq, ws = qs.quantize_weights(torch.from_numpy(gi.w).cuda(), group)
    x = torch.from_numpy(gi.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    y = torch.empty((m, n), dtype=torch.float32, device="cuda")
    assert _call_noalloc(qs, x, wq, ws, n, group, y) == 0
    assert qs.LIB.qspec_gemm_w4a16_noalloc_status(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    cols = np.arange(0, n, 16)
    q, s_h = orc.quantize_weights(gi.w[cols], group)
    assert_close_1e3(y.cpu().numpy()[:, cols], orc.gemm_w4a16(gi.x, q, s_h, group))
