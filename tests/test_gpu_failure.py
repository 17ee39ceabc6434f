"""The GEMM's failure path, made to run on purpose without faulting the GPU.

QSPEC_GEMM_TEST_STALL makes each CTA's first pipeline wait one that nothing
completes, with a 10 ms limit: the wait runs out, every CTA gives up (abort
flag, device status, drained copies, freed tensor memory) and returns.  The
status word then reads QSPEC_ERR_TIMEOUT, reading it readies the workspace,
and the next normal call on the same workspace is bit-identical to a call on
a fresh one.
"""
import pytest
import torch

from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import cuda_bf16, cuda_f32

pytestmark = pytest.mark.gpu

TIMEOUT = 5


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


@pytest.mark.parametrize("mode,m,n,k", [("w4a4", 16, 12288, 4096), ("w4a16", 80, 4096, 11008),
                                        ("w4a4", 130, 384, 512)])
def test_stalled_wait_reports_timeout_and_workspace_recovers(qs, mode, m, n, k):
    gi = synth.gemm_inputs("llama2_7b", m, n, k, 128, stream=90)
    wq, ws = qs.quantize_weights(cuda_f32(gi.w), 128)
    x = cuda_bf16(gi.x_bits)
    fn = qs.gemm_w4a4 if mode == "w4a4" else qs.gemm_w4a16
    op = qs.OP_GEMM_W4A4 if mode == "w4a4" else qs.OP_GEMM_W4A16
    need = qs.workspace_size(op, m, n, k, 128)
    want = fn(x, wq, ws, 128, work=torch.zeros(need, dtype=torch.uint8, device="cuda")).clone()

    work = torch.zeros(need, dtype=torch.uint8, device="cuda")
    y = torch.full((m, n), float("nan"), dtype=torch.float32, device="cuda")
    fn(x, wq, ws, 128, y=y, work=work, flags=qs.GEMM_TEST_STALL)
    assert qs.workspace_status(work) == TIMEOUT
    assert not work[:256 + 4096].any()                 # status word and tickets cleared
    assert qs.workspace_status(work) == 0              # ... and the report is not repeated
    for _ in range(2):
        fn(x, wq, ws, 128, y=y, work=work)
        torch.cuda.synchronize()
        assert torch.equal(y, want)
        assert qs.workspace_status(work) == 0
