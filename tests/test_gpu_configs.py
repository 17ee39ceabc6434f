"""GPU parity on every linear-layer shape of the Llama-3-8B sweep and the
Llama-2-70B large-M workload, both GEMM modes, against the oracle.

Outputs are compared on sampled columns (and, at M = 2048, sampled rows):
the oracle computes each sampled output from the same quantized weights and
activations.  At M = 2048 the W4A4 per-group int32 accumulators are also
dumped for one 1024-column slice of the weights and compared bit-exactly.
"""
import numpy as np
import pytest
import torch

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import assert_close_1e3, cuda_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def _layer(qs, config, n, k, si):
    w = synth.layer_weights_cuda(config, n, k, stream=si)
    wq, ws = qs.quantize_weights(w, 128)
    return w, wq, ws


@pytest.mark.parametrize("si,name,n,k", [(i,) + s for i, s in enumerate(synth.LLAMA3_8B_LAYERS)])
def test_llama3_8b_every_shape_and_m(qs, si, name, n, k):
    w, wq, ws = _layer(qs, "llama3_8b", n, k, si)
    cols = np.sort(synth.rng_for("llama3_8b", 9, si).choice(n, size=128, replace=False))
    w_cols = w[torch.from_numpy(cols).cuda()].cpu().numpy()
    del w
    q, s_h = orc.quantize_weights(w_cols, 128)
    for m in synth.LLAMA3_8B_M_SWEEP:
        bits = synth.layer_activations("llama3_8b", m, k, stream=si)
        x = cuda_bf16(bits)
        xf = synth.bf16_bits_to_f32(bits)
        y4 = qs.gemm_w4a4(x, wq, ws, 128)
        y16 = qs.gemm_w4a16(x, wq, ws, 128)
        torch.cuda.synchronize()
        assert_close_1e3(y4.cpu().numpy()[:, cols], orc.gemm_w4a4(xf, q, s_h, 128))
        assert_close_1e3(y16.cpu().numpy()[:, cols], orc.gemm_w4a16(xf, q, s_h, 128))


@pytest.mark.parametrize("si,name,n,k", [(i,) + s for i, s in enumerate(synth.LLAMA2_70B_LAYERS)])
def test_llama2_70b_every_shape_m2048(qs, si, name, n, k):
    m = 2048
    w, wq, ws = _layer(qs, "llama2_70b", n, k, si)
    rng = synth.rng_for("llama2_70b", 9, si)
    rows = np.sort(rng.choice(m, size=64, replace=False))
    cols = np.sort(rng.choice(n, size=64, replace=False))
    w_cols = w[torch.from_numpy(cols).cuda()].cpu().numpy()
    # 1024 consecutive weight rows for the accumulator dump
    n0 = int(rng.integers(0, n // 1024)) * 1024
    w_slice = w[n0:n0 + 1024].cpu().numpy()
    del w
    bits = synth.layer_activations("llama2_70b", m, k, stream=si)
    x = cuda_bf16(bits)
    xs = synth.bf16_bits_to_f32(bits[rows])
    q, s_h = orc.quantize_weights(w_cols, 128)
    y4 = qs.gemm_w4a4(x, wq, ws, 128)
    y16 = qs.gemm_w4a16(x, wq, ws, 128)
    torch.cuda.synchronize()
    # the W4A4 reference quantizes each sampled row on its own, as the kernel does
    assert_close_1e3(y4.cpu().numpy()[np.ix_(rows, cols)], orc.gemm_w4a4(xs, q, s_h, 128))
    assert_close_1e3(y16.cpu().numpy()[np.ix_(rows, cols)], orc.gemm_w4a16(xs, q, s_h, 128))
    del y4, y16

    # accumulator dump on the slice: a GEMM over rows n0 .. n0+1023 of the same weights
    dbg = torch.zeros((m, 1024, k // 128), dtype=torch.int32, device="cuda")
    qs.gemm_w4a4(x, wq[n0:n0 + 1024], ws[n0:n0 + 1024], 128, dbg_acc=dbg)
    torch.cuda.synchronize()
    got = dbg[torch.from_numpy(rows).cuda()].cpu().numpy()
    del dbg
    q_sl, _ = orc.quantize_weights(w_slice, 128)
    qa, _ = orc.quant_act(xs)
    assert np.array_equal(got, orc.gemm_w4a4_acc(qa, q_sl, 128))
