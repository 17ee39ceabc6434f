"""GPU parity: weight and activation quantizers are bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import cuda_bf16, cuda_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def _check_weights(qs, w, group):
    wq, ws = qs.quantize_weights(cuda_f32(w), group)
    torch.cuda.synchronize()
    q, s_h = orc.quantize_weights(w, group)
    got = ws.cpu().numpy().view(np.uint16)
    g_cnt = s_h.shape[1]
    assert got.shape[1] == qs.scale_row_stride(w.shape[1], group)
    assert np.array_equal(got[:, :g_cnt], s_h.view(np.uint16))
    assert not got[:, g_cnt:].any()                    # row padding is stored as zeros
    assert np.array_equal(wq.cpu().numpy(), orc.pack_int4(q))


@pytest.mark.parametrize("n,k,group", [(256, 256, 64), (300, 384, 128), (7, 128, 64),
                                       (1, 1024, 128), (4096, 11008, 128)])
def test_quantize_weights_bit_exact(qs, n, k, group):
    w = synth.weights(synth.rng_for("llama2_7b", 7, n, k), n, k)
    _check_weights(qs, w, group)


def test_quantize_weights_full_size_gate_up(qs):
    gi = synth.gemm_inputs("llama2_7b", 1, 22016, 4096, 128)
    _check_weights(qs, gi.w, 128)


def test_quantize_weights_edge_values(qs):
    rng = np.random.default_rng(1)
    w = synth.weights(rng, 8, 256)
    w[0] = 0.0                                     # all-zero groups
    w[1, :128] *= 1e-5                             # subnormal fp16 scales
    w[2, 5] = 3.0                                  # one large outlier per group
    w[3] = np.where(np.arange(256) % 2 == 0, 1.0, -1.0).astype(np.float32) * (2.0 ** -6) * 3.5  # exact half levels
    w[4, :64] = 1e-30                              # scale underflows to zero
    _check_weights(qs, w, 64)
    _check_weights(qs, w, 128)


@pytest.mark.parametrize("m,k", [(4, 256), (17, 4096), (80, 11008), (1, 8), (3, 24)])
def test_quant_act_bit_exact(qs, m, k):
    rng = synth.rng_for("llama3_8b", 8, m, k)
    bits = synth.activations(rng, m, k, synth.outlier_channels(rng, k, max(1, k // 100)))
    x = synth.bf16_bits_to_f32(bits).copy()
    if m > 2:
        x[1] = 0.0                                 # zero row
        bits = synth.to_bf16_bits(x)
    xq, xs = qs.quant_act(cuda_bf16(bits))
    torch.cuda.synchronize()
    q, s_a = orc.quant_act(x)
    assert np.array_equal(xs.cpu().numpy().view(np.uint32), s_a.view(np.uint32))
    assert np.array_equal(xq.cpu().numpy(), orc.pack_int4(q))
