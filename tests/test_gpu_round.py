"""A chained draft-verify round on the GPU against the oracle's chain.

One Llama-2-7B-shaped layer (fused QKV -> o_proj -> gate+up -> down), run as
gamma drafting passes (W4A4 at M = 16, each pass its own seeded input) and
one verifying pass (W4A16 at M = 16 (gamma + 1)), every layer fed the
previous layer's fp32 output rounded to bf16 (by the drafting GEMMs' quantizer
as it reads it, by the library's glue kernel before the verifying GEMM), then
the accept / resample step.  The oracle runs the same chain from the same
inputs on its own.

Bars: the cast glue is bit-exact; the first GEMM of each pass meets the
element-wise 1e-3 bar of the single-GEMM tests; later GEMMs are compared by
relative Frobenius error, 1e-3 for the verifying pass and 5e-3 for the
drafting pass.  The looser drafting bar is the chain's, not a kernel's: the
GPU's fp32 sums and the oracle's float64 sums differ in the last bits, a few
inputs then round to neighbouring bf16 values, and a 4-bit activation code
occasionally lands on the other side of a rounding boundary; the oracle run
against itself with 2e-7 relative noise on each output shows the same effect
(about 1.5e-3 after four layers).  Accepted lengths and tokens are identical.
"""
import numpy as np
import pytest
import torch

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import assert_close_1e3, cuda_bf16, cuda_f32, cuda_i32, rel_fro

pytestmark = pytest.mark.gpu

GAMMA, BATCH, VOCAB = 2, 16, 32000


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def test_cast_glue_is_bit_exact(qs):
    rng = np.random.default_rng(51)
    y = (rng.standard_normal((37, 200)) * 10.0 ** rng.integers(-20, 20, (37, 200))).astype(np.float32)
    y[0, :6] = [0.0, -0.0, 1.00390625, 1.01171875, 3.0e38, -1e-40]
    x = qs.cast_bf16(cuda_f32(y), 136)
    torch.cuda.synchronize()
    got = x.view(torch.int16).cpu().numpy().view(np.uint16)
    want = (orc.round_to_bf16(y[:, :136]).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("mode", ["w4a4", "w4a8"])
@pytest.mark.parametrize("m,k,ldx,n", [(16, 4096, 12288, 1024), (5, 1024, 1028, 300), (33, 640, 640, 128)])
def test_f32_input_drafting_equals_cast_then_gemm(qs, mode, m, k, ldx, n):
    """The drafting GEMMs on a layer's fp32 output (a column slice of it) give bit-identical
    accumulators and outputs to qspec_cast_bf16 followed by the bf16-input call, and
    match the oracle's quantize-after-rounding chain."""
    rng = synth.rng_for("llama2_7b", 62, m, k, ldx)
    yprev = (rng.standard_normal((m, ldx)) * 3.0).astype(np.float32)
    yprev[:, 7] *= 40.0                                   # an outlier channel
    w = synth.layer_weights("llama2_7b", n, k, stream=63)
    wq, ws = qs.quantize_weights(cuda_f32(w), 128)
    gemm = qs.gemm_w4a4 if mode == "w4a4" else qs.gemm_w4a8
    G = k // 128
    yf = cuda_f32(yprev)
    acc_a = torch.zeros((m, n, G), dtype=torch.int32, device="cuda")
    acc_b = torch.zeros((m, n, G), dtype=torch.int32, device="cuda")
    out_a = gemm(yf[:, :k], wq, ws, 128, dbg_acc=acc_a)
    out_b = gemm(qs.cast_bf16(yf, k), wq, ws, 128, dbg_acc=acc_b)
    torch.cuda.synchronize()
    assert torch.equal(acc_a, acc_b)
    assert torch.equal(out_a.view(torch.int32), out_b.view(torch.int32))
    q_ref, s_ref = orc.quantize_weights(w, 128)
    x_ref = orc.round_to_bf16(yprev[:, :k])
    y_ref = (orc.gemm_w4a4 if mode == "w4a4" else orc.gemm_w4a8)(x_ref, q_ref, s_ref, 128)
    assert_close_1e3(out_a.cpu().numpy(), y_ref)


def test_chained_round_matches_oracle(qs):
    shapes = synth.LLAMA2_7B_LAYERS
    w_host = [synth.layer_weights("llama2_7b", n, k, stream=si) for si, (_, n, k) in enumerate(shapes)]
    dev = [qs.quantize_weights(cuda_f32(w), 128) for w in w_host]
    ref_layers = [orc.quantize_weights(w, 128) for w in w_host]
    del w_host

    passes = [("w4a4", synth.layer_activations("llama2_7b", BATCH, 4096, stream=20 + p))
              for p in range(GAMMA)]
    passes.append(("w4a16", synth.layer_activations("llama2_7b", BATCH * (GAMMA + 1), 4096, stream=30)))
    for mode, bits in passes:
        outs = qs.linear_chain(cuda_bf16(bits), dev, mode, 128)
        torch.cuda.synchronize()
        ref = orc.linear_chain(synth.bf16_bits_to_f32(bits), ref_layers, mode, 128)
        assert_close_1e3(outs[0].cpu().numpy(), ref[0])
        bar = 1e-3 if mode == "w4a16" else 5e-3
        for j in range(1, len(shapes)):
            err = rel_fro(outs[j].cpu().numpy(), ref[j])
            assert err <= bar, (mode, j, err)

    ai = synth.accept_inputs(synth.rng_for("llama2_7b", 61), BATCH, GAMMA, VOCAB, 2.0, 0.5)
    n, tok = qs.spec_accept(cuda_f32(ai.p), cuda_f32(ai.q), cuda_i32(ai.draft), cuda_f32(ai.u_acc),
                            cuda_f32(ai.u_res))
    torch.cuda.synchronize()
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    assert np.array_equal(n.cpu().numpy(), n_ref) and np.array_equal(tok.cpu().numpy(), tok_ref)
