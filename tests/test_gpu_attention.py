"""The shared KV cache and its decode attention on the GPU against the oracle.

QSpec abstract: the drafting and the verifying stage reuse the KV cache as
well as the weights.  The cache entries the kernels write are compared bit for
bit (bf16 patterns); attention outputs element-wise against the oracle's
float64 evaluation from the same bf16 cache and fp32 queries, within the
bound of fp32 accumulation: each output sums at most n weighted values after
dot products of 128 terms, so |error| <= (n + 128) * 2^-23 * max|v| with n
the number of visible keys (first-order, worst case); the relative Frobenius
error must also stay below 1e-5.
"""
import numpy as np
import pytest
import torch

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import cuda_bf16, cuda_f32, cuda_i32, rel_fro

pytestmark = pytest.mark.gpu

D = 128
BAD_INPUT = 6            # QSPEC_ERR_BAD_INPUT


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def _f32(bits):
    return synth.bf16_bits_to_f32(bits)


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _check_attention(out: np.ndarray, ref: np.ndarray, n_max: int, v_abs_max: float):
    bound = (n_max + 128) * 2.0 ** -23 * v_abs_max
    err = np.abs(out.astype(np.float64) - ref)
    assert err.max() <= bound, (float(err.max()), bound, np.unravel_index(err.argmax(), err.shape))
    assert rel_fro(out, ref) <= 1e-5, rel_fro(out, ref)


def _pass(qs, rng, kv, kc, vc, lens_d, offset, t_new, h_q, h_kv, l_max, ctx_max, work):
    """One append + attention pass on the GPU and in the oracle; returns the new oracle caches."""
    b = len(kv.lens)
    qkv = synth.qkv_rows(rng, b * t_new, h_q, h_kv)
    qkv_d = cuda_f32(qkv)
    qs.kv_append(qkv_d, lens_d, offset, kc, vc, h_q, work=work)
    aw = torch.zeros(qs.attn_workspace_size(b, t_new, h_q, h_kv, ctx_max), dtype=torch.uint8,
                     device="cuda")
    out = qs.attn_decode(qkv_d, lens_d, offset, kc, vc, h_q, ctx_max, work=aw)
    ref_k, ref_v = orc.kv_append(_f32(kv.k_bits), _f32(kv.v_bits), qkv, kv.lens, offset, t_new,
                                 h_q, h_kv, D)
    ref = orc.decode_attention(qkv, ref_k, ref_v, kv.lens, offset, t_new, h_q, h_kv, D)
    torch.cuda.synchronize()
    assert qs.workspace_status(work) == 0 and qs.workspace_status(aw) == 0
    got_k, got_v = _bits(kc), _bits(vc)
    assert np.array_equal(got_k, synth.to_bf16_bits(ref_k)), "key cache"
    assert np.array_equal(got_v, synth.to_bf16_bits(ref_v)), "value cache"
    n_max = int(kv.lens.max()) + offset + t_new
    _check_attention(out.cpu().numpy(), ref, n_max, float(np.abs(ref_v).max()))
    kv.k_bits, kv.v_bits = got_k, got_v
    return out


@pytest.mark.parametrize("b,t_new,h_q,h_kv,lens,offset,l_max,ctx_max", [
    (2, 1, 4, 4, (0, 0), 0, 8, 1),              # one key: the output is that value
    (2, 1, 4, 2, (5, 300), 2, 320, 303),        # ragged lengths, two chunks, a partial one
    (3, 5, 2, 2, (255, 1, 600), 0, 640, 605),   # verifying pass across chunk boundaries
    (2, 5, 8, 2, (17, 513), 0, 1024, 1024),     # grouped heads, 20 rows, empty trailing chunks
    (1, 2, 32, 2, (700,), 1, 768, 703),         # 32 rows per KV head (the maximum)
    (2, 4, 8, 8, (256, 511), 1, 520, 516),      # lengths on chunk edges
])
def test_append_and_attention_match_oracle(qs, b, t_new, h_q, h_kv, lens, offset, l_max, ctx_max):
    rng = synth.rng_for("tiny", 40 + b * 7 + t_new)
    kv = synth.kv_cache_inputs(rng, b, h_kv, l_max, lens)
    kc, vc = cuda_bf16(kv.k_bits), cuda_bf16(kv.v_bits)
    lens_d = cuda_i32(kv.lens)
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    _pass(qs, rng, kv, kc, vc, lens_d, offset, t_new, h_q, h_kv, l_max, ctx_max, work)


def test_draft_verify_commit_round_on_one_cache(qs):
    # gamma drafting passes (one token each, offsets 0 .. gamma-1), the verifying
    # pass over gamma + 1 tokens (offset 0, overwriting the drafts), then the
    # commit; a second round starts from the committed lengths
    gamma, b, h_q, h_kv, l_max = 4, 4, 8, 2, 1200
    rng = synth.rng_for("tiny", 61)
    kv = synth.kv_cache_inputs(rng, b, h_kv, l_max, (3, 250, 511, 900))
    kc, vc = cuda_bf16(kv.k_bits), cuda_bf16(kv.v_bits)
    lens_d = cuda_i32(kv.lens)
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    for rnd, n_acc in enumerate(((0, 4, 2, 1), (3, 0, 4, 2))):
        ctx = int(kv.lens.max()) + gamma + 1
        for j in range(gamma):
            _pass(qs, rng, kv, kc, vc, lens_d, j, 1, h_q, h_kv, l_max, ctx, work)
        _pass(qs, rng, kv, kc, vc, lens_d, 0, gamma + 1, h_q, h_kv, l_max, ctx, work)
        n_acc_d = cuda_i32(np.array(n_acc))
        qs.kv_commit(lens_d, n_acc_d, l_max, work=work)
        kv.lens = orc.kv_commit(kv.lens, n_acc).astype(np.int32)
        assert np.array_equal(lens_d.cpu().numpy(), kv.lens), rnd
        assert qs.workspace_status(work) == 0


def test_llama2_7b_decode_full_size(qs):
    # batch 16, 32 heads, context 1024 before the round: one drafting pass and
    # the verifying pass, every output against the oracle
    b, h_q, h_kv, gamma = 16, 32, 32, 4
    rng = synth.rng_for("llama2_7b", 71)
    lens = rng.integers(900, 1025, size=b)
    l_max = 1040
    kv = synth.kv_cache_inputs(rng, b, h_kv, l_max, lens)
    kc, vc = cuda_bf16(kv.k_bits), cuda_bf16(kv.v_bits)
    lens_d = cuda_i32(kv.lens)
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ctx = int(kv.lens.max()) + gamma + 1
    _pass(qs, rng, kv, kc, vc, lens_d, 0, 1, h_q, h_kv, l_max, ctx, work)
    _pass(qs, rng, kv, kc, vc, lens_d, 0, gamma + 1, h_q, h_kv, l_max, ctx, work)


def test_grouped_llama3_8b_verify_full_size(qs):
    b, (h_q, h_kv), gamma = 8, synth.LLAMA3_8B_ATTN, 4
    rng = synth.rng_for("llama3_8b", 72)
    lens = rng.integers(1500, 2049, size=b)
    l_max = 2064
    kv = synth.kv_cache_inputs(rng, b, h_kv, l_max, lens)
    kc, vc = cuda_bf16(kv.k_bits), cuda_bf16(kv.v_bits)
    lens_d = cuda_i32(kv.lens)
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    _pass(qs, rng, kv, kc, vc, lens_d, 0, gamma + 1, h_q, h_kv, l_max, int(kv.lens.max()) + gamma + 1,
          work)


def test_repeat_calls_are_identical_and_the_workspace_recovers(qs):
    b, h_q, h_kv, t_new, l_max = 3, 8, 2, 5, 2048
    rng = synth.rng_for("tiny", 81)
    kv = synth.kv_cache_inputs(rng, b, h_kv, l_max, (2000, 40, 1300))
    kc, vc = cuda_bf16(kv.k_bits), cuda_bf16(kv.v_bits)
    lens_d = cuda_i32(kv.lens)
    qkv = cuda_f32(synth.qkv_rows(rng, b * t_new, h_q, h_kv))
    work = torch.zeros(qs.attn_workspace_size(b, t_new, h_q, h_kv, 2005), dtype=torch.uint8,
                       device="cuda")
    outs = [qs.attn_decode(qkv, lens_d, 0, kc, vc, h_q, 2005, work=work).clone() for _ in range(4)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert qs.workspace_status(work) == 0


def test_lengths_outside_the_cache_are_reported_and_write_nothing(qs):
    b, h_q, h_kv, l_max = 3, 4, 2, 64
    rng = synth.rng_for("tiny", 91)
    kv = synth.kv_cache_inputs(rng, b, h_kv, l_max, (10, 63, -1))   # 63 + 1 is outside; -1 invalid
    kc, vc = cuda_bf16(kv.k_bits), cuda_bf16(kv.v_bits)
    lens_d = cuda_i32(kv.lens)
    qkv = cuda_f32(synth.qkv_rows(rng, b * 2, h_q, h_kv))
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    qs.kv_append(qkv, lens_d, 0, kc, vc, h_q, work=work)
    torch.cuda.synchronize()
    assert qs.workspace_status(work) == BAD_INPUT
    k_after = _bits(kc)
    # sequence 0 written at 10 and 11; sequence 1 at 63 only; sequence 2 untouched
    assert np.array_equal(k_after[2], kv.k_bits[2])
    assert np.array_equal(k_after[1, :, :63], kv.k_bits[1, :, :63])
    assert not np.array_equal(k_after[1, :, 63], kv.k_bits[1, :, 63])
    assert np.array_equal(k_after[0, :, 12:], kv.k_bits[0, :, 12:])
    aw = torch.zeros(qs.attn_workspace_size(b, 2, h_q, h_kv, 64), dtype=torch.uint8, device="cuda")
    out = qs.attn_decode(qkv, lens_d, 0, kc, vc, h_q, 64, work=aw)
    torch.cuda.synchronize()
    assert qs.workspace_status(aw) == BAD_INPUT
    o = out.cpu().numpy().reshape(b, 2, h_q * D)
    assert np.all(o[1] == 0) and np.all(o[2] == 0)          # past the context: zero output
    assert np.all(np.isfinite(o[0])) and np.any(o[0] != 0)
    # the same workspace serves a valid call afterwards
    lens_ok = cuda_i32(np.array([10, 20, 30]))
    again = qs.attn_decode(qkv, lens_ok, 0, kc, vc, h_q, 64, work=aw)
    torch.cuda.synchronize()
    assert qs.workspace_status(aw) == 0 and np.all(np.isfinite(again.cpu().numpy()))
    wk = torch.zeros(256, dtype=torch.uint8, device="cuda")
    lens2 = cuda_i32(np.array([10, 63, 5]))
    qs.kv_commit(lens2, cuda_i32(np.array([3, 0, 0])), l_max, work=wk)
    torch.cuda.synchronize()
    assert lens2.cpu().tolist() == [14, 64, 6] and qs.workspace_status(wk) == 0
    qs.kv_commit(lens2, cuda_i32(np.array([-1, 0, 1])), l_max, work=wk)
    torch.cuda.synchronize()
    assert qs.workspace_status(wk) == BAD_INPUT
    assert lens2.cpu().tolist() == [14, 64, 8]              # -1 and 64 + 1 > 64 leave theirs unchanged
