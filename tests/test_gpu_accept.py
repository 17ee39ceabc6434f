"""GPU parity of the speculative accept / residual resample kernel: accepted
lengths and tokens identical to the oracle."""
import numpy as np
import pytest
import torch

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import cuda_f32, cuda_i32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def _run(qs, ai, work=None):
    n, tok = qs.spec_accept(cuda_f32(ai.p), cuda_f32(ai.q), cuda_i32(ai.draft),
                            cuda_f32(ai.u_acc), cuda_f32(ai.u_res), work=work)
    torch.cuda.synchronize()
    return n.cpu().numpy(), tok.cpu().numpy()


def near_ties(ai) -> int:
    """Positions where |u - p/q| < 1e-6 (reported; the exact test makes them agree anyway)."""
    b = np.arange(ai.draft.shape[0])[:, None]
    i = np.arange(ai.draft.shape[1])[None, :]
    ratio = ai.p[b, i, ai.draft].astype(np.float64) / ai.q[b, i, ai.draft].astype(np.float64)
    return int((np.abs(ai.u_acc.astype(np.float64) - ratio) < 1e-6).sum())


def test_tiny_config_identical(qs):
    ai = synth.tiny_accept_inputs()
    n, tok = _run(qs, ai)
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)


@pytest.mark.parametrize("sigma", synth.ACCEPT_SIGMAS)
def test_vocab_128256_batch_64_identical(qs, sigma):
    ai = synth.big_accept_inputs(sigma)
    n, tok = _run(qs, ai)
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    print(f"sigma={sigma}: near ties {near_ties(ai)}, mean accepted {n.mean():.3f}")
    assert np.array_equal(n, n_ref)
    assert np.array_equal(tok, tok_ref)


@pytest.mark.parametrize("b,g,v", [(1, 1, 4), (3, 16, 36), (5, 2, 1000), (130, 3, 2048)])
def test_ragged_sizes_identical(qs, b, g, v):
    ai = synth.accept_inputs(synth.rng_for("accept", 11, b, g, v), b, g, v, 1.0, 0.7)
    n, tok = _run(qs, ai)
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)


@pytest.mark.parametrize("sigma", [0.3, 3.0])
def test_largest_vocab_identical(qs, sigma):
    """The largest vocabulary the entry points accept (409600): the most blocks a warp records."""
    ai = synth.accept_inputs(synth.rng_for("accept", 18, int(10 * sigma)), 3, 4, 409600, 2.0, sigma)
    n, tok = _run(qs, ai)
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)
    p, draft = synth.greedy_inputs(synth.rng_for("accept", 19, int(10 * sigma)), ai.p, follow=0.7)
    n, tok = _run_greedy(qs, p, draft)
    n_ref, tok_ref = orc.greedy_accept(p, draft)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)


def test_exact_ratio_ties_and_extreme_uniforms(qs):
    """u * q(x) == p(x) exactly rejects (the strict reading), one ulp of u below it accepts;
    u_res = 0 and the largest float below 1 draw the first and the last token of the CDF."""
    ai = synth.accept_inputs(synth.rng_for("accept", 20), 8, 4, 64, 1.0, 0.5)
    below = np.nextafter(np.float32(0.5), np.float32(0.0))
    for b in range(8):
        for i in range(4):
            x = ai.draft[b, i]
            ai.q[b, i, x] = np.float32(0.5)
            ai.p[b, i, x] = np.float32(0.25)
            # sequences 0..3 tie at position b % 4 (reject there), accept before it
            ai.u_acc[b, i] = np.float32(0.5) if i == b % 4 else below
    ai.u_res[0::2] = np.float32(0.0)
    ai.u_res[1::2] = np.nextafter(np.float32(1.0), np.float32(0.0))
    n, tok = _run(qs, ai)
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)
    assert np.array_equal(n, np.arange(8) % 4)


def test_p_equals_q_accepts_all_and_draws_bonus(qs):
    ai = synth.accept_inputs(synth.rng_for("accept", 12), 8, 5, 5000, 2.0, 0.5)
    ai.q = ai.p[:, :5, :].copy()
    n, tok = _run(qs, ai)
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    assert np.all(n == 5) and np.array_equal(tok, tok_ref)


def test_empty_residual_falls_back_to_target_row(qs):
    ai = synth.accept_inputs(synth.rng_for("accept", 13), 4, 4, 64, 1.0, 0.5)
    ai.q = ai.p[:, :4, :].copy()
    for b in range(4):
        ai.p[b, b % 4, ai.draft[b, b % 4]] = 0.0    # forces a rejection with an empty residual
    n, tok = _run(qs, ai)
    n_ref, tok_ref = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)


def test_out_of_range_draft_is_reported(qs):
    ai = synth.tiny_accept_inputs()
    ai.draft = ai.draft.copy()
    ai.draft[1, 1] = 32                              # == vocab: invalid
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    n, tok = _run(qs, ai, work=work)
    assert n[1] <= 1
    assert qs.workspace_status(work) == 6
    assert qs.workspace_status(work) == 0           # reading clears it


# ---------------------------------------------------------------- greedy verification
def _run_greedy(qs, p, draft, work=None):
    n, tok = qs.spec_accept_greedy(cuda_f32(p), cuda_i32(draft), work=work)
    torch.cuda.synchronize()
    return n.cpu().numpy(), tok.cpu().numpy()


@pytest.mark.parametrize("sigma", synth.ACCEPT_SIGMAS)
def test_greedy_vocab_128256_batch_64_identical(qs, sigma):
    ai = synth.big_accept_inputs(sigma)
    p, draft = synth.greedy_inputs(synth.rng_for("accept", 14, int(10 * sigma)), ai.p, follow=0.8)
    n, tok = _run_greedy(qs, p, draft)
    n_ref, tok_ref = orc.greedy_accept(p, draft)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)
    assert 0 < n.mean() < 5


@pytest.mark.parametrize("b,g,v", [(1, 1, 4), (2, 4, 32), (3, 16, 36), (5, 2, 1000), (130, 3, 2048)])
def test_greedy_ragged_sizes_and_ties_identical(qs, b, g, v):
    rng = synth.rng_for("accept", 15, b, g, v)
    levels = rng.integers(0, 3, size=(b, g + 1, v)).astype(np.float32)   # many ties
    p, draft = synth.greedy_inputs(rng, levels, follow=0.7, plant_prob=0.6, top=3.0)
    n, tok = _run_greedy(qs, p, draft)
    n_ref, tok_ref = orc.greedy_accept(p, draft)
    assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref)


def test_greedy_all_match_takes_bonus_and_bad_draft_is_reported(qs):
    ai = synth.accept_inputs(synth.rng_for("accept", 16), 4, 3, 4096, 2.0, 0.5)
    p, draft = synth.greedy_inputs(synth.rng_for("accept", 17), ai.p, follow=1.0)
    n, tok = _run_greedy(qs, p, draft)
    n_ref, tok_ref = orc.greedy_accept(p, draft)
    assert np.all(n == 3) and np.array_equal(tok, tok_ref)
    draft[2, 1] = 4096                                # == vocab: invalid, never matches
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    n, tok = _run_greedy(qs, p, draft, work=work)
    n_ref, tok_ref = orc.greedy_accept(p, draft)
    assert n[2] == 1 and np.array_equal(tok, tok_ref)
    assert qs.workspace_status(work) == 6
