"""Pins for the CPU oracle, against things other than the oracle itself.

Each test checks one oracle function against brute force on tiny inputs, a
closed form, an invariant, a special case with a known answer, or exact
rational enumeration, chosen so that a dropped term, a wrong sign or index or
a transposed operand in the oracle fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TIE_TOL = 2.0 ** -20


def _half_even(fr: Fraction) -> int:
    """Round an exact rational to the nearest integer, ties to even."""
    fl = math.floor(fr)
    d = fr - fl
    if d > Fraction(1, 2):
        return fl + 1
    if d < Fraction(1, 2):
        return fl
    return fl if fl % 2 == 0 else fl + 1


def _near_half(fr: Fraction) -> bool:
    d = abs((fr - math.floor(fr)) - Fraction(1, 2))
    return d <= abs(fr) * TIE_TOL + Fraction(1, 1 << 40)


# ---------------------------------------------------------------- weights
def test_hand_worked_quantization_fixture():
    fields = {}
    with open(os.path.join(GOLDEN, "quantize_row_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, *vals = line.split()
            fields[key] = vals
    group = int(fields["group"][0])
    w = np.array([float(v) for v in fields["w"]], dtype=np.float32)[None, :]
    q, s_h = orc.quantize_weights(w, group)
    assert q[0].tolist() == [int(v) for v in fields["q"]]
    assert int(s_h.view(np.uint16)[0, 0]) == int(fields["s_h_bits"][0], 16)
    assert orc.pack_int4(q)[0].tolist() == [int(v, 16) for v in fields["bytes"]]


def test_quantize_matches_brute_force_nearest_level():
    gi = synth.tiny_gemm_inputs()
    q, s_h = orc.quantize_weights(gi.w, gi.group)
    n, k = gi.w.shape
    s_full = np.repeat(s_h.astype(np.float64), gi.group, axis=1)
    w64 = gi.w.astype(np.float64)
    levels = np.arange(-8, 8, dtype=np.float64)
    # float64 differences of these fp32/fp16-derived values are exact
    err = np.abs(levels[None, None, :] * s_full[:, :, None] - w64[:, :, None])
    best = err.min(axis=2, keepdims=True)
    cand = err == best
    # ties: the even level wins
    even = (np.arange(-8, 8) % 2 == 0)[None, None, :]
    pick = np.where(cand.sum(axis=2) > 1,
                    np.argmax(cand & even, axis=2), np.argmax(cand, axis=2)) - 8
    mismatch = np.argwhere(pick != q)
    for (i, j) in mismatch:   # allowed only where the fp32 quotient sits on a half-integer
        assert _near_half(Fraction(float(gi.w[i, j])) / Fraction(float(s_h[i, j // gi.group])))
    assert len(mismatch) <= 2


def test_quantize_error_bound_and_absmax_maps_to_seven():
    gi = synth.gemm_inputs("llama2_7b", 1, 512, 1024, 128)
    q, s_h = orc.quantize_weights(gi.w, 128)
    deq = orc.dequantize(q, s_h, 128)
    s_full = np.repeat(s_h.astype(np.float64), 128, axis=1)
    assert np.all(np.abs(deq - gi.w.astype(np.float64)) <= s_full / 2 * (1 + 2.0 ** -20))
    wg = gi.w.reshape(512, 8, 128)
    arg = np.abs(wg).argmax(axis=2)
    qg = q.reshape(512, 8, 128)
    top = np.take_along_axis(qg, arg[:, :, None], axis=2)[:, :, 0]
    sign = np.sign(np.take_along_axis(wg, arg[:, :, None], axis=2)[:, :, 0])
    assert np.all(top == 7 * sign)
    assert q.min() >= -8 and q.max() <= 7


def test_quantize_exact_grid_reconstructs_and_zero_group():
    rng = np.random.default_rng(5)
    c = 2.0 ** -6
    lv = rng.integers(-7, 8, size=(3, 256))
    lv[:, 0] = 7
    lv[:, 128] = -7
    w = (lv * c).astype(np.float32)
    w[2, 128:] = 0.0                         # one all-zero group
    q, s_h = orc.quantize_weights(w, 128)
    expect = lv.copy()
    expect[2, 128:] = 0
    assert np.array_equal(q, expect)
    assert s_h[0, 0] == np.float16(c) and s_h[1, 1] == np.float16(c)
    assert s_h[2, 1] == 0
    assert np.array_equal(orc.dequantize(q, s_h, 128), expect * c)


def test_quantize_deterministic_and_pack_roundtrip():
    gi = synth.tiny_gemm_inputs()
    q1, s1 = orc.quantize_weights(gi.w, 64)
    q2, s2 = orc.quantize_weights(gi.w.copy(), 64)
    b1 = orc.pack_int4(q1)
    assert np.array_equal(b1, orc.pack_int4(q2)) and np.array_equal(s1.view(np.uint16), s2.view(np.uint16))
    assert np.array_equal(orc.unpack_int4(b1), q1)
    # independent byte decode: low nibble = even k, high nibble = odd k
    b = int(b1[3, 7])
    lo, hi = b & 15, b >> 4
    assert (lo - 16 if lo >= 8 else lo) == q1[3, 14]
    assert (hi - 16 if hi >= 8 else hi) == q1[3, 15]


# ---------------------------------------------------------------- activations
def test_quant_act_brute_force_and_special_rows():
    gi = synth.tiny_gemm_inputs()
    x = gi.x.copy()
    x[3, :] = 0.0                            # zero row
    q, s_a = orc.quant_act(x)
    assert s_a[3] == 0 and np.all(q[3] == 0)
    for m in range(3):
        a = Fraction(float(np.abs(x[m]).max()))
        assert s_a[m] == np.float32(float(a) / 7.0) or abs(float(s_a[m]) - float(a) / 7) < 1e-12
        j = int(np.abs(x[m]).argmax())
        assert q[m, j] == (7 if x[m, j] > 0 else -7)
        for k in range(x.shape[1]):
            exact = Fraction(float(x[m, k])) * 7 / a
            want = max(-8, min(7, _half_even(exact)))
            if want != q[m, k]:
                assert _near_half(exact)
    assert q.min() >= -8 and q.max() <= 7


# ---------------------------------------------------------------- W4A4
def _decode_nibble(byte_row, k):
    v = (int(byte_row[k // 2]) >> (4 * (k & 1))) & 15
    return v - 16 if v >= 8 else v


def test_w4a4_accumulators_brute_force():
    gi = synth.tiny_gemm_inputs()
    qw, s_h = orc.quantize_weights(gi.w, gi.group)
    packed = orc.pack_int4(qw)
    qa, s_a = orc.quant_act(gi.x)
    y, acc = orc.gemm_w4a4(gi.x, qw, s_h, gi.group, return_acc=True)
    m_, k_ = qa.shape
    n_ = qw.shape[0]
    g_ = k_ // gi.group
    rows = [[_decode_nibble(packed[n], k) for k in range(k_)] for n in range(n_)]
    qa_l = qa.tolist()
    for m in range(m_):
        for n in range(n_):
            for g in range(g_):
                s = 0
                for k in range(g * gi.group, (g + 1) * gi.group):
                    s += qa_l[m][k] * rows[n][k]
                assert acc[m, n, g] == s
    assert np.abs(acc).max() <= 64 * gi.group
    # closed form: the grouped rescale equals the plain product of the two dequantized operands
    deq_a = qa.astype(np.float64) * s_a.astype(np.float64)[:, None]
    plain = deq_a @ orc.dequantize(qw, s_h, gi.group).T
    assert np.allclose(y, plain, rtol=1e-12, atol=1e-12 * np.abs(plain).max())
    # exact rational value of a few outputs
    for (m, n) in [(0, 0), (1, 77), (3, 255)]:
        ex = Fraction(float(s_a[m])) * sum(Fraction(float(s_h[n, g])) * int(acc[m, n, g]) for g in range(g_))
        assert abs(float(ex) - y[m, n]) <= 1e-14 * max(1.0, abs(float(ex)))


# ---------------------------------------------------------------- W4A8 draft variant
def test_quant_act8_brute_force_and_special_rows():
    gi = synth.tiny_gemm_inputs()
    x = gi.x.copy()
    x[2, :] = 0.0                            # zero row
    q, s_a = orc.quant_act8(x)
    assert s_a[2] == 0 and np.all(q[2] == 0)
    for m in (0, 1, 3):
        a = Fraction(float(np.abs(x[m]).max()))
        j = int(np.abs(x[m]).argmax())
        assert q[m, j] == (127 if x[m, j] > 0 else -127)
        for k in range(x.shape[1]):
            exact = Fraction(float(x[m, k])) * 127 / a
            want = max(-128, min(127, _half_even(exact)))
            if want != q[m, k]:
                assert _near_half(exact)
        # the 8-bit codes resolve the row 127/7 times finer than the 4-bit ones
        err8 = np.abs(q[m].astype(np.float64) * float(s_a[m]) - x[m]).max()
        assert err8 <= float(a) / 127 / 2 * (1 + 1e-6)
    assert q.min() >= -128 and q.max() <= 127


def test_w4a8_accumulators_brute_force_and_closed_form():
    gi = synth.tiny_gemm_inputs()
    qw, s_h = orc.quantize_weights(gi.w, gi.group)
    packed = orc.pack_int4(qw)
    qa, s_a = orc.quant_act8(gi.x)
    y, acc = orc.gemm_w4a8(gi.x, qw, s_h, gi.group, return_acc=True)
    rows = [[_decode_nibble(packed[n], k) for k in range(qw.shape[1])] for n in (0, 5, 200)]
    qa_l = qa.tolist()
    for m in range(qa.shape[0]):
        for ni, n in enumerate((0, 5, 200)):
            for g in range(acc.shape[2]):
                s = sum(qa_l[m][k] * rows[ni][k] for k in range(g * gi.group, (g + 1) * gi.group))
                assert acc[m, n, g] == s
    assert np.abs(acc).max() <= 128 * 8 * gi.group
    deq_a = qa.astype(np.float64) * s_a.astype(np.float64)[:, None]
    plain = deq_a @ orc.dequantize(qw, s_h, gi.group).T
    assert np.allclose(y, plain, rtol=1e-12, atol=1e-12 * np.abs(plain).max())
    # closer to the verifying mode than the 4-bit draft on the outlier-heavy inputs
    y16 = orc.gemm_w4a16(gi.x, qw, s_h, gi.group)
    y4 = orc.gemm_w4a4(gi.x, qw, s_h, gi.group)
    assert np.linalg.norm(y - y16) < 0.5 * np.linalg.norm(y4 - y16)


# ---------------------------------------------------------------- W4A16
def test_w4a16_exact_rational_and_integer_special_case():
    gi = synth.tiny_gemm_inputs()
    qw, s_h = orc.quantize_weights(gi.w, gi.group)
    y = orc.gemm_w4a16(gi.x, qw, s_h, gi.group)
    x = gi.x
    for (m, n) in [(0, 0), (2, 31), (3, 200), (1, 255)]:
        ex = sum(Fraction(float(x[m, k])) * int(qw[n, k]) * Fraction(float(s_h[n, k // gi.group]))
                 for k in range(x.shape[1]))
        assert abs(float(ex) - y[m, n]) <= 1e-12 * float(sum(abs(Fraction(float(x[m, k])) * int(qw[n, k]) * Fraction(float(s_h[n, k // gi.group]))) for k in range(x.shape[1])))
    # scale exactly 1: integer weights with absmax 7 in every group, integer activations
    rng = np.random.default_rng(11)
    lv = rng.integers(-7, 8, size=(32, 256))
    lv[:, ::64] = 7
    q1, s1 = orc.quantize_weights(lv.astype(np.float32), 64)
    assert np.all(s1 == 1) and np.array_equal(q1, lv)
    xi = rng.integers(-20, 21, size=(5, 256)).astype(np.float32)
    assert np.array_equal(orc.gemm_w4a16(xi, q1, s1, 64), xi.astype(np.int64) @ lv.T)


# ---------------------------------------------------------------- accept / resample
def _exact_inverse_cdf(r, u):
    fr = [Fraction(float(v)) for v in r]
    total = sum(fr)
    t = Fraction(float(u)) * total
    c = Fraction(0)
    for j, v in enumerate(fr):
        c += v
        if c > t:
            return j
    return len(fr) - 1


def test_fixed_point_sampler_matches_exact_inverse_cdf():
    rng = np.random.default_rng(3)
    for trial in range(40):
        v = int(rng.integers(2, 300))
        r = rng.random(v).astype(np.float32) ** 3
        r[rng.random(v) < 0.3] = 0.0
        if r.sum() == 0:
            r[0] = 1.0
        r = (r / np.float32(r.sum() * 1.0001)).astype(np.float32)   # a probability row
        u = np.float32(rng.random())
        assert orc.sample_fixed_point(r, u) == _exact_inverse_cdf(r, u)
    # u = 0 picks the first token with positive weight; u just below 1 the last one
    r = np.array([0, 0, 0.25, 0.5, 0, 0.25, 0], np.float32)
    assert orc.sample_fixed_point(r, np.float32(0.0)) == 2
    assert orc.sample_fixed_point(r, np.float32(1 - 2 ** -24)) == 5
    assert orc.sample_fixed_point(np.zeros(4, np.float32), np.float32(0.3)) is None


def test_accept_p_equals_q_accepts_everything():
    ai = synth.tiny_accept_inputs()
    q = ai.p[:, :4, :].copy()
    n, tok = orc.spec_accept(ai.p, q, ai.draft, ai.u_acc, ai.u_res)
    assert np.all(n == 4)
    for b in range(2):
        assert tok[b, :4].tolist() == ai.draft[b].tolist()
        assert tok[b, 4] == _exact_inverse_cdf(ai.p[b, 4], ai.u_res[b])


def test_accept_zero_target_probability_rejects():
    ai = synth.tiny_accept_inputs()
    p = ai.p.copy()
    q = ai.p[:, :4, :].copy()                # everything would be accepted ...
    x = ai.draft[0, 2]
    p[0, 2, x] = 0.0                         # ... except position 2 of sequence 0
    n, tok = orc.spec_accept(p, q, ai.draft, ai.u_acc, ai.u_res)
    assert n[0] == 2 and n[1] == 4
    r = np.maximum(np.float32(0), p[0, 2] - q[0, 2])
    assert not r.any()                       # residual is empty here: the draw falls back to p_n
    assert tok[0, 2] == _exact_inverse_cdf(p[0, 2], ai.u_res[0]) and tok[0, 2] != x
    assert tok[0, 3] == -1 and tok[0, 4] == -1
    assert tok[0, :2].tolist() == ai.draft[0, :2].tolist()


def test_accept_one_hot_draft():
    v = 6
    p = np.array([[[0.1, 0.2, 0.3, 0.15, 0.05, 0.2], [1 / 6] * 6]], np.float32)
    q = np.zeros((1, 1, v), np.float32)
    q[0, 0, 2] = 1.0
    draft = np.array([[2]], np.int32)
    for u, acc in [(0.29, True), (0.3, False), (0.31, False), (0.0, True)]:
        n, tok = orc.spec_accept(p, q, draft, np.array([[u]], np.float32), np.array([0.5], np.float32))
        assert (n[0] == 1) == (u < np.float32(0.3))
        if not acc:
            # residual is p with token 2 removed
            r = p[0, 0].copy()
            r[2] = 0
            assert tok[0, 0] == _exact_inverse_cdf(r, np.float32(0.5)) and tok[0, 0] != 2


def test_rule_reproduces_target_exactly_in_rationals():
    """Exact enumeration (no oracle code): accept-or-resample emits y with probability p(y)."""
    for p, q in [([Fraction(1, 2), Fraction(1, 4), Fraction(1, 8), Fraction(1, 8)],
                  [Fraction(1, 10), Fraction(6, 10), Fraction(2, 10), Fraction(1, 10)]),
                 ([Fraction(1, 3), Fraction(1, 3), Fraction(1, 3), 0, 0],
                  [Fraction(1, 5)] * 5)]:
        res = [max(Fraction(0), a - b) for a, b in zip(p, q)]
        z = sum(res)
        beta = sum(min(a, b) for a, b in zip(p, q))
        for y in range(len(p)):
            acc_y = q[y] * (min(Fraction(1), p[y] / q[y]) if q[y] > 0 else 0)
            assert acc_y + (1 - beta) * res[y] / z == p[y]


def test_oracle_emitted_distribution_matches_target_on_uniform_grids():
    """The oracle's accept + resample, driven over uniform grids, reproduces p within the grid error."""
    p = np.array([[[0.5, 0.25, 0.125, 0.125], [0.25] * 4]], np.float32)
    q = np.array([[[0.1, 0.6, 0.2, 0.1]]], np.float32)
    k1 = 1 << 12
    grid = ((np.arange(k1) + 0.5) / k1).astype(np.float32)
    emitted = np.zeros(4)
    for x in range(4):
        d = np.full((k1, 1), x, np.int32)
        acc = orc.accept_mask(np.repeat(p, k1, 0), np.repeat(q, k1, 0), d, grid[:, None])
        frac_acc = acc.mean()
        res = np.zeros(4)
        r = np.maximum(np.float32(0), p[0, 0] - q[0, 0])
        for u in grid[::16]:
            res[orc.sample_fixed_point(r, u)] += 1
        res /= res.sum()
        emitted += q[0, 0, x] * (frac_acc * np.eye(4)[x] + (1 - frac_acc) * res)
    assert np.allclose(emitted, p[0, 0], atol=4 * 16 / k1)
    # and the full routine over a coarse joint grid
    kk = 32
    g = ((np.arange(kk) + 0.5) / kk).astype(np.float32)
    ua = np.repeat(g, kk)[:, None]
    ur = np.tile(g, kk)
    counts = np.zeros(4)
    for x in range(4):
        d = np.full((kk * kk, 1), x, np.int32)
        _, tok = orc.spec_accept(np.repeat(p, kk * kk, 0), np.repeat(q, kk * kk, 0), d, ua, ur)
        counts += q[0, 0, x] * np.bincount(tok[:, 0], minlength=4) / (kk * kk)
    assert np.allclose(counts, p[0, 0], atol=4 / kk + 1e-6)


def test_mean_acceptance_matches_overlap_closed_form():
    ai = synth.big_accept_inputs(0.5, batch=64, gamma=5, vocab=8192)
    acc = orc.accept_mask(ai.p, ai.q, ai.draft, ai.u_acc)
    alpha = np.minimum(ai.p[:, :5, :].astype(np.float64), ai.q.astype(np.float64)).sum(axis=2)
    se = math.sqrt(float(np.mean(alpha * (1 - alpha))) / acc.size)
    assert abs(acc.mean() - alpha.mean()) < 4 * se + 1e-9


def test_accept_outputs_shape_and_prefix():
    ai = synth.tiny_accept_inputs()
    n, tok = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
    mask = orc.accept_mask(ai.p, ai.q, ai.draft, ai.u_acc)
    for b in range(2):
        first = int(np.argmin(mask[b])) if not mask[b].all() else 4
        assert n[b] == first
        assert tok[b, :first].tolist() == ai.draft[b, :first].tolist()
        assert 0 <= tok[b, first] < 32
        assert np.all(tok[b, first + 1:] == -1)


# ---------------------------------------------------------------- greedy verification
def _first_max(row) -> int:
    """Index of the largest entry, the lowest one among equals (plain scan)."""
    best = 0
    for j in range(1, len(row)):
        if row[j] > row[best]:
            best = j
    return best


def _greedy_brute(p, draft):
    bsz, gamma = draft.shape
    out_n, out_t = [], []
    for b in range(bsz):
        t = [_first_max(list(map(float, p[b, i]))) for i in range(gamma + 1)]
        n = 0
        while n < gamma and int(draft[b, n]) == t[n]:
            n += 1
        out_n.append(n)
        out_t.append([int(d) for d in draft[b, :n]] + [t[n]] + [-1] * (gamma - n))
    return np.array(out_n), np.array(out_t)


def test_greedy_matches_brute_force_scan():
    rng = np.random.default_rng(31)
    for trial in range(40):
        bsz, gamma, vocab = 3, int(rng.integers(1, 6)), int(rng.integers(2, 9))
        p = rng.integers(0, 4, size=(bsz, gamma + 1, vocab)).astype(np.float32)   # many ties
        t = np.array([[_first_max(list(p[b, i])) for i in range(gamma)] for b in range(bsz)])
        # drafts that follow the target for a random prefix, then may deviate
        draft = t.copy()
        for b in range(bsz):
            cut = int(rng.integers(0, gamma + 1))
            if cut < gamma:
                draft[b, cut] = int(rng.integers(0, vocab))
        n, tok = orc.greedy_accept(p, draft.astype(np.int32))
        n_ref, tok_ref = _greedy_brute(p, draft)
        assert np.array_equal(n, n_ref) and np.array_equal(tok, tok_ref), trial


def test_greedy_ties_go_to_the_lowest_index():
    p = np.zeros((1, 2, 6), dtype=np.float32)
    p[0, 0, [1, 4]] = 0.5          # tie between tokens 1 and 4
    p[0, 1, [2, 5]] = 0.5
    n, tok = orc.greedy_accept(p, np.array([[4]], dtype=np.int32))
    assert n.tolist() == [0] and tok.tolist() == [[1, -1]]
    n, tok = orc.greedy_accept(p, np.array([[1]], dtype=np.int32))
    assert n.tolist() == [1] and tok.tolist() == [[1, 2]]


def test_greedy_equals_sampling_rule_for_deterministic_models():
    """With one-hot target rows and one-hot draft rows at the draft tokens, the
    speculative sampling rule (a separately pinned function) accepts exactly
    where the draft equals the target's token and resamples that token."""
    rng = np.random.default_rng(32)
    bsz, gamma, vocab = 6, 4, 7
    t = rng.integers(0, vocab, size=(bsz, gamma + 1))
    p = np.zeros((bsz, gamma + 1, vocab), dtype=np.float32)
    for b in range(bsz):
        for i in range(gamma + 1):
            p[b, i, t[b, i]] = 1.0
    draft = t[:, :gamma].copy()
    for b in range(bsz):
        cut = b % (gamma + 1)
        if cut < gamma:
            draft[b, cut] = (t[b, cut] + 1 + b) % vocab
    q = np.zeros((bsz, gamma, vocab), dtype=np.float32)
    for b in range(bsz):
        for i in range(gamma):
            q[b, i, draft[b, i]] = 1.0
    u_acc = synth.uniforms24(rng, (bsz, gamma))
    u_res = synth.uniforms24(rng, (bsz,))
    n_s, tok_s = orc.spec_accept(p, q, draft.astype(np.int32), u_acc, u_res)
    n_g, tok_g = orc.greedy_accept(p, draft.astype(np.int32))
    assert np.array_equal(n_s, n_g) and np.array_equal(tok_s, tok_g)
    assert n_g.tolist() == [0, 1, 2, 3, 4, 0]


# ---------------------------------------------------------------- chained pass
def test_round_to_bf16_matches_a_library_conversion():
    rng = np.random.default_rng(41)
    y = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.0078125, 3.0e38]])
    got = orc.round_to_bf16(y).view(np.uint32) >> 16
    want = synth.to_bf16_bits(y.astype(np.float32)).astype(np.uint32)
    assert np.array_equal(got, want)


def test_linear_chain_is_the_composition_of_the_pinned_gemms():
    rng = np.random.default_rng(42)
    m, group = 5, 64
    shapes = [(384, 256), (256, 256), (512, 256)]   # (N, K): slices 384 -> 256, 256 -> 256, ...
    layers = []
    for (n, k) in shapes:
        w = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
        layers.append(orc.quantize_weights(w, group))
    x0 = synth.bf16_bits_to_f32(synth.to_bf16_bits(rng.standard_normal((m, 256)).astype(np.float32)))
    for mode, fn in (("w4a4", orc.gemm_w4a4), ("w4a16", orc.gemm_w4a16)):
        outs = orc.linear_chain(x0, layers, mode, group)
        x = x0
        for j, (q, s_h) in enumerate(layers):
            if j:
                # the next input: the first K columns, to fp32 then bf16 (textbook RNE on the bits)
                x = synth.bf16_bits_to_f32(synth.to_bf16_bits(outs[j - 1][:, :q.shape[1]].astype(np.float32)))
            assert np.array_equal(outs[j], fn(x, q, s_h, group)), (mode, j)
        assert outs[-1].shape == (m, 512)


# ---------------------------------------------------------------- shared KV cache, decode attention
def _kv_case(rng, b=2, t_new=3, h_q=4, h_kv=2, d=8, l_max=12, lens=(4, 7)):
    kc = synth.bf16_bits_to_f32(synth.to_bf16_bits(rng.standard_normal((b, h_kv, l_max, d)).astype(np.float32)))
    vc = synth.bf16_bits_to_f32(synth.to_bf16_bits(rng.standard_normal((b, h_kv, l_max, d)).astype(np.float32)))
    qkv = rng.standard_normal((b * t_new, (h_q + 2 * h_kv) * d)).astype(np.float32)
    return kc, vc, qkv, np.array(lens, dtype=np.int64)


def test_kv_append_places_each_column_where_the_layout_says():
    # qkv column c holds the value c (exact in bf16 below 256): the cache entry
    # of kv head g, element i must hold the column (H + g) * D + i (keys) or
    # (H + H_kv + g) * D + i (values), at position lens + offset + t only
    b, t_new, h_q, h_kv, d, l_max = 2, 2, 4, 2, 8, 10
    lens, offset = np.array([3, 6]), 1
    qkv = np.tile(np.arange((h_q + 2 * h_kv) * d, dtype=np.float32), (b * t_new, 1))
    kc = np.full((b, h_kv, l_max, d), -1.0, dtype=np.float32)
    vc = np.full((b, h_kv, l_max, d), -2.0, dtype=np.float32)
    k2, v2 = orc.kv_append(kc, vc, qkv, lens, offset, t_new, h_q, h_kv, d)
    for bb in range(b):
        for g in range(h_kv):
            for pos in range(l_max):
                written = lens[bb] + offset <= pos < lens[bb] + offset + t_new
                for i in range(d):
                    assert k2[bb, g, pos, i] == ((h_q + g) * d + i if written else -1.0)
                    assert v2[bb, g, pos, i] == ((h_q + h_kv + g) * d + i if written else -2.0)
    # values are stored rounded to bf16 (1 + 2^-9 is not a bf16 value; RNE gives 1)
    qkv2 = np.full_like(qkv, 1.0 + 2.0 ** -9)
    k3, _ = orc.kv_append(kc, vc, qkv2, lens, 0, t_new, h_q, h_kv, d)
    assert k3[0, 0, lens[0], 0] == 1.0


def test_attention_single_key_returns_its_value():
    rng = np.random.default_rng(51)
    kc, vc, qkv, _ = _kv_case(rng)
    lens = np.array([0, 0])
    out = orc.decode_attention(qkv, kc, vc, lens, 0, 1, 4, 2, 8)   # one key per row
    for b in range(2):
        for h in range(4):
            assert np.array_equal(out[b, h * 8:(h + 1) * 8], vc[b, h // 2, 0].astype(np.float64))


def test_attention_equal_scores_average_the_values():
    # identical keys (or a zero query) weight every visible position equally
    rng = np.random.default_rng(52)
    kc, vc, qkv, lens = _kv_case(rng)
    kc[:] = kc[:, :, :1, :]
    out = orc.decode_attention(qkv, kc, vc, lens, 1, 3, 4, 2, 8)
    for b in range(2):
        for t in range(3):
            n = lens[b] + 1 + t + 1
            for h in range(4):
                want = vc[b, h // 2, :n].astype(np.float64).mean(axis=0)
                assert np.allclose(out[b * 3 + t, h * 8:(h + 1) * 8], want, rtol=0, atol=1e-12)
    kc2, vc2, qkv2, lens2 = _kv_case(rng)
    qkv2[:, :4 * 8] = 0.0
    out2 = orc.decode_attention(qkv2, kc2, vc2, lens2, 0, 3, 4, 2, 8)
    assert np.allclose(out2[0, :8], vc2[0, 0, :lens2[0] + 1].astype(np.float64).mean(axis=0),
                       rtol=0, atol=1e-12)


def test_attention_two_keys_hand_worked_weights():
    # D = 4, so scores are q.k / 2.  k0 = 0 and k1 = e0 with q = 2 ln 3 e0 give
    # scores 0 and ln 3: weights 1/4 and 3/4, so the output is (v0 + 3 v1) / 4.
    d, h_q, h_kv = 4, 1, 1
    kc = np.zeros((1, 1, 2, d), dtype=np.float32)
    kc[0, 0, 1, 0] = 1.0
    vc = np.zeros((1, 1, 2, d), dtype=np.float32)
    vc[0, 0, 0] = [4.0, 0.0, -8.0, 1.0]
    vc[0, 0, 1] = [0.0, 8.0, 4.0, 1.0]
    qkv = np.zeros((1, (h_q + 2 * h_kv) * d), dtype=np.float32)
    qkv[0, 0] = 2.0 * math.log(3.0)
    out = orc.decode_attention(qkv, kc, vc, np.array([1]), 0, 1, h_q, h_kv, d)
    assert np.allclose(out[0], [1.0, 6.0, 1.0, 1.0], rtol=0, atol=1e-7)
    # the reversed query prefers k0 by the same factor
    qkv[0, 0] = -2.0 * math.log(3.0)
    out = orc.decode_attention(qkv, kc, vc, np.array([1]), 0, 1, h_q, h_kv, d)
    assert np.allclose(out[0], [3.0, 2.0, -5.0, 1.0], rtol=0, atol=1e-7)


def test_attention_is_causal_and_maps_query_heads_to_their_kv_head():
    rng = np.random.default_rng(53)
    b, t_new, h_q, h_kv, d, l_max = 2, 3, 8, 2, 8, 16
    kc, vc, qkv, lens = _kv_case(rng, b, t_new, h_q, h_kv, d, l_max, (5, 9))
    offset = 2
    out = orc.decode_attention(qkv, kc, vc, lens, offset, t_new, h_q, h_kv, d)
    # entries past each row's last visible position change nothing
    kc2, vc2 = kc.copy(), vc.copy()
    for bb in range(b):
        first_hidden = lens[bb] + offset + 1          # row t = 0 sees lens + offset + 1 keys
        kc2[bb, :, first_hidden + t_new - 1:] = 1e3
        vc2[bb, :, first_hidden + t_new - 1:] = -1e3
    out2 = orc.decode_attention(qkv, kc2, vc2, lens, offset, t_new, h_q, h_kv, d)
    assert np.array_equal(out, out2)
    # every value of KV head g equal to g: query head h must read g = h // (H / H_kv)
    vc3 = np.broadcast_to(np.arange(h_kv, dtype=np.float32)[None, :, None, None], vc.shape).copy()
    out3 = orc.decode_attention(qkv, kc, vc3, lens, offset, t_new, h_q, h_kv, d)
    for h in range(h_q):
        assert np.allclose(out3[:, h * d:(h + 1) * d], h // (h_q // h_kv), rtol=0, atol=1e-12)


def test_attention_dominant_score_selects_one_value():
    rng = np.random.default_rng(54)
    d = 8
    kc = np.zeros((1, 1, 6, d), dtype=np.float32)
    kc[0, 0, :, :] = np.eye(6, d, dtype=np.float32)      # key j = e_j
    vc = synth.bf16_bits_to_f32(synth.to_bf16_bits(rng.standard_normal((1, 1, 6, d)).astype(np.float32)))
    qkv = np.zeros((1, 3 * d), dtype=np.float32)
    qkv[0, 4] = 400.0                                      # score of key 4: 400 / sqrt(8) = 141
    out = orc.decode_attention(qkv, kc, vc, np.array([5]), 0, 1, 1, 1, d)
    assert np.allclose(out[0], vc[0, 0, 4], rtol=0, atol=1e-30)


def test_kv_commit_and_a_round_on_the_shared_cache():
    # gamma drafts append one entry each; the verifier overwrites the same
    # positions; the commit keeps the accepted drafts plus one
    rng = np.random.default_rng(55)
    b, gamma, h_q, h_kv, d, l_max = 2, 3, 2, 1, 8, 16
    lens = np.array([2, 5])
    kc = np.zeros((b, h_kv, l_max, d), dtype=np.float32)
    vc = np.zeros_like(kc)
    for j in range(gamma):
        qkv = rng.standard_normal((b, (h_q + 2 * h_kv) * d)).astype(np.float32)
        kc, vc = orc.kv_append(kc, vc, qkv, lens, j, 1, h_q, h_kv, d)
    qkv_v = rng.standard_normal((b * (gamma + 1), (h_q + 2 * h_kv) * d)).astype(np.float32)
    kc, vc = orc.kv_append(kc, vc, qkv_v, lens, 0, gamma + 1, h_q, h_kv, d)
    for bb in range(b):
        for t in range(gamma + 1):
            want = synth.bf16_bits_to_f32(synth.to_bf16_bits(qkv_v[bb * (gamma + 1) + t, h_q * d:(h_q + 1) * d]))
            assert np.array_equal(kc[bb, 0, lens[bb] + t], want)
    n_acc = np.array([0, 3])
    assert orc.kv_commit(lens, n_acc).tolist() == [3, 9]
