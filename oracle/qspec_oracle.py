"""CPU oracle for the shared-INT4 QSpec hot path.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never calls it, and this module imports nothing from the
product: the two sides share only the seeded input generators.

It is deliberately plain and slow: numpy float32 arithmetic where a decision
is taken in fp32 (IEEE-754 round-to-nearest-even, the same precision the
kernels use), float64 or exact integers/rationals for every reference value.
No blocking, fusion or reordering beyond what each definition states.

Sources.  The method is QSpec ("QSpec: Speculative Decoding with
Complementary Quantization Schemes", abstract): one set of 4-bit weights is
shared by a W4A4 drafting mode (weights and activations both quantized) and a
W4A16 verifying mode (weight-only quantization); the explainer essay on the
same paper (paragraph 4) adds that the two modes differ mainly in how the
activations are handled.  Verification follows the speculative-sampling rule
named on the SpecQuant review page (the "Leviathan rule", paragraph 5) and in
the cited titles "Fast Inference from Transformers via Speculative Decoding"
and "Accelerating Large Language Model Decoding with Speculative Sampling".
The pages print no formula, recipe or layout; the readings taken here
(symmetric INT4, group 128 along K, absmax/7 scales rounded to fp16, per-token
absmax/7 activation scales, the strict ratio test and the fixed-point residual
sampler) are listed, with reasons, in the design notes of this repository.

Parity pins for every function live in ``tests/test_oracle.py``.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

F32 = np.float32
SEVEN = F32(7.0)
FIXED_POINT_BITS = 62


# --------------------------------------------------------------------------
# Weight quantization (offline, once per model).
# QSpec abstract: both stages reuse ONE set of quantized weights.
# Recipe (a reading; the pages give none): per output channel n and group g of
# `group` consecutive input channels, s = absmax / 7 in fp32, rounded to fp16
# (RNE); q = clamp(rint(w / s_h), -8, 7) with the division in fp32 and rint
# ties-to-even; a zero scale gives q = 0.
# --------------------------------------------------------------------------
def quantize_weights(w: np.ndarray, group: int):
    """fp32 [N][K] -> (q int8 [N][K], s_h float16 [N][K/group])."""
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    assert k % group == 0
    wg = w.reshape(n, k // group, group)
    a = np.abs(wg).max(axis=2)                      # fp32 absmax per group
    s = (a / SEVEN).astype(np.float32)              # fp32 IEEE division
    s_h = s.astype(np.float16)                      # RNE to fp16
    sf = s_h.astype(np.float32)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = (wg / sf).astype(np.float32)            # fp32 IEEE division
    q = np.clip(np.rint(t), -8, 7)
    q = np.where(sf == 0, 0, q)
    return q.astype(np.int8).reshape(n, k), s_h


def pack_int4(q: np.ndarray) -> np.ndarray:
    """int8 codes [R][K] in [-8,7] -> bytes [R][K/2]; byte j holds k=2j in its
    low nibble and k=2j+1 in its high nibble (two's complement nibbles)."""
    q = np.asarray(q).astype(np.int64)
    lo = q[:, 0::2] & 0xF
    hi = q[:, 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_int4(b: np.ndarray) -> np.ndarray:
    """Inverse of pack_int4: bytes [R][K/2] -> int8 codes [R][K]."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    lo = b & 0xF
    hi = b >> 4
    r, half = b.shape
    out = np.empty((r, 2 * half), dtype=np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    out = np.where(out >= 8, out - 16, out)
    return out.astype(np.int8)


def dequantize(q: np.ndarray, s_h: np.ndarray, group: int) -> np.ndarray:
    """The dequantized weight q * s_h, exact in float64 (4-bit x 11-bit)."""
    n, k = q.shape
    s = np.repeat(s_h.astype(np.float64), group, axis=1)
    return q.astype(np.float64) * s


# --------------------------------------------------------------------------
# Per-token activation quantization for the W4A4 drafting mode.
# Explainer essay (paragraph 2): W4A4 quantizes both weights and activations
# to 4 bits.  Reading: one symmetric scale per token (row): a = max_k |x|,
# s_a = a / 7 and inv = 7 / a in fp32, q = clamp(rint(x * inv), -8, 7), the
# product x * inv rounded to fp32; a zero row gives s_a = 0 and q = 0.
# --------------------------------------------------------------------------
def quant_act(x: np.ndarray):
    """bf16-valued fp32 [M][K] -> (q int8 [M][K], s_a fp32 [M])."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        s_a = (a / SEVEN).astype(np.float32)
        inv = (SEVEN / a).astype(np.float32)
        t = (x * inv[:, None]).astype(np.float32)
    q = np.clip(np.rint(t), -8, 7)
    q = np.where((a == 0)[:, None], 0, q)
    return q.astype(np.int8), s_a


# --------------------------------------------------------------------------
# W4A4 drafting GEMM (QSpec abstract: "low-precision joint quantization for
# fast drafting").  Per group g the integer dot product
#     acc[m, n, g] = sum_{k in g} qa[m, k] * qw[n, k]
# is exact; the output is  y[m, n] = s_a[m] * sum_g s_h[n, g] * acc[m, n, g],
# evaluated here in float64.
# --------------------------------------------------------------------------
def gemm_w4a4_acc(qa: np.ndarray, qw: np.ndarray, group: int) -> np.ndarray:
    """int64 [M][N][K/group] per-group integer accumulators."""
    m, k = qa.shape
    n = qw.shape[0]
    ng = k // group
    acc = np.empty((m, n, ng), dtype=np.int64)
    a64 = qa.astype(np.int64)
    w64 = qw.astype(np.int64)
    for g in range(ng):
        sl = slice(g * group, (g + 1) * group)
        acc[:, :, g] = a64[:, sl] @ w64[:, sl].T
    return acc


def gemm_w4a4(x: np.ndarray, qw: np.ndarray, s_h: np.ndarray, group: int,
              return_acc: bool = False):
    qa, s_a = quant_act(x)
    acc = gemm_w4a4_acc(qa, qw, group)
    y = np.einsum("mng,ng->mn", acc.astype(np.float64), s_h.astype(np.float64))
    y = y * s_a.astype(np.float64)[:, None]
    if return_acc:
        return y, acc
    return y


# --------------------------------------------------------------------------
# W4A8 drafting variant: a higher-precision draft activation (the SpecQuant
# abstract's family of INT4 / FP8 / FP16 model copies; the QSpec page names
# outlier-aware activation handling as the lever on draft quality).  Reading:
# the per-token recipe of quant_act with 8-bit levels: s_a = a / 127 and
# inv = 127 / a in fp32, q = clamp(rint(x * inv), -128, 127), the product x * inv
# rounded to fp32; a zero row gives 0.  The GEMM is the W4A4 one with these codes:
#     y[m, n] = s_a[m] * sum_g s_h[n, g] * sum_{k in g} qa[m, k] * qw[n, k].
# --------------------------------------------------------------------------
S127 = F32(127.0)


def quant_act8(x: np.ndarray):
    """bf16-valued fp32 [M][K] -> (q int16 [M][K] in [-128, 127], s_a fp32 [M])."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        s_a = (a / S127).astype(np.float32)
        inv = (S127 / a).astype(np.float32)
        t = (x * inv[:, None]).astype(np.float32)
    q = np.clip(np.rint(t), -128, 127)
    q = np.where((a == 0)[:, None], 0, q)
    return q.astype(np.int16), s_a


def gemm_w4a8(x: np.ndarray, qw: np.ndarray, s_h: np.ndarray, group: int,
              return_acc: bool = False):
    qa, s_a = quant_act8(x)
    acc = gemm_w4a4_acc(qa, qw, group)
    y = np.einsum("mng,ng->mn", acc.astype(np.float64), s_h.astype(np.float64))
    y = y * s_a.astype(np.float64)[:, None]
    if return_acc:
        return y, acc
    return y


# --------------------------------------------------------------------------
# W4A16 verifying GEMM (QSpec abstract: "high-precision weight-only
# quantization for accurate verification").  y = x . (q * s_h)^T with the
# bf16 activations and the exactly dequantized weights, in float64.
# --------------------------------------------------------------------------
def gemm_w4a16(x: np.ndarray, qw: np.ndarray, s_h: np.ndarray, group: int) -> np.ndarray:
    wd = dequantize(qw, s_h, group)
    return np.asarray(x, dtype=np.float64) @ wd.T


# --------------------------------------------------------------------------
# Speculative accept / residual resample.
# SpecQuant review (paragraph 5) names the usual Leviathan rule; the titles
# "Fast Inference from Transformers via Speculative Decoding" and
# "Accelerating Large Language Model Decoding with Speculative Sampling" are
# the rule's sources.  For draft position i with draft token x:
#   accept iff u_acc * q_i(x) < p_i(x)            (strict; exact in float64)
# n = first rejected position (gamma if none).  If n < gamma the new token is
# drawn from the residual r = max(0, p_n - q_n) (fp32 subtraction), else from
# p_gamma (bonus token).  The draw uses a fixed-point inverse CDF so that any
# summation order gives the same token:
#   F_j = floor(r_j * 2^62),  C_j = sum_{i<=j} F_i,  S = C_{V-1},
#   T = floor(u_res * S)  (exact product),  token = min{ j : C_j > T }.
# If S == 0 the draw falls back to p_n (and gives -1 if that row is empty too).
# --------------------------------------------------------------------------
def accept_mask(p: np.ndarray, q: np.ndarray, draft: np.ndarray, u_acc: np.ndarray) -> np.ndarray:
    """Boolean [B][gamma]: the ratio test at every draft position."""
    b_idx = np.arange(draft.shape[0])[:, None]
    i_idx = np.arange(draft.shape[1])[None, :]
    pv = p[b_idx, i_idx, draft].astype(np.float64)
    qv = q[b_idx, i_idx, draft].astype(np.float64)
    return u_acc.astype(np.float64) * qv < pv


def fixed_point_cdf(r: np.ndarray) -> np.ndarray:
    """uint64 inclusive prefix sums of floor(r_j * 2^62).

    Domain: r is a (sub-)probability row, sum_j r_j < 3, so the sum fits in
    64 bits; target and residual rows satisfy this with room to spare.
    """
    r64 = np.asarray(r, dtype=np.float32).astype(np.float64)
    assert float(r64.sum()) < 3.0, "fixed-point CDF needs a probability row"
    f = np.floor(r64 * float(2 ** FIXED_POINT_BITS))
    f = np.maximum(f, 0.0).astype(np.uint64)
    return np.cumsum(f, dtype=np.uint64)


def fixed_point_threshold(u: float, total: int) -> int:
    """floor(u * total), exact (u is an fp32 value in [0, 1))."""
    return int(Fraction(float(np.float32(u))) * total)


def sample_fixed_point(r: np.ndarray, u: float):
    """Token drawn from weights r by the fixed-point inverse CDF, or None if sum F == 0."""
    c = fixed_point_cdf(r)
    total = int(c[-1])
    if total == 0:
        return None
    t = fixed_point_threshold(u, total)
    tok = int(np.searchsorted(c, np.uint64(t), side="right"))
    return min(tok, len(c) - 1)


def spec_accept(p: np.ndarray, q: np.ndarray, draft: np.ndarray, u_acc: np.ndarray,
                u_res: np.ndarray):
    """-> (n_accepted int32 [B], tokens int32 [B][gamma+1]; -1 pads after the new token)."""
    bsz, gamma = draft.shape
    n_acc = np.empty(bsz, dtype=np.int32)
    tokens = np.full((bsz, gamma + 1), -1, dtype=np.int32)
    for b in range(bsz):
        n = gamma
        for i in range(gamma):
            x = int(draft[b, i])
            if not (np.float64(u_acc[b, i]) * np.float64(q[b, i, x]) < np.float64(p[b, i, x])):
                n = i
                break
        if n < gamma:
            r = np.maximum(np.float32(0.0), (p[b, n] - q[b, n]).astype(np.float32))
        else:
            r = p[b, gamma]
        tok = sample_fixed_point(r, u_res[b])
        if tok is None:
            tok = sample_fixed_point(p[b, n], u_res[b])
        if tok is None:          # both rows empty (degenerate input): no token
            tok = -1
        n_acc[b] = n
        tokens[b, :n] = draft[b, :n]
        tokens[b, n] = tok
    return n_acc, tokens


# --------------------------------------------------------------------------
# Greedy verification (SpecQuant review, paragraph 5: a draft that matches in
# full is kept, and at the first mismatch the target model's own choice
# replaces the draft token).  Reading: the target's choice at position i is
# its most probable token t_i = argmax_j p[b, i, j], ties going to the lowest
# index; draft position i is accepted while draft[b, i] == t_i; n = first
# mismatch (gamma if none); the new token is t_n (the correction at the
# mismatch, or the bonus token from row gamma when every draft matched).
# --------------------------------------------------------------------------
def greedy_accept(p: np.ndarray, draft: np.ndarray):
    """-> (n_accepted int32 [B], tokens int32 [B][gamma+1]; -1 pads after the new token)."""
    bsz, gamma = draft.shape
    n_acc = np.empty(bsz, dtype=np.int32)
    tokens = np.full((bsz, gamma + 1), -1, dtype=np.int32)
    for b in range(bsz):
        n = gamma
        for i in range(gamma):
            if int(draft[b, i]) != int(np.argmax(p[b, i])):   # first maximum: lowest index
                n = i
                break
        n_acc[b] = n
        tokens[b, :n] = draft[b, :n]
        tokens[b, n] = int(np.argmax(p[b, n]))
    return n_acc, tokens


# --------------------------------------------------------------------------
# A chained pass over linear layers (the synthetic draft-verify round: QSpec
# abstract, the drafter and the verifier run the same layers on the same
# quantized weights).  Each layer's input is the previous layer's fp32 output,
# its first k columns (the next layer's input width), rounded to bf16;
# `mode` picks the GEMM of every layer.  The pages describe no model around
# the linear layers, so nothing else (attention, norms, activations) is in
# the chain.
# --------------------------------------------------------------------------
def round_to_bf16(y: np.ndarray) -> np.ndarray:
    """fp64/fp32 values -> fp32 (RN) -> bf16 (RN, ties to even), returned as fp32."""
    b = np.asarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return (b.astype(np.uint32) << 16).view(np.float32)


def linear_chain(x0: np.ndarray, layers, mode: str, group: int):
    """x0: bf16-valued fp32 [M][K0]; layers: [(q, s_h)] per GEMM in order.
    Returns the float64 output of every layer."""
    gemm = {"w4a4": gemm_w4a4, "w4a8": gemm_w4a8, "w4a16": gemm_w4a16}[mode]
    outs = []
    x = np.asarray(x0, dtype=np.float32)
    for (q, s_h) in layers:
        k = q.shape[1]
        x = round_to_bf16(outs[-1][:, :k]) if outs else x
        outs.append(gemm(x, q, s_h, group))
    return outs


# --------------------------------------------------------------------------
# The KV cache shared by the two stages (QSpec abstract: the drafter and the
# verifier reuse the KV cache as well as the weights).  The pages print no
# layout or rule; the readings taken here:
#  * one cache per layer, K and V each [B][H_kv][L_max][D], stored in bf16;
#  * a pass over T new tokens per sequence appends their keys and values at
#    positions lens[b] + offset + t (draft pass j: T = 1, offset = j; the
#    verifying pass: T = gamma + 1, offset = 0, overwriting the drafted
#    entries with the verifier's);
#  * token (b, t) then attends causally to positions 0 .. lens[b] + offset + t
#    with the textbook scaled dot-product softmax, query head h reading KV
#    head h // (H / H_kv) (grouped-query attention);
#  * after the accept step, lens[b] advances by n_accepted[b] + 1: the
#    entries past it (rejected drafts) are simply overwritten later.
# The token rows come from a fused QKV projection: row b * T + t holds the
# H query heads, then the H_kv key heads, then the H_kv value heads, D
# columns each.
# --------------------------------------------------------------------------
def kv_append(k_cache, v_cache, qkv, lens, offset: int, t_new: int, h_q: int, h_kv: int, d: int):
    """Returns copies of the caches with the T new keys/values written (bf16-rounded)."""
    k_out = np.array(k_cache, dtype=np.float32, copy=True)
    v_out = np.array(v_cache, dtype=np.float32, copy=True)
    qkv = np.asarray(qkv, dtype=np.float32)
    for b in range(len(lens)):
        for t in range(t_new):
            pos = int(lens[b]) + offset + t
            row = qkv[b * t_new + t]
            for g in range(h_kv):
                k_out[b, g, pos] = round_to_bf16(row[(h_q + g) * d:(h_q + g + 1) * d])
                v_out[b, g, pos] = round_to_bf16(row[(h_q + h_kv + g) * d:(h_q + h_kv + g + 1) * d])
    return k_out, v_out


def decode_attention(qkv, k_cache, v_cache, lens, offset: int, t_new: int, h_q: int, h_kv: int,
                     d: int) -> np.ndarray:
    """Attention output [B*T][H*D] in float64 (query values as given, cache values as stored)."""
    qkv = np.asarray(qkv, dtype=np.float64)
    kc = np.asarray(k_cache, dtype=np.float64)
    vc = np.asarray(v_cache, dtype=np.float64)
    group = h_q // h_kv
    out = np.zeros((len(lens) * t_new, h_q * d))
    for b in range(len(lens)):
        for t in range(t_new):
            n_keys = int(lens[b]) + offset + t + 1
            for h in range(h_q):
                g = h // group
                q = qkv[b * t_new + t, h * d:(h + 1) * d]
                s = kc[b, g, :n_keys] @ q / np.sqrt(d)
                w = np.exp(s - s.max())
                out[b * t_new + t, h * d:(h + 1) * d] = (w / w.sum()) @ vc[b, g, :n_keys]
    return out


def kv_commit(lens, n_accepted) -> np.ndarray:
    """Cache lengths after a round: the accepted drafts plus the token the
    verifier produced at the first rejection (or the bonus token)."""
    return np.asarray(lens, dtype=np.int64) + np.asarray(n_accepted, dtype=np.int64) + 1
