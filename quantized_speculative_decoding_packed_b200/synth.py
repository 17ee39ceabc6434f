"""Seeded synthetic inputs for the shared-INT4 QSpec hot path.

This module only draws random numbers and arranges them into the shapes of
the workloads; it contains none of the method's arithmetic (no quantization,
no GEMM, no acceptance rule).  Both the CUDA path and the CPU oracle are fed
from here, so the two sides always see identical bytes.

Workloads (QSpec: Speculative Decoding with Complementary Quantization
Schemes, abstract: one INT4 weight set drives a W4A4 drafter and a W4A16
verifier; the shapes below are Llama-family linear layers standing in for the
trained models, which are not available):

* ``tiny``      one linear layer M=4, K=256, N=256, group 64, plus an accept
                step with V=32, gamma=4, B=2.
* ``llama2_7b`` decode GEMMs K=4096, N in {12288, 4096, 22016}, down K=11008
                N=4096; W4A4 draft at M=16, W4A16 verify at M=80, group 128.
* ``llama3_8b`` K=4096, N in {6144, 4096, 28672}, down K=14336 N=4096,
                M in {1, 8, 32, 128, 256}, group 128.
* ``accept``    V=128256, B=64, gamma=5, draft logits = target logits plus
                N(0, sigma^2) noise, sigma in {0.1, 0.5, 1.0}.
* ``llama2_70b`` M=2048, K=8192, N in {10240, 57344}, down K=28672 N=8192,
                group 128.

Value distributions: weights N(0, 0.02^2) fp32; activations N(0, 1) with a
fixed seeded set of round(0.01 K) outlier channels (exactly 4 for the tiny
case) scaled by 20, then rounded to bf16; target/draft probabilities are
softmaxes of Gaussian logits computed in float64 and rounded to fp32;
uniforms are k / 2^24 with k a uniform 24-bit integer (exact in fp32).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

SEED_BASE = 20241015

# Linear-layer shapes (name, N, K) per model family.
LLAMA2_7B_LAYERS = (("qkv", 12288, 4096), ("o_proj", 4096, 4096),
                    ("gate_up", 22016, 4096), ("down", 4096, 11008))
LLAMA3_8B_LAYERS = (("qkv", 6144, 4096), ("o_proj", 4096, 4096),
                    ("gate_up", 28672, 4096), ("down", 4096, 14336))
LLAMA2_70B_LAYERS = (("qkv", 10240, 8192), ("gate_up", 57344, 8192),
                     ("down", 8192, 28672))
LLAMA3_8B_M_SWEEP = (1, 8, 32, 128, 256)
ACCEPT_SIGMAS = (0.1, 0.5, 1.0)

CONFIG_IDS = {"tiny": 0, "llama2_7b": 1, "llama3_8b": 2, "accept": 3,
              "llama2_70b": 4}


def rng_for(config: str, *stream: int) -> np.random.Generator:
    """One independent generator per (config, stream...) tuple."""
    ss = np.random.SeedSequence([SEED_BASE + CONFIG_IDS[config], *stream])
    return np.random.default_rng(ss)


def weights(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """fp32 [n][k] weights drawn from N(0, 0.02^2)."""
    return (rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.02))


def outlier_channels(rng: np.random.Generator, k: int, count: int | None = None) -> np.ndarray:
    if count is None:
        count = int(round(0.01 * k))
    return np.sort(rng.choice(k, size=count, replace=False))


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def activations(rng: np.random.Generator, m: int, k: int, outliers: np.ndarray) -> np.ndarray:
    """bf16 activations [m][k] as uint16 bit patterns: N(0,1), outlier channels x20."""
    x = rng.standard_normal((m, k), dtype=np.float32)
    x[:, outliers] *= np.float32(20.0)
    return to_bf16_bits(x)


def uniforms24(rng: np.random.Generator, shape) -> np.ndarray:
    """fp32 uniforms on the grid k / 2^24, k uniform in [0, 2^24)."""
    k = rng.integers(0, 1 << 24, size=shape, dtype=np.int64)
    return (k.astype(np.float64) / float(1 << 24)).astype(np.float32)


def softmax64(logits: np.ndarray) -> np.ndarray:
    z = logits - logits.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


@dataclasses.dataclass
class AcceptInputs:
    p: np.ndarray       # fp32 [B][gamma+1][V] target probabilities
    q: np.ndarray       # fp32 [B][gamma][V]   draft probabilities
    draft: np.ndarray   # int32 [B][gamma]     draft tokens (sampled from q)
    u_acc: np.ndarray   # fp32 [B][gamma]      acceptance uniforms
    u_res: np.ndarray   # fp32 [B]             residual / bonus uniform


def accept_inputs(rng: np.random.Generator, batch: int, gamma: int, vocab: int,
                  logit_std: float, noise_std: float) -> AcceptInputs:
    """Target logits ~ N(0, logit_std^2); draft logits = target + N(0, noise_std^2).

    Draft tokens are drawn from q by a float64 inverse CDF on a separate
    uniform stream (an input-generation step; the method never sees it).
    """
    lp = rng.standard_normal((batch, gamma + 1, vocab)) * logit_std
    lq = lp[:, :gamma, :] + rng.standard_normal((batch, gamma, vocab)) * noise_std
    p = softmax64(lp).astype(np.float32)
    q = softmax64(lq).astype(np.float32)
    ud = rng.random((batch, gamma))
    draft = np.empty((batch, gamma), dtype=np.int32)
    for b in range(batch):
        for i in range(gamma):
            c = np.cumsum(q[b, i].astype(np.float64))
            j = int(np.searchsorted(c, ud[b, i] * c[-1], side="right"))
            j = min(j, vocab - 1)
            while q[b, i, j] == 0.0:    # never hand the method a zero-probability draft
                j = (j + 1) % vocab
            draft[b, i] = j
    u_acc = uniforms24(rng, (batch, gamma))
    u_res = uniforms24(rng, (batch,))
    return AcceptInputs(p=p, q=q, draft=draft, u_acc=u_acc, u_res=u_res)


@dataclasses.dataclass
class GemmInputs:
    w: np.ndarray        # fp32 [N][K]
    x_bits: np.ndarray   # uint16 [M][K] bf16 bit patterns
    group: int

    @property
    def x(self) -> np.ndarray:
        return bf16_bits_to_f32(self.x_bits)


def gemm_inputs(config: str, m: int, n: int, k: int, group: int, stream: int = 0,
                n_outliers: int | None = None) -> GemmInputs:
    rng = rng_for(config, 1, stream, m, n, k)
    w = weights(rng, n, k)
    outl = outlier_channels(rng_for(config, 2, k), k, n_outliers)
    x = activations(rng, m, k, outl)
    return GemmInputs(w=w, x_bits=x, group=group)


def tiny_gemm_inputs() -> GemmInputs:
    return gemm_inputs("tiny", 4, 256, 256, 64, n_outliers=4)


def tiny_accept_inputs() -> AcceptInputs:
    return accept_inputs(rng_for("tiny", 3), batch=2, gamma=4, vocab=32,
                         logit_std=1.0, noise_std=0.5)


def big_accept_inputs(sigma: float, batch: int = 64, gamma: int = 5,
                      vocab: int = 128256) -> AcceptInputs:
    idx = ACCEPT_SIGMAS.index(sigma) if sigma in ACCEPT_SIGMAS else 99
    return accept_inputs(rng_for("accept", 3, idx, batch, vocab), batch=batch, gamma=gamma,
                         vocab=vocab, logit_std=2.0, noise_std=sigma)


def layer_weights(config: str, n: int, k: int, stream: int = 0) -> np.ndarray:
    """fp32 [n][k] weights of one linear layer of a workload, N(0, 0.02^2)."""
    return weights(rng_for(config, 4, stream, n, k), n, k)


def layer_activations(config: str, m: int, k: int, stream: int = 0) -> np.ndarray:
    """bf16 bit patterns [m][k] of a layer's input: N(0, 1), round(0.01 k) outlier channels x20."""
    outl = outlier_channels(rng_for(config, 2, k), k)
    return activations(rng_for(config, 5, stream, m, k), m, k, outl)


def layer_weights_cuda(config: str, n: int, k: int, stream: int = 0, device="cuda") -> torch.Tensor:
    """fp32 [n][k] N(0, 0.02^2) weights drawn on the device by a seeded torch
    generator (for the large shapes, where drawing on the host is slow).  The
    host-side checks read back the rows they sample."""
    seed = int(np.random.SeedSequence([SEED_BASE + CONFIG_IDS[config], 6, stream, n, k])
               .generate_state(1, dtype=np.uint64)[0] >> 1)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn((n, k), generator=gen, device=device, dtype=torch.float32) * 0.02


def greedy_inputs(rng: np.random.Generator, p: np.ndarray, follow: float = 0.8,
                  plant_prob: float = 1.0, top: float = 2.0):
    """Inputs for the greedy rule built without ranking anything: in each row
    (with probability plant_prob) one uniformly drawn token is planted with the
    value `top`, larger than every other entry; the draft copies the row's
    planted token with probability `follow`, else takes a uniformly drawn token.
    Returns (p with the planted values, int32 drafts [B][gamma])."""
    p = p.copy()
    bsz, g1, vocab = p.shape
    planted = rng.integers(0, vocab, size=(bsz, g1))
    mask = rng.random((bsz, g1)) < plant_prob
    b_idx, i_idx = np.nonzero(mask)
    p[b_idx, i_idx, planted[b_idx, i_idx]] = np.float32(top)
    other = rng.integers(0, vocab, size=(bsz, g1 - 1))
    keep = rng.random((bsz, g1 - 1)) < follow
    draft = np.where(keep, planted[:, :g1 - 1], other).astype(np.int32)
    return p, draft


# ---------------------------------------------------------------- shared KV cache
# Decode attention of Llama-2-7B (32 heads, head dim 128, no grouping) and of
# the grouped Llama-3-8B layout (32 query heads over 8 KV heads): cached keys
# and values N(0, 1) rounded to bf16, and fused-QKV rows N(0, 1) in fp32 (a
# projection output).  Positions past each sequence's length hold values too
# (stale entries of rejected drafts), so a kernel that reads past the causal
# limit gets a different answer.
LLAMA2_7B_ATTN = (32, 32)          # (query heads, KV heads)
LLAMA3_8B_ATTN = (32, 8)
HEAD_DIM = 128


@dataclasses.dataclass
class KVInputs:
    k_bits: np.ndarray      # uint16 [B][H_kv][L_max][128]
    v_bits: np.ndarray
    lens: np.ndarray        # int32 [B]


def kv_cache_inputs(rng: np.random.Generator, batch: int, h_kv: int, l_max: int,
                    lens) -> KVInputs:
    shape = (batch, h_kv, l_max, HEAD_DIM)
    k = to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))
    v = to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))
    return KVInputs(k, v, np.asarray(lens, dtype=np.int32))


def qkv_rows(rng: np.random.Generator, rows: int, h_q: int, h_kv: int) -> np.ndarray:
    """fp32 [rows][(h_q + 2 h_kv) * 128]: query heads, key heads, value heads."""
    return rng.standard_normal((rows, (h_q + 2 * h_kv) * HEAD_DIM), dtype=np.float32)
