#!/usr/bin/env python
"""Benchmark of the shared-INT4 QSpec hot path on B200.

One step = one draft-verify round over the linear layers of a
Llama-2-7B-shaped decoder (32 layers x {fused QKV 12288x4096, o_proj
4096x4096, gate+up 22016x4096, down 4096x11008}, group 128), all served from
ONE packed INT4 weight set:
  * gamma = 4 drafting passes, W4A4 at M = 16 (batch 16, one token each),
  * one verifying pass, W4A16 at M = 80 (batch 16 x (gamma + 1)),
  * the accept / residual-resample step for batch 16, gamma 4, vocab 32000.
The step is captured once as a CUDA graph and replayed.  Weights (3.3 GB
packed per pass) exceed the 126 MB L2 many times over, so every pass streams
them from HBM.  Synthetic, seeded inputs; random-init weights.

Prints ONE JSON line (rank 0).  `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "shared-INT4-weight GEMM TOPS/GB/s (W4A4 draft, W4A16 verify) vs roofline"
LAYERS = (("qkv", 12288, 4096), ("o_proj", 4096, 4096), ("gate_up", 22016, 4096),
          ("down", 4096, 11008))
GROUP = 128
GAMMA = 4
BATCH = 16
M_DRAFT = BATCH
M_VERIFY = BATCH * (GAMMA + 1)
VOCAB = 32000
N_LAYERS = 32


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("qspec", "reference"), default="qspec")
    ap.add_argument("--layers", type=int, default=N_LAYERS,
                    help="decoder layers (32 = the full model; smaller only for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-large-m", action="store_true",
                    help="skip the M = 2048 (Llama-2-70B-shaped) GEMM report")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the Llama-3-8B-shaped M sweep report")
    ap.add_argument("--no-accept-report", action="store_true",
                    help="skip the vocab-128256 accept/resample report")
    ap.add_argument("--no-chained", action="store_true",
                    help="skip the chained-round report (layers fed by the previous layer)")
    ap.add_argument("--no-draft-variants", action="store_true",
                    help="skip the W4A4 / W4A8 drafting-variant report")
    ap.add_argument("--no-attention", action="store_true",
                    help="skip the shared-KV-cache decode attention report")
    ap.add_argument("--profile-attn", metavar="T", type=int, default=None,
                    help="profiling driver: three decode-attention calls over one Llama-2-7B "
                         "layer's cache (batch 16, context 1024) with T new tokens, then exit")
    ap.add_argument("--profile-accept", metavar="RULE", default=None,
                    help="profiling driver: three calls of the accept step (RULE sampling|greedy) "
                         "at vocab 128256, batch 64, gamma 5, sigma 0.5, then exit")
    ap.add_argument("--profile-gemm", metavar="MODE:SHAPE", default=None,
                    help="profiling driver: three calls of one GEMM (MODE w4a4|w4a16, SHAPE "
                         "qkv|o_proj|gate_up|down of the workload, 'decode' for all four in "
                         "turn, or 70b_qkv|70b_gate_up|70b_down at M=2048) on seeded weights, "
                         "then exit")
    return ap.parse_args()


def profile_gemm(spec):
    """Three calls of one GEMM of the workload, for a profiler to capture one of them.
    SHAPE is a Llama-2-7B layer (decode M), "decode" for each of the four Llama-2-7B
    layers in turn, or one of the Llama-2-70B layers with a "70b_" prefix (M = 2048)."""
    import torch
    from quantized_speculative_decoding_packed_b200 import qspec
    mode, spec_shape = spec.split(":")
    shapes = [name for name, _, _ in LAYERS] if spec_shape == "decode" else [spec_shape]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(0))
    fn = qspec.gemm_w4a4 if mode == "w4a4" else qspec.gemm_w4a16
    for shape in shapes:
        if shape.startswith("70b_"):
            n, k = {name: (n, k) for name, n, k in LARGE_SHAPES}[shape[4:]]
            m = LARGE_M
        else:
            n, k = {name: (n, k) for name, n, k in LAYERS}[shape]
            m = M_DRAFT if mode == "w4a4" else M_VERIFY
        w = torch.randn((n, k), generator=gen, device="cuda", dtype=torch.float32) * 0.02
        wq, ws = qspec.quantize_weights(w, GROUP)
        del w
        x = torch.randn((m, k), generator=gen, device="cuda").to(torch.bfloat16)
        for _ in range(3):
            y = fn(x, wq, ws, GROUP)
        torch.cuda.synchronize()
        print(f"{mode} {shape}: y[{m}][{n}] sum |y| = {float(y.abs().sum()):.6g}")
        del wq, ws, x, y


ATTN_BATCH, ATTN_CTX, ATTN_HEADS = 16, 1024, (32, 32)   # Llama-2-7B: 32 query heads, 32 KV heads


def attn_bytes(lens, offset, t_new, h_q, h_kv):
    """Compulsory HBM bytes of one decode-attention call: every visible key and value
    (bf16) once, the query rows read (fp32) and the outputs written (fp32)."""
    kv = sum(int(n) + offset + t_new for n in lens) * h_kv * 128 * 2 * 2
    return kv + 2 * len(lens) * t_new * h_q * 128 * 4


def append_bytes(batch, t_new, h_kv):
    """The new keys and values: read in fp32 from the QKV rows, written in bf16."""
    return batch * t_new * 2 * h_kv * 128 * (4 + 2)


def _attn_setup(torch, qspec, layers, t_max, heads=ATTN_HEADS, batch=ATTN_BATCH, ctx=ATTN_CTX,
                stream_id=0):
    from quantized_speculative_decoding_packed_b200 import synth
    h_q, h_kv = heads
    l_max = ctx + t_max + 8
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(0) + 31 + stream_id)
    caches = []
    for _ in range(layers):
        kc = torch.randn((batch, h_kv, l_max, 128), generator=gen, device="cuda").to(torch.bfloat16)
        vc = torch.randn((batch, h_kv, l_max, 128), generator=gen, device="cuda").to(torch.bfloat16)
        caches.append((kc, vc))
    lens = torch.full((batch,), ctx, dtype=torch.int32, device="cuda")
    qkv = torch.randn((batch * t_max, (h_q + 2 * h_kv) * 128), generator=gen, device="cuda")
    return caches, lens, qkv, l_max


def profile_attn(t_new):
    """Three decode-attention calls over one layer's cache, for a profiler to capture one."""
    import torch
    from quantized_speculative_decoding_packed_b200 import qspec
    caches, lens, qkv, l_max = _attn_setup(torch, qspec, 1, t_new)
    h_q, h_kv = ATTN_HEADS
    kc, vc = caches[0]
    x = qkv[: ATTN_BATCH * t_new]
    ctx = ATTN_CTX + t_new
    for _ in range(3):
        out = qspec.attn_decode(x, lens, 0, kc, vc, h_q, ctx)
    torch.cuda.synchronize()
    print(f"attention T={t_new}: sum |out| = {float(out.abs().sum()):.6g}")


def attention_report(torch, qspec, hbm):
    """Decode attention over the shared KV cache (Llama-2-7B: 32 heads of 128, batch 16,
    context 1024 at the start of the round), per layer: a drafting pass (append + attention
    of 1 token at offset 0) and the verifying pass (5 tokens); plus the grouped Llama-3-8B
    layout (32 query heads over 8 KV heads) for the verifying pass.  Device time per call in
    a CUDA graph over 4 layers' caches (1.1 GB, past L2), median of 5 replays."""
    out = {"workload": "shared KV cache, batch 16, head dim 128, context 1024 before the round",
           "timing": "CUDA graph of calls over 4 layers' caches (past L2), median of 5 replays",
           "peak_hbm_gbs": hbm}
    for name, heads, passes in (("llama2_7b", ATTN_HEADS, ((1, "draft"), (5, "verify"))),
                                ("llama3_8b_gqa", (32, 8), ((5, "verify"),))):
        h_q, h_kv = heads
        caches, lens, qkv, l_max = _attn_setup(torch, qspec, 4, 5, heads)
        lens_h = [ATTN_CTX] * ATTN_BATCH
        for t_new, label in passes:
            x = qkv[: ATTN_BATCH * t_new]
            ctx = ATTN_CTX + t_new
            o = torch.empty((ATTN_BATCH * t_new, h_q * 128), dtype=torch.float32, device="cuda")
            work = torch.zeros(qspec.attn_workspace_size(ATTN_BATCH, t_new, h_q, h_kv, ctx),
                               dtype=torch.uint8, device="cuda")
            att = [(lambda c=c: qspec.attn_decode(x, lens, 0, c[0], c[1], h_q, ctx, out=o,
                                                  work=work)) for c in caches] * 2
            app = [(lambda c=c: qspec.kv_append(x, lens, 0, c[0], c[1], h_q)) for c in caches] * 2
            t_att = _graph_time_per_call(torch, att)
            t_app = _graph_time_per_call(torch, app)
            b_att = attn_bytes(lens_h, 0, t_new, h_q, h_kv)
            b_app = append_bytes(ATTN_BATCH, t_new, h_kv)
            out[f"{name}_{label}_t{t_new}"] = {
                "h_q": h_q, "h_kv": h_kv, "t_new": t_new,
                "attn_us": t_att * 1e6, "attn_gbs": b_att / t_att / 1e9,
                "attn_frac_hbm": b_att / t_att / 1e9 / hbm, "attn_bytes": b_att,
                "append_us": t_app * 1e6, "append_gbs": b_app / t_app / 1e9}
        del caches
        torch.cuda.empty_cache()
    return out


def profile_accept(rule, batch=64, gamma=5, vocab=128256, sigma=0.5):
    """Three calls of the accept step on seeded inputs, for a profiler to capture one."""
    import torch
    from quantized_speculative_decoding_packed_b200 import qspec
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(0) + 13)
    lp = torch.randn((batch, gamma + 1, vocab), generator=gen, device="cuda", dtype=torch.float64) * 2
    lq = lp[:, :gamma] + torch.randn((batch, gamma, vocab), generator=gen, device="cuda",
                                     dtype=torch.float64) * sigma
    p = torch.softmax(lp, -1).float().contiguous()
    q = torch.softmax(lq, -1).float().contiguous()
    draft = torch.multinomial(q.reshape(-1, vocab).double(), 1, generator=gen).reshape(
        batch, gamma).to(torch.int32)
    u_acc = torch.rand((batch, gamma), generator=gen, device="cuda")
    u_res = torch.rand((batch,), generator=gen, device="cuda")
    for _ in range(3):
        if rule == "greedy":
            n, tok = qspec.spec_accept_greedy(p, draft)
        else:
            n, tok = qspec.spec_accept(p, q, draft, u_acc, u_res)
    torch.cuda.synchronize()
    print(f"accept {rule}: mean accepted {float(n.float().mean()):.3f}")


# ---------------------------------------------------------------- algorithmic bytes / ops
def gemm_bytes(m, n, k, mode):
    """Compulsory HBM bytes of one GEMM call: packed weights + fp16 scales +
    activations as the kernel reads them + fp32 output."""
    w = n * k // 2 + n * (k // GROUP) * 2
    x = m * k * (1 if mode in ("w4a4", "w4a8") else 2)   # int8 codes, or bf16
    return w + x + m * n * 4


def packed_bytes(n, k):
    return n * k // 2 + n * (k // GROUP) * 2


def accept_bytes(n_acc, gamma, vocab):
    """Per sequence: 2 gathered elements per tested position, then one row of
    p and q (rejection) or one row of p (bonus), plus the outputs."""
    total = 0
    for n in n_acc:
        tested = min(int(n) + 1, gamma)
        total += tested * 2 * 4 + (2 * vocab * 4 if n < gamma else vocab * 4) + (gamma + 2) * 4
    return total


def greedy_bytes(n_acc, gamma, vocab):
    """Per sequence (greedy rule): the draft tokens it compares, rows 0..n of p
    (the first mismatch's row, or the bonus row when all match), plus the outputs."""
    total = 0
    for n in n_acc:
        total += min(int(n) + 1, gamma) * 4 + (int(n) + 1) * vocab * 4 + (gamma + 2) * 4
    return total


def step_work(layers):
    b = 0
    ops = 0
    for (_, n, k) in LAYERS:
        b += layers * (GAMMA * gemm_bytes(M_DRAFT, n, k, "w4a4") + gemm_bytes(M_VERIFY, n, k, "w4a16"))
        ops += layers * (GAMMA * 2 * M_DRAFT * n * k + 2 * M_VERIFY * n * k)
    return b, ops


# ---------------------------------------------------------------- multi-rank plumbing
def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float over all ranks (the job time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step: float, world: int, ms_step: float) -> float:
    """Whole-job GB/s: every rank processes its own replica of the step (weak scaling)."""
    return world * bytes_per_rank_step / (ms_step * 1e-3) / 1e9


def rank_seed(rank: int) -> int:
    return 20241015 + 1000 * rank


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running (read only)."""

    def __init__(self, index):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        names = {getattr(nv, k): k for k in dir(nv) if k.startswith("nvmlClocksEventReason") or
                 k.startswith("nvmlClocksThrottleReason")}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for bit, name in names.items():
                    if isinstance(bit, int) and bit and (r & bit) == bit and bit != 0xFFFFFFFFFFFFFFFF:
                        self.reasons.add(name.replace("nvmlClocksEventReason", "").replace(
                            "nvmlClocksThrottleReason", ""))
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self._nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        reasons = sorted(r for r in self.reasons if r not in ("None", "All", "GpuIdle",
                                                              "ApplicationsClocksSetting"))
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------- CPU oracle sample
def _oracle_shape_job(job):
    """Oracle time of one layer shape on `c` sampled columns, both modes (one thread)."""
    from threadpoolctl import threadpool_limits

    from oracle import qspec_oracle as orc
    from quantized_speculative_decoding_packed_b200 import synth
    si, n, k, c, seed = job
    with threadpool_limits(limits=1):
        rng = synth.rng_for("llama2_7b", 50 + seed, si, c)
        w = synth.weights(rng, c, k)
        outl = synth.outlier_channels(synth.rng_for("llama2_7b", 2, k), k)
        x16 = synth.bf16_bits_to_f32(synth.activations(rng, M_DRAFT, k, outl))
        x80 = synth.bf16_bits_to_f32(synth.activations(rng, M_VERIFY, k, outl))
        q, s_h = orc.quantize_weights(w, GROUP)
        t0 = time.perf_counter()
        orc.gemm_w4a4(x16, q, s_h, GROUP)
        t1 = time.perf_counter()
        orc.gemm_w4a16(x80, q, s_h, GROUP)
        t2 = time.perf_counter()
    return si, t1 - t0, t2 - t1


def oracle_sample_all_cores(columns=2048, seed=0):
    """The same sample as oracle_sample, split into column blocks run by a spawn
    pool of single-threaded processes, one per host core.  The blocks' own
    times add up to the single-thread step time (scaled exactly as in
    oracle_sample); the pool's wall time against that sum is the measured
    speed-up, and the step time on all cores is the single-thread time over it."""
    import multiprocessing as mp
    cores = os.cpu_count() or 1
    jobs = []
    for si, (name, n, k) in enumerate(LAYERS):
        c = min(columns, n)
        per = max(1, -(-c // cores))
        for j in range(0, c, per):
            jobs.append((si, n, k, min(per, c - j), seed + 7 * j))
    ctx = mp.get_context("spawn")
    with ctx.Pool(cores) as pool:
        pool.map(_oracle_shape_job, [(0, 256, 256, 1, 0)] * cores)   # start and warm the workers
        t0 = time.perf_counter()
        res = pool.map(_oracle_shape_job, jobs)
        wall = time.perf_counter() - t0
    busy = sum(t4 + t16 for (_, t4, t16) in res)
    t_single = 0.0
    for si, (name, n, k) in enumerate(LAYERS):
        t4 = sum(r[1] for r in res if r[0] == si)
        t16 = sum(r[2] for r in res if r[0] == si)
        t_single += N_LAYERS * (n / min(columns, n)) * (GAMMA * t4 + t16)
    speedup = busy / wall
    desc = (f"oracle on {columns} output columns of each of the 4 layer shapes (W4A4 at M=16, "
            f"W4A16 at M=80), split into {len(jobs)} column blocks over a spawn pool of {cores} "
            f"single-threaded processes; single-thread step time (blocks' own times scaled by "
            f"N/{columns} x 32 layers x ({GAMMA} draft + 1 verify passes)) divided by the "
            f"measured pool speed-up {speedup:.2f}; accept step excluded")
    return t_single / speedup, desc, cores


def oracle_sample(columns=2048, seed=0):
    """Time the oracle on `columns` output columns of every layer shape (both
    modes) plus the full accept step; return (seconds per full step scaled
    to the bench workload, description)."""
    from threadpoolctl import threadpool_limits

    from oracle import qspec_oracle as orc
    from quantized_speculative_decoding_packed_b200 import synth

    with threadpool_limits(limits=1):
        t_step = 0.0
        for si, (name, n, k) in enumerate(LAYERS):
            c = min(columns, n)
            rng = synth.rng_for("llama2_7b", 50 + seed, si)
            w = synth.weights(rng, c, k)
            outl = synth.outlier_channels(synth.rng_for("llama2_7b", 2, k), k)
            x16 = synth.bf16_bits_to_f32(synth.activations(rng, M_DRAFT, k, outl))
            x80 = synth.bf16_bits_to_f32(synth.activations(rng, M_VERIFY, k, outl))
            q, s_h = orc.quantize_weights(w, GROUP)
            t0 = time.perf_counter()
            orc.gemm_w4a4(x16, q, s_h, GROUP)
            t1 = time.perf_counter()
            orc.gemm_w4a16(x80, q, s_h, GROUP)
            t2 = time.perf_counter()
            scale = n / c
            t_step += N_LAYERS * scale * (GAMMA * (t1 - t0) + (t2 - t1))
        ai = synth.accept_inputs(synth.rng_for("llama2_7b", 60 + seed), BATCH, GAMMA, VOCAB, 2.0, 0.5)
        t0 = time.perf_counter()
        n_acc, _ = orc.spec_accept(ai.p, ai.q, ai.draft, ai.u_acc, ai.u_res)
        t_accept = time.perf_counter() - t0
        t_step += t_accept
    desc = (f"oracle on {columns} output columns of each of the 4 layer shapes (W4A4 at M=16, "
            f"W4A16 at M=80) plus the full accept step, extrapolated to the step by N/{columns} x "
            f"32 layers x ({GAMMA} draft + 1 verify) passes; single thread")
    return t_step, desc, n_acc, t_accept


# ---------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    bytes_step, ops_step = step_work(N_LAYERS)
    times = []
    n_acc = None
    for i in range(args.warmup + args.steps):
        t, desc, n_acc, _ = oracle_sample(columns=256, seed=i)
        if i >= args.warmup:
            times.append(t)
    acc_b = accept_bytes(n_acc, GAMMA, VOCAB)
    t = sum(times) / len(times)
    value = (bytes_step + acc_b) / t / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "ms_per_step_note": "extrapolated from each step's 256-column sample of every layer "
                                "shape (x N/256 x 32 layers x 5 passes); the run itself is short",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64/f64",
            "data": "synthetic", "config": workload_config(N_LAYERS),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": desc.replace("2048", "256")},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def workload_config(layers):
    return {"workload": "Llama-2-7B-shaped decode GEMMs, one QSpec round per step: "
                        f"{layers} layers x (qkv 12288x4096, o_proj 4096x4096, gate_up 22016x4096, "
                        f"down 4096x11008), gamma={GAMMA} W4A4 draft passes at M={M_DRAFT}, one W4A16 "
                        f"verify pass at M={M_VERIFY}, accept B={BATCH} V={VOCAB}",
            "layers": layers, "group": GROUP, "gamma": GAMMA, "draft_m": M_DRAFT,
            "verify_m": M_VERIFY, "accept": {"batch": BATCH, "gamma": GAMMA, "vocab": VOCAB},
            "l2": "inputs larger than L2 (packed weights of all layers streamed every pass)",
            "parallelism": "replicas" }


# ---------------------------------------------------------------- GPU arm
def main():
    args = parse()
    if args.profile_attn:
        profile_attn(args.profile_attn)
        return
    if args.profile_gemm:
        profile_gemm(args.profile_gemm)
        return
    if args.profile_accept:
        profile_accept(args.profile_accept)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    from quantized_speculative_decoding_packed_b200 import qspec

    L = args.layers
    gen = torch.Generator(device=dev)
    gen.manual_seed(rank_seed(rank))

    # ---- one packed INT4 weight set, shared by both modes
    wq = [[None] * len(LAYERS) for _ in range(L)]
    ws = [[None] * len(LAYERS) for _ in range(L)]
    for li in range(L):
        for si, (_, n, k) in enumerate(LAYERS):
            w = torch.randn((n, k), generator=gen, device=dev, dtype=torch.float32) * 0.02
            wq[li][si], ws[li][si] = qspec.quantize_weights(w, GROUP)
            del w
    torch.cuda.synchronize()

    def acts(m, k):
        x = torch.randn((m, k), generator=gen, device=dev, dtype=torch.float32)
        idx = torch.randperm(k, generator=gen, device=dev)[: round(0.01 * k)]
        x[:, idx] *= 20.0
        return x.to(torch.bfloat16)

    x16 = [acts(M_DRAFT, k) for (_, n, k) in LAYERS]
    x80 = [acts(M_VERIFY, k) for (_, n, k) in LAYERS]
    y16 = [torch.empty((M_DRAFT, n), device=dev) for (_, n, k) in LAYERS]
    y80 = [torch.empty((M_VERIFY, n), device=dev) for (_, n, k) in LAYERS]
    need = max(max(qspec.workspace_size(qspec.OP_GEMM_W4A4, M_DRAFT, n, k, GROUP),
                   qspec.workspace_size(qspec.OP_GEMM_W4A16, M_VERIFY, n, k, GROUP))
               for (_, n, k) in LAYERS)
    work = torch.zeros(need, dtype=torch.uint8, device=dev)
    acc_work = torch.zeros(256, dtype=torch.uint8, device=dev)

    # accept inputs: p, q softmaxes of N(0, 2^2) logits, q = p-logits + N(0, 0.5^2)
    lp = torch.randn((BATCH, GAMMA + 1, VOCAB), generator=gen, device=dev, dtype=torch.float64) * 2
    lq = lp[:, :GAMMA] + torch.randn((BATCH, GAMMA, VOCAB), generator=gen, device=dev,
                                     dtype=torch.float64) * 0.5
    p = torch.softmax(lp, -1).float().contiguous()
    q = torch.softmax(lq, -1).float().contiguous()
    draft = torch.multinomial(q.reshape(-1, VOCAB).double(), 1, generator=gen).reshape(
        BATCH, GAMMA).to(torch.int32)
    u_acc = (torch.randint(0, 1 << 24, (BATCH, GAMMA), generator=gen, device=dev).double()
             / (1 << 24)).float()
    u_res = (torch.randint(0, 1 << 24, (BATCH,), generator=gen, device=dev).double()
             / (1 << 24)).float()
    n_acc = torch.empty((BATCH,), dtype=torch.int32, device=dev)
    tokens = torch.empty((BATCH, GAMMA + 1), dtype=torch.int32, device=dev)

    # Events at the section boundaries of the step only: before the first drafting pass,
    # after each pass, after the verifying pass and after the accept step.  An event node
    # between two calls ends the programmatic overlap of the second call with the first,
    # so none is placed between the calls of a section: each section is timed as it runs.
    ev = {}

    def mark(key):
        e = ev.setdefault(key, torch.cuda.Event(enable_timing=True, external=True))
        e.record()

    def step(with_events):
        if with_events:
            mark("start")
        for pss in range(GAMMA):
            for li in range(L):
                for si, (_, n, k) in enumerate(LAYERS):
                    qspec.gemm_w4a4(x16[si], wq[li][si], ws[li][si], GROUP, y=y16[si], work=work,
                                    weights_ready=True)
            if with_events:
                mark(("draft", pss))
        for li in range(L):
            for si, (_, n, k) in enumerate(LAYERS):
                qspec.gemm_w4a16(x80[si], wq[li][si], ws[li][si], GROUP, y=y80[si], work=work,
                                 weights_ready=True)
        if with_events:
            mark("verify")
        qspec.spec_accept(p, q, draft, u_acc, u_res, n_accepted=n_acc, tokens=tokens, work=acc_work)
        if with_events:
            mark("accept")

    launches_per_step = GAMMA * L * len(LAYERS) * 2 + L * len(LAYERS) + 1
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        step(False)                                  # eager first call: per-kernel setup
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream, capture_error_mode="thread_local"):
            step(True)
        for _ in range(max(args.warmup, 3)):
            graph.replay()
        stream.synchronize()
        if qspec.workspace_status(work, stream) != 0:
            raise RuntimeError("device status reported a fault during warm-up")

        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            start.record(stream)
            for _ in range(args.steps):
                graph.replay()
            end.record(stream)
            end.synchronize()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms_total = start.elapsed_time(end)
    ms_step = ms_total / args.steps
    if world > 1:
        ms_total = max_over_ranks(ms_total, dev)
        ms_step = ms_total / args.steps

    # section durations from the last timed step (ms)
    bounds = ["start"] + [("draft", pss) for pss in range(GAMMA)]
    t_pass = [ev[a].elapsed_time(ev[b]) for a, b in zip(bounds, bounds[1:])]
    t_draft = sum(t_pass)
    t_verify = ev[("draft", GAMMA - 1)].elapsed_time(ev["verify"])
    t_acc = ev["verify"].elapsed_time(ev["accept"])
    calls_pass = L * len(LAYERS)
    b_pass = L * sum(gemm_bytes(M_DRAFT, n, k, "w4a4") for (_, n, k) in LAYERS)
    b_verify = L * sum(gemm_bytes(M_VERIFY, n, k, "w4a16") for (_, n, k) in LAYERS)
    acc_b = accept_bytes(n_acc.cpu().numpy(), GAMMA, VOCAB)
    kern = {
        "drafting": {"passes": GAMMA, "calls_per_pass": calls_pass,
                     "us_per_pass": [1e3 * t for t in t_pass],
                     "us_per_call": 1e3 * t_draft / (GAMMA * calls_pass),
                     "gbs": GAMMA * b_pass / (t_draft * 1e-3) / 1e9,
                     "share_of_step": t_draft / ms_step},
        "verifying": {"calls": calls_pass, "us": 1e3 * t_verify,
                      "us_per_call": 1e3 * t_verify / calls_pass,
                      "gbs": b_verify / (t_verify * 1e-3) / 1e9,
                      "share_of_step": t_verify / ms_step},
        "accept": {"us": 1e3 * t_acc, "gbs": acc_b / (t_acc * 1e-3) / 1e9,
                   "share_of_step": t_acc / ms_step},
        "timing": "CUDA events at the section boundaries of the last timed step",
    }

    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    # Dominant kernel: the W4A4 drafting GEMM call (activation quantizer + qgemm), over
    # all its launches in the step: achieved = the drafting passes' algorithmic bytes over
    # their event-timed duration, i.e. average bytes per launch over average launch time.
    drafting_calls = GAMMA * calls_pass
    achieved = kern["drafting"]["gbs"]
    traffic, traffic_src = traffic_from_profile()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic,
                "kernel": "W4A4 drafting GEMM call (per-token quant pre-pass + "
                          "qgemm_kernel<int8,16>), M=16, all four Llama-2-7B decode shapes "
                          "(qkv, o_proj, gate_up, down) as they run back to back in the step",
                "launches_timed": drafting_calls,
                "us_per_launch": 1e3 * t_draft / drafting_calls,
                "bytes_per_launch": GAMMA * b_pass / drafting_calls,
                "traffic_source": traffic_src,
                "peak_source": "MEASURED_PEAKS.json hbm_gbs (measured)" if "hbm_gbs" in peaks
                else "fallback 6650 GB/s"}

    bytes_step, ops_step = step_work(L)
    bytes_step += acc_b
    value = job_throughput(bytes_step, world, ms_step)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(torch, stream, graph, [x16, x80], [p, q, draft, u_acc, u_res],
                          [n_acc, tokens], args.steps, bytes_step)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, desc, _, t_acc_cpu = oracle_sample()
        t_all, desc_all, cores = oracle_sample_all_cores()
        t_all += t_acc_cpu
        cpu = {"value": bytes_step / t_all / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": desc_all + "; plus the accept step on one thread",
               "single_thread": {"value": bytes_step / t_cpu / 1e9, "unit": "GB/s", "cores": 1,
                                 "sample": desc}}

    shapes_rep = None
    if rank == 0 and world == 1:
        shapes_rep = decode_shapes_report(torch, qspec, hbm_peak, wq, ws, L, x16, x80, work)
        roofline["gate_up_back_to_back"] = {
            "us_per_call": shapes_rep["gate_up"]["w4a4_us"],
            "frac": shapes_rep["gate_up"]["w4a4_frac_hbm"]}

    large = None
    if rank == 0 and world == 1 and not args.no_large_m:
        large = large_m_report(torch, qspec, peaks)
    sweep = None
    if rank == 0 and world == 1 and not args.no_sweep:
        sweep = m_sweep_report(torch, qspec, peaks)
    acc_rep = None
    if rank == 0 and world == 1 and not args.no_accept_report:
        acc_rep = accept_report(torch, qspec, peaks)
    variants = None
    if rank == 0 and world == 1 and not args.no_draft_variants:
        variants = draft_variants_report(torch, qspec, peaks)
    attn = None
    if rank == 0 and world == 1 and not args.no_attention:
        attn = attention_report(torch, qspec, hbm_peak)
    fused_ab = None
    if rank == 0 and world == 1 and not args.no_chained:
        fused_ab = fused_quant_report(torch, qspec, wq, ws, L, x16)
    chained = None
    if rank == 0 and world == 1 and not args.no_chained:
        chained = chained_round_report(torch, qspec, peaks, wq, ws, L, x16, p, q, draft, u_acc,
                                       u_res, n_acc, tokens, acc_work, bytes_step, ms_step)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "s8/bf16", "data": "synthetic (seeded), random-init weights",
                "config": workload_config(L),
                "tops": world * ops_step / (ms_step * 1e-3) / 1e12,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps,
                "clocks": clk.summary(), "kernels": kern, "decode_shapes": shapes_rep,
                "large_m": large,
                "m_sweep": sweep, "accept_large_vocab": acc_rep, "round_chained": chained,
                "draft_variants": variants, "attention": attn,
                "fused_quant_ab": fused_ab}
        print(json.dumps(line))
    if world > 1:
        del graph
        dist.destroy_process_group()


LARGE_M = 2048
LARGE_SHAPES = (("qkv", 10240, 8192), ("gate_up", 57344, 8192), ("down", 8192, 28672))


def large_m_report(torch, qspec, peaks):
    """Llama-2-70B-shaped GEMMs at M = 2048 in both modes, each timed alone (one warm-up
    call, then 3 calls between CUDA events on the launching stream), against the dense
    tensor peaks: bf16 = the measured burst figure, int8 = twice it (nominal ratio)."""
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(0) + 7)
    shapes = {}
    for name, n, k in LARGE_SHAPES:
        w = torch.randn((n, k), generator=gen, device="cuda", dtype=torch.float32) * 0.02
        wq, ws = qspec.quantize_weights(w, GROUP)
        del w
        x = torch.randn((LARGE_M, k), generator=gen, device="cuda").to(torch.bfloat16)
        y = torch.empty((LARGE_M, n), dtype=torch.float32, device="cuda")
        for mode in ("w4a4", "w4a16"):
            fn = qspec.gemm_w4a4 if mode == "w4a4" else qspec.gemm_w4a16
            op = qspec.OP_GEMM_W4A4 if mode == "w4a4" else qspec.OP_GEMM_W4A16
            work = qspec.workspace(qspec.workspace_size(op, LARGE_M, n, k, GROUP))
            fn(x, wq, ws, GROUP, y=y, work=work, weights_ready=True)
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(3):
                fn(x, wq, ws, GROUP, y=y, work=work, weights_ready=True)
            e1.record()
            e1.synchronize()
            t = e0.elapsed_time(e1) / 3 * 1e-3
            tops = 2.0 * LARGE_M * n * k / t / 1e12
            peak = bf16 * (2.0 if mode == "w4a4" else 1.0)
            shapes[f"{name}_{mode}"] = {"n": n, "k": k, "us": t * 1e6, "tops": tops,
                                        "frac": tops / peak}
        del wq, ws, x, y
    torch.cuda.empty_cache()
    return {"m": LARGE_M, "bound": "tensor", "peak_bf16_tflops": bf16, "peak_int8_tops": 2 * bf16,
            "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst, measured); int8 = 2x"
            if "bf16_tflops" in peaks else "fallback 1590 TFLOP/s; int8 = 2x",
            "shapes": shapes}


SWEEP_SHAPES = (("qkv", 6144, 4096), ("o_proj", 4096, 4096), ("gate_up", 28672, 4096),
                ("down", 4096, 14336))
SWEEP_M = (1, 8, 32, 128, 256)


def decode_shapes_report(torch, qspec, hbm, wq, ws, layers, x16, x80, work):
    """Per decode shape and mode: device time per call in a CUDA graph of the shape's calls
    over all the step's layers, back to back (the layers' weights together exceed the L2),
    as the calls run inside a drafting or verifying pass."""
    out = {}
    for si, (name, n, k) in enumerate(LAYERS):
        row = {"n": n, "k": k}
        for mode, x, m in (("w4a4", x16[si], M_DRAFT), ("w4a16", x80[si], M_VERIFY)):
            fn = qspec.gemm_w4a4 if mode == "w4a4" else qspec.gemm_w4a16
            y = torch.empty((m, n), dtype=torch.float32, device="cuda")
            calls = [(lambda li=li: fn(x, wq[li][si], ws[li][si], GROUP, y=y, work=work,
                                       weights_ready=True)) for li in range(layers)]
            t = _graph_time_per_call(torch, calls)
            b = gemm_bytes(m, n, k, mode)
            row[f"{mode}_us"] = t * 1e6
            row[f"{mode}_gbs"] = b / t / 1e9
            row[f"{mode}_frac_hbm"] = b / t / 1e9 / hbm
        out[name] = row
    out["timing"] = (f"CUDA graph of the shape's calls over {layers} layers' weights, back to "
                     "back, median of 5 replays")
    return out


def _graph_time_per_call(torch, calls, reps=5):
    """Device time per call of a CUDA graph of `calls` (a list of thunks), median of reps."""
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for c in calls:
            c()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for c in calls:
                c()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) / len(calls) * 1e-3)
    del graph
    return statistics.median(ts)


def m_sweep_report(torch, qspec, peaks):
    """Llama-3-8B-shaped GEMMs (GQA: fused QKV 6144) at M in {1, 8, 32, 128, 256}, both
    modes: device time per call in a CUDA graph of back-to-back calls whose weights
    rotate over copies that together exceed the L2 three times (weights streamed from
    HBM), with QSPEC_GEMM_WEIGHTS_READY.  Reported against both bounds: packed bytes
    over the measured HBM bandwidth, and 2MNK over the dense tensor peak (bf16 = the
    measured burst figure; int8 = twice it); `bound` names the larger time."""
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    bf16 = float(peaks.get("bf16_tflops", 1590.0))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(0) + 11)
    out = {}
    for name, n, k in SWEEP_SHAPES:
        pb = packed_bytes(n, k)
        copies = max(2, -(-3 * 126 * 2 ** 20 // pb))
        wqs = []
        for _ in range(copies):
            w = torch.randn((n, k), generator=gen, device="cuda", dtype=torch.float32) * 0.02
            wqs.append(qspec.quantize_weights(w, GROUP))
            del w
        for m in SWEEP_M:
            x = torch.randn((m, k), generator=gen, device="cuda").to(torch.bfloat16)
            y = torch.empty((m, n), dtype=torch.float32, device="cuda")
            for mode in ("w4a4", "w4a16"):
                fn = qspec.gemm_w4a4 if mode == "w4a4" else qspec.gemm_w4a16
                op = qspec.OP_GEMM_W4A4 if mode == "w4a4" else qspec.OP_GEMM_W4A16
                work = torch.zeros(qspec.workspace_size(op, m, n, k, GROUP), dtype=torch.uint8,
                                   device="cuda")
                calls = [(lambda c=c: fn(x, wqs[c][0], wqs[c][1], GROUP, y=y, work=work,
                                         weights_ready=True)) for c in range(copies)] * 2
                t = _graph_time_per_call(torch, calls)
                peak = bf16 * (2.0 if mode == "w4a4" else 1.0)
                t_hbm = gemm_bytes(m, n, k, mode) / (hbm * 1e9)
                t_tc = 2.0 * m * n * k / (peak * 1e12)
                out[f"{name}_m{m}_{mode}"] = {
                    "n": n, "k": k, "m": m, "us": t * 1e6, "packed_gbs": pb / t / 1e9,
                    "tops": 2.0 * m * n * k / t / 1e12,
                    "frac_hbm": t_hbm / t, "frac_tensor": t_tc / t,
                    "bound": "hbm" if t_hbm >= t_tc else "tensor"}
            del x, y
        del wqs
        torch.cuda.empty_cache()
    return {"workload": "Llama-3-8B-shaped GEMMs (GQA 32/8 heads), group 128",
            "timing": "CUDA graph of back-to-back calls, weights rotating past L2 (3x L2)",
            "peak_hbm_gbs": hbm, "peak_bf16_tflops": bf16, "peak_int8_tops": 2 * bf16,
            "frac": "roofline time / measured time for each bound (frac_hbm uses all compulsory "
                    "bytes: packed weights, scales, activations, output)",
            "shapes": out}


def draft_variants_report(torch, qspec, peaks):
    """The two drafting variants on the Llama-2-7B decode shapes at M = 16: W4A4 (4-bit
    per-token activation codes) and W4A8 (8-bit codes), on the same packed weights.
    Speed: device time per call in a CUDA graph of back-to-back calls over weights
    rotating past L2.  Draft quality: relative Frobenius distance of each draft's output
    from the verifying (W4A16) output on the same weights and inputs, with the inputs'
    outlier channels (x20) that make 4-bit activations lossy."""
    from quantized_speculative_decoding_packed_b200 import synth
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(0) + 19)
    out = {}
    for si, (name, n, k) in enumerate(LAYERS):
        pb = packed_bytes(n, k)
        copies = max(2, -(-3 * 126 * 2 ** 20 // pb))
        wqs = []
        for _ in range(copies):
            w = torch.randn((n, k), generator=gen, device="cuda", dtype=torch.float32) * 0.02
            wqs.append(qspec.quantize_weights(w, GROUP))
            del w
        bits = synth.layer_activations("llama2_7b", M_DRAFT, k, stream=70 + si)
        x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        y = torch.empty((M_DRAFT, n), dtype=torch.float32, device="cuda")
        ref = qspec.gemm_w4a16(x, wqs[0][0], wqs[0][1], GROUP)
        row = {"n": n, "k": k, "m": M_DRAFT}
        for mode in ("w4a4", "w4a8"):
            fn = qspec.gemm_w4a4 if mode == "w4a4" else qspec.gemm_w4a8
            op = qspec.OP_GEMM_W4A4 if mode == "w4a4" else qspec.OP_GEMM_W4A8
            work = torch.zeros(qspec.workspace_size(op, M_DRAFT, n, k, GROUP), dtype=torch.uint8,
                               device="cuda")
            calls = [(lambda c=c: fn(x, wqs[c][0], wqs[c][1], GROUP, y=y, work=work,
                                     weights_ready=True)) for c in range(copies)] * 2
            t = _graph_time_per_call(torch, calls)
            yd = fn(x, wqs[0][0], wqs[0][1], GROUP, work=work)
            torch.cuda.synchronize()
            err = float(torch.linalg.vector_norm(yd.double() - ref.double()) /
                        torch.linalg.vector_norm(ref.double()))
            row[mode] = {"us": t * 1e6, "gbs": gemm_bytes(M_DRAFT, n, k, mode) / t / 1e9,
                         "frac_hbm": gemm_bytes(M_DRAFT, n, k, mode) / t / 1e9 / hbm,
                         "rel_err_vs_verify": err}
        out[name] = row
        del wqs, x, y, ref
        torch.cuda.empty_cache()
    return {"workload": f"Llama-2-7B decode shapes, drafting at M={M_DRAFT}, group {GROUP}; "
                        "inputs N(0,1) with round(0.01 K) outlier channels x20, bf16",
            "timing": "CUDA graph of back-to-back calls, weights rotating past L2 (3x L2)",
            "quality": "||y_draft - y_w4a16|| / ||y_w4a16|| (Frobenius) on the same weights "
                       "and inputs: how far each draft is from the verifying model",
            "shapes": out}


def accept_report(torch, qspec, peaks, sigmas=(0.1, 0.5, 1.0), batch=64, gamma=5, vocab=128256):
    """The accept / residual-resample step at vocab 128256, batch 64, gamma 5, once per
    draft-noise sigma: target logits N(0, 2^2), draft logits = target + N(0, sigma^2),
    seeded; each call timed alone between CUDA events with the L2 flushed before it.
    Algorithmic bytes come from the measured accepted lengths.  near_ties counts tested
    positions whose uniform lies within 1e-6 of p/q (where a rounding difference could
    flip the decision)."""
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    gen = torch.Generator(device="cuda")
    gen.manual_seed(rank_seed(0) + 13)
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device="cuda")
    work = torch.zeros(256, dtype=torch.uint8, device="cuda")
    out = {}
    for sigma in sigmas:
        lp = torch.randn((batch, gamma + 1, vocab), generator=gen, device="cuda",
                         dtype=torch.float64) * 2.0
        lq = lp[:, :gamma] + torch.randn((batch, gamma, vocab), generator=gen, device="cuda",
                                         dtype=torch.float64) * sigma
        p = torch.softmax(lp, -1).float().contiguous()
        q = torch.softmax(lq, -1).float().contiguous()
        del lp, lq
        draft = torch.multinomial(q.reshape(-1, vocab).double(), 1, generator=gen).reshape(
            batch, gamma).to(torch.int32)
        u_acc = (torch.randint(0, 1 << 24, (batch, gamma), generator=gen, device="cuda").double()
                 / (1 << 24)).float()
        u_res = (torch.randint(0, 1 << 24, (batch,), generator=gen, device="cuda").double()
                 / (1 << 24)).float()
        n_acc = torch.empty((batch,), dtype=torch.int32, device="cuda")
        tokens = torch.empty((batch, gamma + 1), dtype=torch.int32, device="cuda")
        ts = []
        for rep in range(8):
            flush.fill_(rep & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            qspec.spec_accept(p, q, draft, u_acc, u_res, n_accepted=n_acc, tokens=tokens, work=work)
            e1.record()
            e1.synchronize()
            if rep >= 2:
                ts.append(e0.elapsed_time(e1) * 1e-3)
        if qspec.workspace_status(work) != 0:
            raise RuntimeError("accept kernel reported bad input")
        t = statistics.median(ts)
        na = n_acc.cpu().numpy()
        byts = accept_bytes(na, gamma, vocab)
        # the greedy rule on the same target rows and drafts
        tg = []
        for rep in range(8):
            flush.fill_(rep & 0xFF)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            ng, _ = qspec.spec_accept_greedy(p, draft, work=work)
            e1.record()
            e1.synchronize()
            if rep >= 2:
                tg.append(e0.elapsed_time(e1) * 1e-3)
        if qspec.workspace_status(work) != 0:
            raise RuntimeError("greedy accept kernel reported bad input")
        t_g = statistics.median(tg)
        ng = ng.cpu().numpy()
        byts_g = greedy_bytes(ng, gamma, vocab)
        # near-tie count over the positions the rule tested
        idx = draft.long().unsqueeze(-1)
        pv = p[:, :gamma].gather(2, idx).squeeze(-1).double()
        qv = q.gather(2, idx).squeeze(-1).double()
        tested = torch.arange(gamma, device="cuda")[None, :] <= n_acc[:, None].long().clamp(max=gamma - 1)
        near = ((u_acc.double() - pv / qv).abs() < 1e-6) & tested
        out[f"sigma_{sigma}"] = {"us": t * 1e6, "bytes": byts, "gbs": byts / t / 1e9,
                                 "frac_hbm": byts / t / 1e9 / hbm,
                                 "mean_accepted": float(na.mean()),
                                 "acceptance_per_position": float(
                                     (na.sum()) / (na.sum() + (na < gamma).sum())),
                                 "near_ties": int(near.sum()),
                                 "greedy": {"us": t_g * 1e6, "bytes": byts_g,
                                            "gbs": byts_g / t_g / 1e9,
                                            "frac_hbm": byts_g / t_g / 1e9 / hbm,
                                            "mean_accepted": float(ng.mean())}}
        del p, q
    del flush
    torch.cuda.empty_cache()
    return {"workload": f"accept/resample, vocab {vocab}, batch {batch}, gamma {gamma}, "
                        "target logits N(0, 2^2), draft = target + N(0, sigma^2)",
            "timing": "each call alone between CUDA events, L2 flushed (256 MB write) before it",
            "bytes": "per sequence: 2 gathered elements per tested position + one vocab row of p "
                     "and q (rejection) or of p (all accepted) + outputs; greedy: the compared "
                     "drafts + rows 0..n of p + outputs",
            "peak_hbm_gbs": hbm, "sigmas": out}


def fused_quant_report(torch, qspec, wq, ws, L, x16):
    """One W4A4 drafting pass of the step (L layers x 4 GEMMs at M = 16), timed as a CUDA
    graph with the activations quantized by the separate per-token pre-pass kernel (the
    default) and inside the GEMM kernel (QSPEC_GEMM_FUSED_QUANT)."""
    dev = x16[0].device
    need = max(qspec.workspace_size(qspec.OP_GEMM_W4A4, M_DRAFT, n, k, GROUP) for (_, n, k) in LAYERS)
    work = torch.zeros(need, dtype=torch.uint8, device=dev)
    ys = [torch.empty((M_DRAFT, n), dtype=torch.float32, device=dev) for (_, n, k) in LAYERS]
    out = {}
    for name, flags in (("pre_pass", 0), ("fused", qspec.GEMM_FUSED_QUANT)):
        def pass_(flags=flags):
            for li in range(L):
                for si in range(len(LAYERS)):
                    qspec.gemm_w4a4(x16[si], wq[li][si], ws[li][si], GROUP, y=ys[si], work=work,
                                    weights_ready=True, flags=flags)
        t = _graph_time_per_call(torch, [pass_], reps=5)
        out[name] = {"us_per_pass": t * 1e6, "us_per_gemm": t * 1e6 / (L * len(LAYERS))}
    if qspec.workspace_status(work) != 0:
        raise RuntimeError("device status reported a fault in the fused-quantization pass")
    return {"workload": f"one W4A4 drafting pass: {L} layers x 4 GEMMs at M={M_DRAFT}",
            "pre_pass": out["pre_pass"], "fused": out["fused"]}


def chained_round_report(torch, qspec, peaks, wq, ws, L, x16, p, q, draft, u_acc, u_res, n_acc,
                         tokens, acc_work, bytes_unchained, ms_unchained):
    """The round with its layers chained: in every pass each of the L layers' four GEMMs
    takes the previous GEMM's fp32 output (its first K columns, cast to bf16 by the glue
    kernel) as input: gamma W4A4 drafting passes at M = 16 (each from its own input),
    one W4A16 verifying pass at M = 80, then accept.  Captured once as a CUDA graph.
    Also the mode-switch cost: the same weights called W4A4 then W4A16 alternately,
    against the same calls grouped by mode (CUDA graphs of back-to-back calls)."""
    dev = x16[0].device
    gen = torch.Generator(device=dev)
    gen.manual_seed(rank_seed(0) + 17)
    hbm = float(peaks.get("hbm_gbs", 6650.0))
    layers = [(wq[li][si], ws[li][si]) for li in range(L) for si in range(len(LAYERS))]
    x0 = [torch.randn((M_DRAFT, 4096), generator=gen, device=dev).to(torch.bfloat16)
          for _ in range(GAMMA)]
    x0v = torch.randn((M_VERIFY, 4096), generator=gen, device=dev).to(torch.bfloat16)

    def bufs(m):
        ys = [torch.empty((m, wq_.shape[0]), dtype=torch.float32, device=dev) for (wq_, _) in layers]
        xs = [None] + [torch.empty((m, wq_.shape[1] * 2), dtype=torch.bfloat16, device=dev)
                       for (wq_, _) in layers[1:]]
        return ys, xs

    dbufs = [bufs(M_DRAFT) for _ in range(GAMMA)]
    vbufs = bufs(M_VERIFY)
    need = max(qspec.workspace_size(op, m, n, k, GROUP) for (_, n, k) in LAYERS
               for (op, m) in ((qspec.OP_GEMM_W4A4, M_DRAFT), (qspec.OP_GEMM_W4A16, M_VERIFY)))
    work = torch.zeros(need, dtype=torch.uint8, device=dev)

    def round_():
        for pss in range(GAMMA):
            qspec.linear_chain(x0[pss], layers, "w4a4", GROUP, ys=dbufs[pss][0], xs=dbufs[pss][1],
                               work=work, weights_ready=True)
        qspec.linear_chain(x0v, layers, "w4a16", GROUP, ys=vbufs[0], xs=vbufs[1], work=work,
                           weights_ready=True)
        qspec.spec_accept(p, q, draft, u_acc, u_res, n_accepted=n_acc, tokens=tokens, work=acc_work)

    t_round = _graph_time_per_call(torch, [round_], reps=5)
    if qspec.workspace_status(work) != 0:
        raise RuntimeError("device status reported a fault in the chained round")
    # chained inputs: a drafting quantizer reads 4 bytes (fp32) instead of 2 per
    # element; the verifying pass's cast reads 4 and writes 2
    glue = sum((GAMMA * M_DRAFT * 2 + M_VERIFY * (4 + 2)) * k
               for (wq_, _) in layers[1:] for k in (wq_.shape[1] * 2,))
    byts = bytes_unchained + glue
    # mode switch: layer-0 gate_up weights, W4A4 at M=16 and W4A16 at M=80
    wq0, ws0 = wq[0][2], ws[0][2]
    xa = x16[2]
    xv = torch.randn((M_VERIFY, 4096), generator=gen, device=dev).to(torch.bfloat16)
    ya = torch.empty((M_DRAFT, 22016), dtype=torch.float32, device=dev)
    yv = torch.empty((M_VERIFY, 22016), dtype=torch.float32, device=dev)
    a = lambda: qspec.gemm_w4a4(xa, wq0, ws0, GROUP, y=ya, work=work, weights_ready=True)
    v = lambda: qspec.gemm_w4a16(xv, wq0, ws0, GROUP, y=yv, work=work, weights_ready=True)
    t_alt = _graph_time_per_call(torch, [a, v] * 10)
    t_grp = _graph_time_per_call(torch, [a] * 10 + [v] * 10)
    return {"workload": f"{L} Llama-2-7B-shaped layers chained (QKV -> first 4096 columns -> o_proj "
                        "-> gate_up -> first 11008 columns -> down -> next layer), gamma="
                        f"{GAMMA} W4A4 drafting passes at M={M_DRAFT} from their own inputs, one "
                        f"W4A16 verifying pass at M={M_VERIFY}, accept B={BATCH} V={VOCAB}",
            "glue": "drafting passes: the next W4A4 call reads the previous fp32 output and "
                    "rounds it to bf16 in its activation quantizer (qspec_gemm_w4a4_f32in); "
                    "verifying pass: qspec_cast_bf16 between consecutive GEMMs",
            "ms_per_round": t_round * 1e3, "bytes": byts, "gbs": byts / t_round / 1e9,
            "frac_hbm": byts / t_round / 1e9 / hbm,
            "ms_per_round_unchained": ms_unchained,
            "mode_switch": {
                "shape": "gate_up 22016x4096 of layer 0, W4A4 at M=16 and W4A16 at M=80, one weight set",
                "us_per_call_alternating": t_alt * 1e6, "us_per_call_grouped": t_grp * 1e6,
                "switch_cost_us": (t_alt - t_grp) * 20 / 18 * 1e6,
                "note": "20 calls alternating W4A4/W4A16 on the same wq/ws (19 switches) against "
                        "the same 20 calls grouped by mode (1 switch): the time difference over "
                        "the 18 extra switches"}}


def measure_e2e(torch, stream, graph, acts, accept_in, outs, steps, bytes_step):
    """Same step through the public API with host buffers: every step copies the
    step's inputs from pinned host memory and reads the result back."""
    host_in = [t.detach().cpu().pin_memory() for group in acts for t in group] + \
              [t.detach().cpu().pin_memory() for t in accept_in]
    dev_in = [t for group in acts for t in group] + list(accept_in)
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda.synchronize()
        start.record(stream)
        for _ in range(steps):
            for d, h in zip(dev_in, host_in):
                d.copy_(h, non_blocking=True)
            graph.replay()
            for h, d in zip(host_out, outs):
                h.copy_(d, non_blocking=True)
        end.record(stream)
        end.synchronize()
    ms = start.elapsed_time(end) / steps
    return {"value": bytes_step / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


TRAFFIC_PROFILE = "qgemm_w4a4_llama2_7b_decode_m16.json"


def traffic_from_profile():
    """(DRAM bytes per W4A4 drafting call averaged over the four decode shapes, source)
    from the committed ncu summary, if it was taken on the current GEMM and quantizer
    sources; else (None, reason)."""
    path = os.path.join(ROOT, "profiles", TRAFFIC_PROFILE)
    csrc = os.path.join(ROOT, "quantized_speculative_decoding_packed_b200", "csrc")
    try:
        with open(path) as f:
            prof = json.load(f)
        for name, sha in prof["source_sha256"].items():
            if hashlib.sha256(open(os.path.join(csrc, name), "rb").read()).hexdigest() != sha:
                return None, f"profiles/{TRAFFIC_PROFILE} predates the current {name}"
        per_shape = prof["dram_bytes_per_call"]
        return (sum(per_shape.values()) / len(per_shape),
                f"profiles/{TRAFFIC_PROFILE}: ncu dram__bytes_read.sum + dram__bytes_write.sum "
                "of the quantizer and GEMM launches of one call per shape, averaged over the "
                "four shapes")
    except Exception as e:  # missing or malformed summary: no traffic figure
        return None, f"profiles/{TRAFFIC_PROFILE} unreadable ({type(e).__name__})"


if __name__ == "__main__":
    main()
