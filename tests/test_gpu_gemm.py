"""GPU parity of the shared-INT4 GEMMs against the oracle.

W4A4: per-group int32 accumulators bit-exact; outputs within 1e-3 relative.
W4A16: outputs within 1e-3 relative Frobenius of the float64 oracle on the
same dequantized weights (and bit-exact where every partial sum is an
integer below 2^24).
"""
import numpy as np
import pytest
import torch

from oracle import qspec_oracle as orc
from quantized_speculative_decoding_packed_b200 import synth

from gpu_util import assert_close_1e3, cuda_bf16, cuda_f32, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qs():
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def _prep(qs, gi):
    wq, ws = qs.quantize_weights(cuda_f32(gi.w), gi.group)
    q, s_h = orc.quantize_weights(gi.w, gi.group)
    return wq, ws, q, s_h


SHAPES = [  # (m, n, k, group): tiles, ragged tails, both group sizes, every token tile
    (4, 256, 256, 64), (1, 256, 1024, 128), (3, 200, 256, 64), (16, 1000, 1024, 128),
    (17, 384, 512, 128), (33, 256, 384, 64), (48, 130, 256, 128), (64, 512, 768, 128),
    (80, 512, 1024, 128), (95, 256, 256, 64), (100, 256, 384, 128), (128, 384, 512, 128),
    (130, 384, 512, 128), (257, 136, 256, 64),
]


@pytest.mark.parametrize("m,n,k,group", SHAPES)
def test_w4a4_accumulators_exact_and_output(qs, m, n, k, group):
    gi = synth.gemm_inputs("llama3_8b", m, n, k, group, stream=99)
    wq, ws, q, s_h = _prep(qs, gi)
    dbg = torch.zeros((m, n, k // group), dtype=torch.int32, device="cuda")
    y = qs.gemm_w4a4(cuda_bf16(gi.x_bits), wq, ws, group, dbg_acc=dbg)
    torch.cuda.synchronize()
    y_ref, acc = orc.gemm_w4a4(gi.x, q, s_h, group, return_acc=True)
    assert np.array_equal(dbg.cpu().numpy(), acc)
    assert_close_1e3(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("mode", ["w4a4", "w4a8"])
@pytest.mark.parametrize("m,n,k,group", [s for s in SHAPES if s[0] <= 32] + [(16, 12288, 4096, 128)])
def test_fused_quantization_exact(qs, mode, m, n, k, group):
    """Activations quantized inside the GEMM kernel (QSPEC_GEMM_FUSED_QUANT):
    accumulators bit-exact and outputs within the bar, twice in a row on one
    workspace (its counters return to zero after every call)."""
    gi = synth.gemm_inputs("llama3_8b", m, n, k, group, stream=96)
    wq, ws, q, s_h = _prep(qs, gi)
    fn = qs.gemm_w4a4 if mode == "w4a4" else qs.gemm_w4a8
    ref = orc.gemm_w4a4 if mode == "w4a4" else orc.gemm_w4a8
    op = qs.OP_GEMM_W4A4 if mode == "w4a4" else qs.OP_GEMM_W4A8
    work = torch.zeros(qs.workspace_size(op, m, n, k, group), dtype=torch.uint8, device="cuda")
    y_ref, acc = ref(gi.x, q, s_h, group, return_acc=True)
    for _ in range(2):
        dbg = torch.zeros((m, n, k // group), dtype=torch.int32, device="cuda")
        y = fn(cuda_bf16(gi.x_bits), wq, ws, group, dbg_acc=dbg, work=work, flags=qs.GEMM_FUSED_QUANT)
        torch.cuda.synchronize()
        assert np.array_equal(dbg.cpu().numpy(), acc)
        assert_close_1e3(y.cpu().numpy(), y_ref)
    assert qs.workspace_status(work) == 0


@pytest.mark.parametrize("m,n,k,group", SHAPES)
def test_w4a16_output(qs, m, n, k, group):
    gi = synth.gemm_inputs("llama3_8b", m, n, k, group, stream=98)
    wq, ws, q, s_h = _prep(qs, gi)
    y = qs.gemm_w4a16(cuda_bf16(gi.x_bits), wq, ws, group)
    torch.cuda.synchronize()
    y_ref = orc.gemm_w4a16(gi.x, q, s_h, group)
    assert_close_1e3(y.cpu().numpy(), y_ref)
    assert rel_fro(y.cpu().numpy(), y_ref) < 1e-5      # fp32 accumulation only


@pytest.mark.parametrize("mode", ["w4a4", "w4a16"])
def test_integer_special_case_bit_exact(qs, mode):
    """Scale 1 (absmax 7 per group) and integer activations with absmax 7:
    every partial sum is an integer below 2^24, so both modes are exact."""
    rng = np.random.default_rng(21)
    m, n, k = 20, 384, 512
    lv = rng.integers(-7, 8, size=(n, k))
    lv[:, ::128] = 7
    xi = rng.integers(-7, 8, size=(m, k)).astype(np.float32)
    xi[:, 3] = -7
    bits = synth.to_bf16_bits(xi)
    wq, ws = qs.quantize_weights(cuda_f32(lv.astype(np.float32)), 128)
    fn = qs.gemm_w4a4 if mode == "w4a4" else qs.gemm_w4a16
    y = fn(cuda_bf16(bits), wq, ws, 128)
    torch.cuda.synchronize()
    assert np.array_equal(y.cpu().numpy().astype(np.float64), (xi.astype(np.int64) @ lv.T).astype(np.float64))


def test_repeat_calls_are_deterministic(qs):
    gi = synth.gemm_inputs("llama3_8b", 16, 4096, 4096, 128, stream=5)
    wq, ws, q, s_h = _prep(qs, gi)
    x = cuda_bf16(gi.x_bits)
    for fn in (qs.gemm_w4a4, qs.gemm_w4a16):
        y1 = fn(x, wq, ws, 128).clone()
        y2 = fn(x, wq, ws, 128).clone()
        torch.cuda.synchronize()
        assert torch.equal(y1, y2)


def _sampled_full_size(qs, mode, m, name, n, k):
    gi = synth.gemm_inputs("llama2_7b", m, n, k, 128)
    wq, ws = qs.quantize_weights(cuda_f32(gi.w), 128)
    x = cuda_bf16(gi.x_bits)
    cols = np.sort(synth.rng_for("llama2_7b", 9, n).choice(n, size=256, replace=False))
    q, s_h = orc.quantize_weights(gi.w[cols], 128)
    if mode == "w4a4":
        dbg = torch.zeros((m, n, k // 128), dtype=torch.int32, device="cuda")
        y = qs.gemm_w4a4(x, wq, ws, 128, dbg_acc=dbg)
        torch.cuda.synchronize()
        y_ref, acc = orc.gemm_w4a4(gi.x, q, s_h, 128, return_acc=True)
        assert np.array_equal(dbg.cpu().numpy()[:, cols, :], acc)
    else:
        y = qs.gemm_w4a16(x, wq, ws, 128)
        torch.cuda.synchronize()
        y_ref = orc.gemm_w4a16(gi.x, q, s_h, 128)
    assert_close_1e3(y.cpu().numpy()[:, cols], y_ref)


@pytest.mark.parametrize("name,n,k", synth.LLAMA2_7B_LAYERS)
def test_llama2_7b_decode_shapes_sampled(qs, name, n, k):
    _sampled_full_size(qs, "w4a4", 16, name, n, k)
    _sampled_full_size(qs, "w4a16", 80, name, n, k)


@pytest.mark.parametrize("m", synth.LLAMA3_8B_M_SWEEP)
def test_llama3_8b_sweep_sampled(qs, m):
    n, k = 6144, 4096
    gi = synth.gemm_inputs("llama3_8b", m, n, k, 128)
    wq, ws = qs.quantize_weights(cuda_f32(gi.w), 128)
    x = cuda_bf16(gi.x_bits)
    cols = np.sort(synth.rng_for("llama3_8b", 9, m).choice(n, size=128, replace=False))
    q, s_h = orc.quantize_weights(gi.w[cols], 128)
    y4 = qs.gemm_w4a4(x, wq, ws, 128)
    y16 = qs.gemm_w4a16(x, wq, ws, 128)
    torch.cuda.synchronize()
    assert_close_1e3(y4.cpu().numpy()[:, cols], orc.gemm_w4a4(gi.x, q, s_h, 128))
    assert_close_1e3(y16.cpu().numpy()[:, cols], orc.gemm_w4a16(gi.x, q, s_h, 128))


def test_llama2_70b_large_m_sampled(qs):
    """M = 2048 on the 70B QKV shape; outputs checked on sampled rows and columns."""
    m, n, k = 2048, 10240, 8192
    gi = synth.gemm_inputs("llama2_70b", m, n, k, 128)
    wq, ws = qs.quantize_weights(cuda_f32(gi.w), 128)
    x = cuda_bf16(gi.x_bits)
    rows = np.sort(synth.rng_for("llama2_70b", 9, 1).choice(m, size=64, replace=False))
    cols = np.sort(synth.rng_for("llama2_70b", 9, 2).choice(n, size=64, replace=False))
    q, s_h = orc.quantize_weights(gi.w[cols], 128)
    y4 = qs.gemm_w4a4(x, wq, ws, 128)
    y16 = qs.gemm_w4a16(x, wq, ws, 128)
    torch.cuda.synchronize()
    xs = gi.x[rows]
    # the W4A4 reference quantizes each sampled row on its own, as the kernel does
    assert_close_1e3(y4.cpu().numpy()[np.ix_(rows, cols)], orc.gemm_w4a4(xs, q, s_h, 128))
    assert_close_1e3(y16.cpu().numpy()[np.ix_(rows, cols)], orc.gemm_w4a16(xs, q, s_h, 128))


def test_shared_weights_are_one_buffer(qs):
    """Both modes read the same wq/ws bytes; nothing is repacked per mode."""
    gi = synth.gemm_inputs("llama3_8b", 16, 256, 256, 128, stream=3)
    wq, ws = qs.quantize_weights(cuda_f32(gi.w), 128)
    before = (wq.clone(), ws.clone())
    x = cuda_bf16(gi.x_bits)
    qs.gemm_w4a4(x, wq, ws, 128)
    qs.gemm_w4a16(x, wq, ws, 128)
    torch.cuda.synchronize()
    assert torch.equal(before[0], wq) and torch.equal(before[1], ws)


def test_one_workspace_shared_across_shapes(qs):
    """Scratch left by a call of one shape must not disturb a call of another."""
    shapes = [(4, 256, 256, 64), (16, 12288, 4096, 128), (80, 4096, 11008, 128), (3, 200, 256, 64),
              (16, 12288, 4096, 128)]
    need = max(qs.workspace_size(qs.OP_GEMM_W4A4, m, n, k, g) for (m, n, k, g) in shapes)
    work = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, (m, n, k, g) in enumerate(shapes):
        gi = synth.gemm_inputs("llama3_8b", m, n, k, g, stream=40 + i)
        wq, ws = qs.quantize_weights(cuda_f32(gi.w), g)
        x = cuda_bf16(gi.x_bits)
        y4 = qs.gemm_w4a4(x, wq, ws, g, work=work)
        y16 = qs.gemm_w4a16(x, wq, ws, g, work=work)
        torch.cuda.synchronize()
        cols = np.arange(0, n, max(1, n // 64))
        q, s_h = orc.quantize_weights(gi.w[cols], g)
        assert_close_1e3(y4.cpu().numpy()[:, cols], orc.gemm_w4a4(gi.x, q, s_h, g))
        assert_close_1e3(y16.cpu().numpy()[:, cols], orc.gemm_w4a16(gi.x, q, s_h, g))
        assert qs.workspace_status(work) == 0


@pytest.mark.parametrize("weights_ready", [False, True])
def test_back_to_back_calls_overlap_safely(qs, weights_ready):
    """Calls are launched so that each may start while the previous finishes.

    A chain of W4A4 and W4A16 calls on one stream, with no synchronisation,
    shares one workspace (split-tile shares and tickets, quantized
    activations) and rewrites the same outputs; run eagerly and as a CUDA
    graph, every output must be bit-identical to a standalone call.  With
    weights_ready the weights stream before the preceding call completes.
    """
    shapes = [(16, 12288, 4096), (80, 4096, 11008), (16, 4096, 11008), (80, 12288, 4096)]
    ops, want = [], []
    need = 0
    for i, (m, n, k) in enumerate(shapes):
        gi = synth.gemm_inputs("llama2_7b", m, n, k, 128, stream=60 + i)
        wq, ws = qs.quantize_weights(cuda_f32(gi.w), 128)
        x = cuda_bf16(gi.x_bits)
        mode = "w4a4" if m == 16 else "w4a16"
        fn = qs.gemm_w4a4 if mode == "w4a4" else qs.gemm_w4a16
        want.append(fn(x, wq, ws, 128).clone())            # standalone reference
        ops.append((fn, x, wq, ws, m, n))
        need = max(need, qs.workspace_size(qs.OP_GEMM_W4A4, m, n, k, 128))
    torch.cuda.synchronize()
    work = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = {}                                              # one output buffer per (m, n)
    for (fn, x, wq, ws, m, n) in ops:
        outs.setdefault((m, n), torch.empty((m, n), dtype=torch.float32, device="cuda"))

    def chain():
        for _ in range(3):
            for (fn, x, wq, ws, m, n) in ops:
                fn(x, wq, ws, 128, y=outs[(m, n)], work=work, weights_ready=weights_ready)

    for y in outs.values():
        y.fill_(float("nan"))
    chain()
    torch.cuda.synchronize()
    for (fn, x, wq, ws, m, n), ref in zip(ops, want):
        assert torch.equal(outs[(m, n)], ref)
    assert qs.workspace_status(work) == 0

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        chain()
    for y in outs.values():
        y.fill_(float("nan"))
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    for (fn, x, wq, ws, m, n), ref in zip(ops, want):
        assert torch.equal(outs[(m, n)], ref)
    assert qs.workspace_status(work) == 0


@pytest.mark.parametrize("mode", ["w4a4", "w4a16"])
def test_weights_rewritten_just_before_the_call(qs, mode):
    """Without QSPEC_GEMM_WEIGHTS_READY the GEMM reads the weights only after
    the kernel before it has finished: quantizing new weights into the same
    buffers right before the call (no synchronisation) gives the new result."""
    m = 16 if mode == "w4a4" else 80
    n, k = 4096, 4096
    fn = qs.gemm_w4a4 if mode == "w4a4" else qs.gemm_w4a16
    g_old = synth.gemm_inputs("llama2_7b", m, n, k, 128, stream=70)
    g_new = synth.gemm_inputs("llama2_7b", m, n, k, 128, stream=71)
    x = cuda_bf16(g_new.x_bits)
    wq_new, ws_new = qs.quantize_weights(cuda_f32(g_new.w), 128)
    want = fn(x, wq_new, ws_new, 128).clone()
    w_new = cuda_f32(g_new.w)
    wq, ws = qs.quantize_weights(cuda_f32(g_old.w), 128)
    work = torch.zeros(qs.workspace_size(qs.OP_GEMM_W4A4, m, n, k, 128), dtype=torch.uint8,
                       device="cuda")
    y = torch.empty((m, n), dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()
    for _ in range(3):
        fn(x, wq, ws, 128, y=y, work=work)                  # old weights, keeps the GPU busy
        qs.quantize_weights(w_new, 128, wq=wq, ws=ws)       # overwrite in place
        fn(x, wq, ws, 128, y=y, work=work)                  # must see the new weights
        torch.cuda.synchronize()
        assert torch.equal(y, want)
        qs.quantize_weights(cuda_f32(g_old.w), 128, wq=wq, ws=ws)
    assert qs.workspace_status(work) == 0


# ---------------------------------------------------------------- W4A8 drafting variant
@pytest.mark.parametrize("m,n,k,group", SHAPES[:8] + [(130, 384, 512, 128)])
def test_w4a8_accumulators_exact_and_output(qs, m, n, k, group):
    gi = synth.gemm_inputs("llama3_8b", m, n, k, group, stream=97)
    wq, ws, q, s_h = _prep(qs, gi)
    dbg = torch.zeros((m, n, k // group), dtype=torch.int32, device="cuda")
    y = qs.gemm_w4a8(cuda_bf16(gi.x_bits), wq, ws, group, dbg_acc=dbg)
    torch.cuda.synchronize()
    y_ref, acc = orc.gemm_w4a8(gi.x, q, s_h, group, return_acc=True)
    assert np.array_equal(dbg.cpu().numpy(), acc)
    assert_close_1e3(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("name,n,k", synth.LLAMA2_7B_LAYERS)
def test_w4a8_llama2_7b_sampled_and_closer_to_verify(qs, name, n, k):
    """Full 7B decode shapes at M = 16 on sampled columns; the 8-bit draft's outputs sit
    closer to the verifying mode's than the 4-bit draft's (outlier channels x20)."""
    gi = synth.gemm_inputs("llama2_7b", 16, n, k, 128)
    wq, ws = qs.quantize_weights(cuda_f32(gi.w), 128)
    x = cuda_bf16(gi.x_bits)
    cols = np.sort(synth.rng_for("llama2_7b", 9, n).choice(n, size=256, replace=False))
    q, s_h = orc.quantize_weights(gi.w[cols], 128)
    y8 = qs.gemm_w4a8(x, wq, ws, 128)
    y4 = qs.gemm_w4a4(x, wq, ws, 128)
    y16 = qs.gemm_w4a16(x, wq, ws, 128)
    torch.cuda.synchronize()
    assert_close_1e3(y8.cpu().numpy()[:, cols], orc.gemm_w4a8(gi.x, q, s_h, 128))
    d8 = float((y8 - y16).norm())
    d4 = float((y4 - y16).norm())
    assert d8 < 0.5 * d4
