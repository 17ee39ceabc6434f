"""Python binding of libqspec.so (the C ABI in include/qspec.h).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of the library.  Importing this module loads the library and raises
if it is missing; there is no fallback implementation.

Functions take CUDA torch tensors (contiguous, on the current device) and
launch on the current torch stream unless `stream` is given.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqspec.so")

OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported device", 3: "CUDA error",
                4: "workspace too small", 5: "timeout", 6: "bad input"}
OP_QUANTIZE_WEIGHTS, OP_QUANT_ACT, OP_GEMM_W4A4, OP_GEMM_W4A16, OP_SPEC_ACCEPT, OP_GEMM_W4A8 = range(6)

EXPORTED = ("qspec_quantize_weights", "qspec_quant_act", "qspec_cast_bf16", "qspec_gemm_w4a4",
            "qspec_gemm_w4a8",
            "qspec_gemm_w4a16",
            "qspec_spec_accept", "qspec_spec_accept_greedy", "qspec_workspace_size",
            "qspec_workspace_status",
            "qspec_status_string", "qspec_gemm_w4a16_noalloc", "qspec_gemm_w4a16_noalloc_status",
            "qspec_kv_append", "qspec_attn_decode", "qspec_attn_workspace_size", "qspec_kv_commit",
            "qspec_abi_version")
ABI_VERSION = 5
HEAD_DIM = 128           # the KV-cache calls' head dimension
GEMM_WEIGHTS_READY = 1   # flag: wq/ws are not written by work still in flight
GEMM_TEST_STALL = 0x100  # test hook: the GEMM's first wait runs out (QSPEC_GEMM_TEST_STALL)
GEMM_FUSED_QUANT = 0x2   # drafting modes, m <= 32: activations quantized inside the GEMM kernel


class QSpecError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} (status {status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libqspec.so not found at {_LIB_PATH}; build it with "
            "`python -m quantized_speculative_decoding_packed_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, I32, U32, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32,
                            ctypes.c_size_t)
    lib.qspec_quantize_weights.argtypes = [P, I64, I64, I32, P, P, P]
    lib.qspec_quant_act.argtypes = [P, I64, I64, P, P, P]
    lib.qspec_cast_bf16.argtypes = [P, I64, I64, I64, P, P]
    lib.qspec_gemm_w4a4.argtypes = [P, I64, I64, P, P, I64, I32, P, P, SZ, P, U32, P]
    lib.qspec_gemm_w4a8.argtypes = [P, I64, I64, P, P, I64, I32, P, P, SZ, P, U32, P]
    lib.qspec_gemm_w4a4_f32in.argtypes = [P, I64, I64, I64, P, P, I64, I32, P, P, SZ, P, U32, P]
    lib.qspec_gemm_w4a8_f32in.argtypes = [P, I64, I64, I64, P, P, I64, I32, P, P, SZ, P, U32, P]
    lib.qspec_gemm_w4a16.argtypes = [P, I64, I64, P, P, I64, I32, P, P, SZ, U32, P]
    lib.qspec_gemm_w4a16_noalloc.argtypes = [P, I64, I64, P, P, I64, I32, P, U32, P]
    lib.qspec_gemm_w4a16_noalloc_status.argtypes = [P]
    lib.qspec_abi_version.argtypes = []
    lib.qspec_abi_version.restype = I32
    lib.qspec_spec_accept.argtypes = [P, P, P, P, P, I32, I32, I32, P, P, P, SZ, P]
    lib.qspec_spec_accept_greedy.argtypes = [P, P, I32, I32, I32, P, P, P, SZ, P]
    lib.qspec_workspace_size.argtypes = [I32, I64, I64, I64, I32, I32, I32, I32]
    lib.qspec_workspace_size.restype = SZ
    lib.qspec_workspace_status.argtypes = [P, P]
    lib.qspec_kv_append.argtypes = [P, I64, I32, I32, I32, I32, I32, P, I32, P, P, I32, P, SZ, P]
    lib.qspec_attn_decode.argtypes = [P, I64, I32, I32, I32, I32, I32, P, I32, P, P, I32, I32, P,
                                      I64, P, SZ, P]
    lib.qspec_attn_workspace_size.argtypes = [I32, I32, I32, I32, I32, I32]
    lib.qspec_attn_workspace_size.restype = SZ
    lib.qspec_kv_commit.argtypes = [P, P, I32, I32, P, SZ, P]
    lib.qspec_status_string.argtypes = [I32]
    lib.qspec_status_string.restype = ctypes.c_char_p
    for name in ("qspec_quantize_weights", "qspec_quant_act", "qspec_cast_bf16", "qspec_gemm_w4a4",
                 "qspec_gemm_w4a8", "qspec_gemm_w4a4_f32in", "qspec_gemm_w4a8_f32in",
                 "qspec_gemm_w4a16", "qspec_spec_accept", "qspec_spec_accept_greedy",
                 "qspec_workspace_status",
                 "qspec_gemm_w4a16_noalloc", "qspec_gemm_w4a16_noalloc_status",
                 "qspec_kv_append", "qspec_attn_decode", "qspec_kv_commit"):
        getattr(lib, name).restype = ctypes.c_int
    if lib.qspec_abi_version() != ABI_VERSION:
        raise ImportError(f"{_LIB_PATH} has ABI version {lib.qspec_abi_version()}, "
                          f"this binding needs {ABI_VERSION}; rebuild the library")
    return lib


LIB = _load()
LIB_PATH = _LIB_PATH


def _check(status: int, what: str) -> None:
    if status != OK:
        raise QSpecError(status, what)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")


_WS_CACHE: dict = {}


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-initialised per-device scratch buffer of at least `nbytes` bytes.

    The library leaves it ready for reuse after every call that completes.
    Calls that run concurrently on different streams need separate buffers.
    """
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    cur = _WS_CACHE.get(dev)
    if cur is None or cur.numel() < nbytes:
        cur = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
        _WS_CACHE[dev] = cur
    return cur


def workspace_size(op: int, m: int = 0, n: int = 0, k: int = 0, group: int = 128,
                   batch: int = 0, gamma: int = 0, vocab: int = 0) -> int:
    return int(LIB.qspec_workspace_size(op, m, n, k, group, batch, gamma, vocab))


def workspace_status(ws: torch.Tensor, stream=None) -> int:
    return int(LIB.qspec_workspace_status(_ptr(ws), _stream(stream)))


def scale_row_stride(k: int, group: int) -> int:
    """Entries per row of the scale matrix: k/group rounded up to a multiple of 8."""
    return (k // group + 7) // 8 * 8


def quantize_weights(w: torch.Tensor, group: int = 128, wq: torch.Tensor | None = None,
                     ws: torch.Tensor | None = None, stream=None):
    """fp32 [N][K] -> (wq uint8 [N][K/2], ws fp16 [N][scale_row_stride(K, group)]).

    ws[:, :K/group] holds the group scales; the padding columns are zero.
    """
    _need(w, torch.float32, "w")
    n, k = w.shape
    if wq is None:
        wq = torch.empty((n, k // 2), dtype=torch.uint8, device=w.device)
    if ws is None:
        ws = torch.empty((n, scale_row_stride(k, group)), dtype=torch.float16, device=w.device)
    _check(LIB.qspec_quantize_weights(_ptr(w), n, k, group, _ptr(wq), _ptr(ws), _stream(stream)),
           "qspec_quantize_weights")
    return wq, ws


def quant_act(x: torch.Tensor, xq: torch.Tensor | None = None, xs: torch.Tensor | None = None,
              stream=None):
    """bf16 [M][K] -> (xq uint8 [M][K/2] packed INT4, xs fp32 [M] per-token scales)."""
    _need(x, torch.bfloat16, "x")
    m, k = x.shape
    if xq is None:
        xq = torch.empty((m, k // 2), dtype=torch.uint8, device=x.device)
    if xs is None:
        xs = torch.empty((m,), dtype=torch.float32, device=x.device)
    _check(LIB.qspec_quant_act(_ptr(x), m, k, _ptr(xq), _ptr(xs), _stream(stream)),
           "qspec_quant_act")
    return xq, xs


def _flags(weights_ready: bool, flags: int) -> int:
    return (GEMM_WEIGHTS_READY if weights_ready else 0) | flags


def cast_bf16(y: torch.Tensor, k: int | None = None, x: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """fp32 [M][N] -> bf16 [M][k]: the first k columns rounded to nearest even."""
    _need(y, torch.float32, "y")
    m, n = y.shape
    k = n if k is None else k
    if x is None:
        x = torch.empty((m, k), dtype=torch.bfloat16, device=y.device)
    _check(LIB.qspec_cast_bf16(_ptr(y), m, n, k, _ptr(x), _stream(stream)), "qspec_cast_bf16")
    return x


def linear_chain(x0: torch.Tensor, layers, mode: str = "w4a4", group: int = 128,
                 ys=None, xs=None, work: torch.Tensor | None = None, stream=None,
                 weights_ready: bool = False):
    """Runs linear layers back to back on one token batch: layer j's input is
    the first K_j columns of layer j-1's fp32 output, rounded to bf16 (by the
    drafting GEMMs' quantizer as it reads them, or by qspec_cast_bf16 for the
    verifying GEMM).  layers: [(wq, ws)]; mode: w4a4 | w4a8 | w4a16.  ys/xs:
    optional preallocated outputs / intermediate inputs (for CUDA-graph
    capture).  Returns the list of fp32 outputs."""
    gemm = {"w4a4": gemm_w4a4, "w4a8": gemm_w4a8, "w4a16": gemm_w4a16}[mode]
    m = x0.shape[0]
    outs = []
    x = x0
    for j, (wq, ws) in enumerate(layers):
        n, k = wq.shape[0], wq.shape[1] * 2
        if j and mode != "w4a16":
            x = outs[-1][:, :k]
        elif j:
            x = cast_bf16(outs[-1], k, x=None if xs is None else xs[j], stream=stream)
        y = None if ys is None else ys[j]
        outs.append(gemm(x, wq, ws, group, y=y, work=work, stream=stream, weights_ready=weights_ready))
    return outs


def gemm_w4a4(x: torch.Tensor, wq: torch.Tensor, ws: torch.Tensor, group: int = 128,
              y: torch.Tensor | None = None, work: torch.Tensor | None = None,
              dbg_acc: torch.Tensor | None = None, stream=None,
              weights_ready: bool = False, flags: int = 0) -> torch.Tensor:
    """W4A4 drafting GEMM: y[M][N] fp32 = quant(x) . deq(wq, ws)^T.

    weights_ready: wq/ws are not being written by work that may still be
    running (sets QSPEC_GEMM_WEIGHTS_READY; the weights then stream while the
    preceding kernel finishes).  flags: further QSPEC_GEMM_* bits.
    """
    return _drafting("w4a4", x, wq, ws, group, y, work, dbg_acc, stream, weights_ready, flags)


def gemm_w4a8(x: torch.Tensor, wq: torch.Tensor, ws: torch.Tensor, group: int = 128,
              y: torch.Tensor | None = None, work: torch.Tensor | None = None,
              dbg_acc: torch.Tensor | None = None, stream=None,
              weights_ready: bool = False, flags: int = 0) -> torch.Tensor:
    """W4A8 drafting variant: y[M][N] fp32 = quant8(x) . deq(wq, ws)^T (arguments as gemm_w4a4)."""
    return _drafting("w4a8", x, wq, ws, group, y, work, dbg_acc, stream, weights_ready, flags)


def _drafting(mode, x, wq, ws, group, y, work, dbg_acc, stream, weights_ready, flags):
    """The drafting GEMMs: x bf16 [M][K] (contiguous), or fp32 [M][K] with unit column
    stride (e.g. the first K columns of a layer's output), rounded to bf16 as it is
    quantized (qspec_gemm_*_f32in)."""
    m, k = x.shape
    n = wq.shape[0]
    op = OP_GEMM_W4A4 if mode == "w4a4" else OP_GEMM_W4A8
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    need = workspace_size(op, m, n, k, group)
    if work is None:
        work = workspace(need, x.device)
    fl = _flags(weights_ready, flags)
    if x.dtype == torch.float32:
        if not x.is_cuda or x.stride(1) != 1:
            raise ValueError("fp32 x must be a CUDA tensor with unit column stride")
        fn = LIB.qspec_gemm_w4a4_f32in if mode == "w4a4" else LIB.qspec_gemm_w4a8_f32in
        _check(fn(_ptr(x), x.stride(0), m, k, _ptr(wq), _ptr(ws), n, group, _ptr(y), _ptr(work),
                  work.numel(), _ptr(dbg_acc), fl, _stream(stream)), f"qspec_gemm_{mode}_f32in")
        return y
    _need(x, torch.bfloat16, "x")
    fn = LIB.qspec_gemm_w4a4 if mode == "w4a4" else LIB.qspec_gemm_w4a8
    _check(fn(_ptr(x), m, k, _ptr(wq), _ptr(ws), n, group, _ptr(y), _ptr(work), work.numel(),
              _ptr(dbg_acc), fl, _stream(stream)), f"qspec_gemm_{mode}")
    return y


def gemm_w4a16(x: torch.Tensor, wq: torch.Tensor, ws: torch.Tensor, group: int = 128,
               y: torch.Tensor | None = None, work: torch.Tensor | None = None,
               stream=None, weights_ready: bool = False, flags: int = 0) -> torch.Tensor:
    """W4A16 verifying GEMM: y[M][N] fp32 = x . deq(wq, ws)^T (weights_ready, flags: as gemm_w4a4)."""
    _need(x, torch.bfloat16, "x")
    m, k = x.shape
    n = wq.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    need = workspace_size(OP_GEMM_W4A16, m, n, k, group)
    if work is None:
        work = workspace(need, x.device)
    _check(LIB.qspec_gemm_w4a16(_ptr(x), m, k, _ptr(wq), _ptr(ws), n, group, _ptr(y), _ptr(work),
                                work.numel(), _flags(weights_ready, flags),
                                _stream(stream)), "qspec_gemm_w4a16")
    return y


def gemm_w4a16_noalloc(x: torch.Tensor, wq: torch.Tensor, ws: torch.Tensor, group: int = 128,
                       y: torch.Tensor | None = None, stream=None,
                       weights_ready: bool = False) -> torch.Tensor:
    """W4A16 verifying GEMM using the library's built-in scratch (no workspace).

    For callers that cannot allocate device memory where they call; the
    output buffer is still the caller's.  Calls must not overlap on the GPU.
    """
    _need(x, torch.bfloat16, "x")
    m, k = x.shape
    n = wq.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _check(LIB.qspec_gemm_w4a16_noalloc(_ptr(x), m, k, _ptr(wq), _ptr(ws), n, group, _ptr(y),
                                        GEMM_WEIGHTS_READY if weights_ready else 0,
                                        _stream(stream)), "qspec_gemm_w4a16_noalloc")
    return y


def noalloc_status(stream=None) -> int:
    """Device status of gemm_w4a16_noalloc on the current device (read and cleared)."""
    return int(LIB.qspec_gemm_w4a16_noalloc_status(_stream(stream)))


def spec_accept(p: torch.Tensor, q: torch.Tensor, draft: torch.Tensor, u_acc: torch.Tensor,
                u_res: torch.Tensor, n_accepted: torch.Tensor | None = None,
                tokens: torch.Tensor | None = None, work: torch.Tensor | None = None,
                stream=None):
    """Speculative accept / residual resample -> (n_accepted int32 [B], tokens int32 [B][gamma+1])."""
    _need(p, torch.float32, "p")
    _need(q, torch.float32, "q")
    _need(draft, torch.int32, "draft")
    _need(u_acc, torch.float32, "u_acc")
    _need(u_res, torch.float32, "u_res")
    b, g1, v = p.shape
    gamma = g1 - 1
    if n_accepted is None:
        n_accepted = torch.empty((b,), dtype=torch.int32, device=p.device)
    if tokens is None:
        tokens = torch.empty((b, gamma + 1), dtype=torch.int32, device=p.device)
    nbytes = 0 if work is None else work.numel()
    _check(LIB.qspec_spec_accept(_ptr(p), _ptr(q), _ptr(draft), _ptr(u_acc), _ptr(u_res), b, gamma,
                                 v, _ptr(n_accepted), _ptr(tokens), _ptr(work), nbytes,
                                 _stream(stream)), "qspec_spec_accept")
    return n_accepted, tokens


def spec_accept_greedy(p: torch.Tensor, draft: torch.Tensor, n_accepted: torch.Tensor | None = None,
                       tokens: torch.Tensor | None = None, work: torch.Tensor | None = None,
                       stream=None):
    """Greedy verification -> (n_accepted int32 [B], tokens int32 [B][gamma+1])."""
    _need(p, torch.float32, "p")
    _need(draft, torch.int32, "draft")
    b, g1, v = p.shape
    gamma = g1 - 1
    if n_accepted is None:
        n_accepted = torch.empty((b,), dtype=torch.int32, device=p.device)
    if tokens is None:
        tokens = torch.empty((b, gamma + 1), dtype=torch.int32, device=p.device)
    nbytes = 0 if work is None else work.numel()
    _check(LIB.qspec_spec_accept_greedy(_ptr(p), _ptr(draft), b, gamma, v, _ptr(n_accepted),
                                        _ptr(tokens), _ptr(work), nbytes, _stream(stream)),
           "qspec_spec_accept_greedy")
    return n_accepted, tokens


# ---------------------------------------------------------------- shared KV cache
def _kv_cache_check(k_cache: torch.Tensor, v_cache: torch.Tensor):
    for t, name in ((k_cache, "k_cache"), (v_cache, "v_cache")):
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous CUDA bf16 tensor [B][H_kv][L_max][128]")
    if k_cache.shape != v_cache.shape or k_cache.shape[3] != HEAD_DIM:
        raise ValueError("k_cache and v_cache must both be [B][H_kv][L_max][128]")
    b, h_kv, l_max, _ = k_cache.shape
    return b, h_kv, l_max


def _qkv_check(qkv: torch.Tensor):
    if not qkv.is_cuda or qkv.dtype != torch.float32 or qkv.dim() != 2 or qkv.stride(1) != 1:
        raise ValueError("qkv must be a CUDA fp32 [B*T][N] tensor with unit column stride")


def _tokens_per_sequence(qkv: torch.Tensor, batch: int) -> int:
    if qkv.shape[0] % batch != 0 or qkv.shape[0] == 0:
        raise ValueError(f"qkv has {qkv.shape[0]} rows, not a positive multiple of the batch {batch}")
    return qkv.shape[0] // batch


def attn_workspace_size(batch: int, t_new: int, h_q: int, h_kv: int, ctx_max: int) -> int:
    return int(LIB.qspec_attn_workspace_size(batch, t_new, h_q, h_kv, HEAD_DIM, ctx_max))


def kv_append(qkv: torch.Tensor, lens: torch.Tensor, offset: int, k_cache: torch.Tensor,
              v_cache: torch.Tensor, h_q: int, work: torch.Tensor | None = None, stream=None):
    """Write the new tokens' keys and values (rows b*T + t of the fused QKV output)
    into the caches at positions lens[b] + offset + t."""
    _qkv_check(qkv)
    _need(lens, torch.int32, "lens")
    b, h_kv, l_max = _kv_cache_check(k_cache, v_cache)
    t_new = _tokens_per_sequence(qkv, b)
    nbytes = 0 if work is None else work.numel()
    _check(LIB.qspec_kv_append(_ptr(qkv), qkv.stride(0), b, t_new, h_q, h_kv, HEAD_DIM, _ptr(lens),
                               offset, _ptr(k_cache), _ptr(v_cache), l_max, _ptr(work), nbytes,
                               _stream(stream)), "qspec_kv_append")


def attn_decode(qkv: torch.Tensor, lens: torch.Tensor, offset: int, k_cache: torch.Tensor,
                v_cache: torch.Tensor, h_q: int, ctx_max: int, out: torch.Tensor | None = None,
                work: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode attention of the new tokens over the shared cache -> fp32 [B*T][H*128]."""
    _qkv_check(qkv)
    _need(lens, torch.int32, "lens")
    b, h_kv, l_max = _kv_cache_check(k_cache, v_cache)
    t_new = _tokens_per_sequence(qkv, b)
    if out is None:
        out = torch.empty((b * t_new, h_q * HEAD_DIM), dtype=torch.float32, device=qkv.device)
    if work is None:
        work = workspace(attn_workspace_size(b, t_new, h_q, h_kv, ctx_max), qkv.device)
    _check(LIB.qspec_attn_decode(_ptr(qkv), qkv.stride(0), b, t_new, h_q, h_kv, HEAD_DIM,
                                 _ptr(lens), offset, _ptr(k_cache), _ptr(v_cache), l_max, ctx_max,
                                 _ptr(out), out.stride(0), _ptr(work), work.numel(),
                                 _stream(stream)), "qspec_attn_decode")
    return out


def kv_commit(lens: torch.Tensor, n_accepted: torch.Tensor, l_max: int,
              work: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """lens += n_accepted + 1 on the device (the round's accepted drafts plus one)."""
    _need(lens, torch.int32, "lens")
    _need(n_accepted, torch.int32, "n_accepted")
    nbytes = 0 if work is None else work.numel()
    _check(LIB.qspec_kv_commit(_ptr(lens), _ptr(n_accepted), lens.numel(), l_max, _ptr(work),
                               nbytes, _stream(stream)), "qspec_kv_commit")
    return lens
