"""Host-side checks that need no GPU: the C ABI library loads, exports every
symbol the header declares, and rejects bad arguments before launching."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qspec.h")


@pytest.fixture(scope="module")
def lib():
    from quantized_speculative_decoding_packed_b200 import build
    build.build()
    from quantized_speculative_decoding_packed_b200 import qspec
    return qspec


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:qspec_status|size_t|int32_t|const char\*)\s+(qspec_\w+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("qspec_quantize_weights", "qspec_quant_act", "qspec_gemm_w4a4",
                 "qspec_gemm_w4a16", "qspec_spec_accept", "qspec_workspace_size",
                 "qspec_workspace_status", "qspec_status_string", "qspec_abi_version",
                 "qspec_spec_accept_greedy", "qspec_gemm_w4a16_noalloc_status",
                 "qspec_gemm_w4a4_f32in", "qspec_gemm_w4a8_f32in", "qspec_kv_append",
                 "qspec_attn_decode", "qspec_attn_workspace_size", "qspec_kv_commit"):
        assert name in syms


def test_abi_version(lib):
    assert lib.LIB.qspec_abi_version() == lib.ABI_VERSION == 5


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(raw, name), name


def test_status_strings(lib):
    for code, text in [(0, b"ok"), (1, b"invalid argument"), (4, b"workspace too small"),
                       (5, b"kernel wait timed out")]:
        assert lib.LIB.qspec_status_string(code) == text


FAKE = ctypes.c_void_p(0x10000)      # 16-byte aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("args", [
    (None, 4, 256, 64, FAKE, FAKE, None),            # null input
    (FAKE, 4, 256, 32, FAKE, FAKE, None),            # unsupported group
    (FAKE, 4, 200, 64, FAKE, FAKE, None),            # k not a multiple of group
    (FAKE, 0, 256, 64, FAKE, FAKE, None),            # empty
])
def test_quantize_weights_rejects(lib, args):
    assert lib.LIB.qspec_quantize_weights(*args) == 1


@pytest.mark.parametrize("m,k,n,group", [(0, 256, 256, 64), (4, 200, 256, 64), (4, 256, 0, 64),
                                         (4, 256, 256, 96), (4, 64, 256, 64)])
def test_gemm_rejects_bad_shapes(lib, m, k, n, group):
    assert lib.LIB.qspec_gemm_w4a4(FAKE, m, k, FAKE, FAKE, n, group, FAKE, FAKE, 1 << 30, None,
                                   0, None) == 1
    assert lib.LIB.qspec_gemm_w4a16(FAKE, m, k, FAKE, FAKE, n, group, FAKE, FAKE, 1 << 30,
                                    0, None) == 1


def test_gemm_rejects_misaligned_pointers(lib):
    odd = ctypes.c_void_p(0x10008)
    assert lib.LIB.qspec_gemm_w4a16(odd, 4, 256, FAKE, FAKE, 256, 64, FAKE, FAKE, 1 << 30, 0, None) == 1
    assert lib.LIB.qspec_gemm_w4a16(FAKE, 4, 256, odd, FAKE, 256, 64, FAKE, FAKE, 1 << 30, 0, None) == 1
    assert lib.LIB.qspec_gemm_w4a16(FAKE, 4, 256, FAKE, FAKE, 256, 64, FAKE, None, 1 << 30, 0, None) == 1


def test_gemm_rejects_reserved_flags(lib):
    # a valid-looking call (aligned fake pointers, a supported shape) with a reserved bit set
    assert lib.LIB.qspec_gemm_w4a16(FAKE, 4, 256, FAKE, FAKE, 256, 64, FAKE, FAKE, 1 << 30, 2, None) == 1
    assert lib.LIB.qspec_gemm_w4a4(FAKE, 4, 256, FAKE, FAKE, 256, 64, FAKE, FAKE, 1 << 30, None,
                                   0x80000000, None) == 1
    assert lib.LIB.qspec_gemm_w4a16_noalloc(FAKE, 4, 256, FAKE, FAKE, 256, 64, FAKE, 4, None) == 1


@pytest.mark.parametrize("fn", ["qspec_gemm_w4a4_f32in", "qspec_gemm_w4a8_f32in"])
def test_f32_input_gemm_rejects(lib, fn):
    f = getattr(lib.LIB, fn)
    ok = (FAKE, 256, 4, 256, FAKE, FAKE, 256, 64, FAKE, FAKE, 1 << 30, None)
    assert f(FAKE, 252, *ok[2:], 0, None) == 1            # ldx < k
    assert f(FAKE, 258, *ok[2:], 0, None) == 1            # ldx not a multiple of 4
    assert f(ctypes.c_void_p(0x10008), *ok[1:], 0, None) == 1   # x not 16-byte aligned
    assert f(None, *ok[1:], 0, None) == 1                 # no input
    assert f(*ok, 2, None) == 1                           # QSPEC_GEMM_FUSED_QUANT not accepted here
    assert f(FAKE, 256, 4, 255, *ok[4:], 0, None) == 1    # k not a multiple of the group


@pytest.mark.parametrize("b,g,v", [(0, 4, 32), (2, 0, 32), (2, 17, 32), (2, 4, 30), (2, 4, 0),
                                   (2, 4, 409604)])
def test_accept_rejects(lib, b, g, v):
    assert lib.LIB.qspec_spec_accept(FAKE, FAKE, FAKE, FAKE, FAKE, b, g, v, FAKE, FAKE, None, 0,
                                     None) == 1


def test_quant_act_rejects(lib):
    assert lib.LIB.qspec_quant_act(FAKE, 4, 12, FAKE, FAKE, None) == 1
    assert lib.LIB.qspec_quant_act(FAKE, 0, 16, FAKE, FAKE, None) == 1
    assert lib.LIB.qspec_quant_act(None, 4, 16, FAKE, FAKE, None) == 1


def test_workspace_size_of_invalid_shapes_is_zero(lib):
    assert lib.workspace_size(lib.OP_GEMM_W4A4, 4, 256, 200, 64) == 0
    assert lib.workspace_size(lib.OP_QUANT_ACT, 4, 0, 256) == 0
    assert lib.workspace_size(lib.OP_SPEC_ACCEPT, batch=2, gamma=4, vocab=32) == 256


def test_stream_k_schedule_invariants(tmp_path):
    """Compile the scheduling helpers of the GEMM for the host and check the
    partition, ticket and partial-slot invariants over many shapes."""
    import subprocess
    from quantized_speculative_decoding_packed_b200 import build as b
    exe = tmp_path / "schedule_check"
    src = os.path.join(ROOT, "tests", "schedule_check.cu")
    cmd = [b.nvcc(), "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", b.INCLUDE, "-I", b.CSRC, "-o", str(exe), src]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0 and run.stdout.startswith("ok"), run.stdout


@pytest.mark.parametrize("b,g,v", [(0, 4, 32), (2, 0, 32), (2, 17, 32), (2, 4, 30), (2, 4, 0)])
def test_greedy_accept_rejects(lib, b, g, v):
    assert lib.LIB.qspec_spec_accept_greedy(FAKE, FAKE, b, g, v, FAKE, FAKE, None, 0, None) == 1
    assert lib.LIB.qspec_spec_accept_greedy(None, FAKE, 2, 4, 32, FAKE, FAKE, None, 0, None) == 1


def test_attn_workspace_size_closed_form(lib):
    # batch 2, 3 new tokens, 4 query heads over 2 KV heads (6 rows per KV head),
    # context 300 (3 chunks of 128 keys): 256-byte status block, 4 counters,
    # 2x2x3x6 (max, sum) pairs, 2x2x3x6 rows of 128 floats, each part 256-aligned
    assert lib.attn_workspace_size(2, 3, 4, 2, 300) == 256 + 256 + 768 + 36864
    assert lib.attn_workspace_size(2, 3, 4, 2, 32768) > 0
    assert lib.attn_workspace_size(2, 3, 4, 2, 32769) == 0      # past 256 chunks
    assert lib.attn_workspace_size(2, 9, 8, 2, 300) == 0        # 36 rows per KV head
    assert lib.attn_workspace_size(2, 3, 6, 4, 300) == 0        # 6 heads over 4 KV heads
    assert lib.LIB.qspec_attn_workspace_size(2, 3, 4, 2, 64, 300) == 0   # head_dim 64


def _attn(lib, **kw):
    a = dict(qkv=FAKE, ld=1024, b=2, t=3, hq=4, hkv=2, d=128, lens=FAKE, off=0, kc=FAKE, vc=FAKE,
             lmax=512, ctx=300, out=FAKE, ldo=512, ws=FAKE, nb=1 << 30)
    a.update(kw)
    return lib.LIB.qspec_attn_decode(a["qkv"], a["ld"], a["b"], a["t"], a["hq"], a["hkv"], a["d"],
                                     a["lens"], a["off"], a["kc"], a["vc"], a["lmax"], a["ctx"],
                                     a["out"], a["ldo"], a["ws"], a["nb"], None)


def test_attn_decode_rejects(lib):
    odd = ctypes.c_void_p(0x10008)
    assert _attn(lib, d=64) == 1                     # head_dim other than 128
    assert _attn(lib, hq=6) == 1                     # query heads not a multiple of KV heads
    assert _attn(lib, t=9, hq=8) == 1                # 36 rows per KV head
    assert _attn(lib, ld=1020) == 1                  # row stride below (4 + 2*2) * 128
    assert _attn(lib, ld=1026) == 1                  # row stride not a multiple of 4
    assert _attn(lib, ldo=500) == 1                  # output stride below 4 * 128
    assert _attn(lib, ctx=513) == 1                  # context past the cache
    assert _attn(lib, ctx=0) == 1
    assert _attn(lib, off=-1) == 1
    assert _attn(lib, kc=odd) == 1                   # cache not 16-byte aligned
    assert _attn(lib, qkv=None) == 1
    assert _attn(lib, ws=None) == 1
    assert _attn(lib, nb=1024) == 4                  # workspace too small


def test_kv_append_and_commit_reject(lib):
    f = lib.LIB.qspec_kv_append
    ok = [FAKE, 1024, 2, 3, 4, 2, 128, FAKE, 0, FAKE, FAKE, 512, None, 0, None]
    bad = [(6, 64), (4, 6), (1, 1020), (8, -1), (11, 0), (0, None), (9, ctypes.c_void_p(0x10008))]
    for i, v in bad:
        args = list(ok)
        args[i] = v
        assert f(*args) == 1, (i, v)
    assert f(*(ok[:12] + [FAKE, 64, None])) == 1       # a workspace below 256 bytes
    assert lib.LIB.qspec_kv_commit(FAKE, FAKE, 0, 512, None, 0, None) == 1
    assert lib.LIB.qspec_kv_commit(None, FAKE, 2, 512, None, 0, None) == 1
    assert lib.LIB.qspec_kv_commit(FAKE, FAKE, 2, 0, None, 0, None) == 1


def test_kv_binding_checks_its_tensors(lib):
    import torch
    qkv = torch.zeros((4, 8 * 128))
    lens = torch.zeros(2, dtype=torch.int32)
    cache = torch.zeros((2, 2, 16, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="qkv"):
        lib.attn_decode(qkv, lens, 0, cache, cache, 4, 16)          # host tensors
    with pytest.raises(ValueError, match="qkv"):
        lib.kv_append(qkv.half(), lens, 0, cache, cache, 4)
    with pytest.raises(ValueError):
        lib.kv_commit(lens, lens.long(), 16)
