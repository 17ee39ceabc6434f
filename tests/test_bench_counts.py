"""The work counts behind bench.py's throughput and roofline figures, against values
computed by hand from the layouts (packed INT4 weights, fp16 group scales, int8 or bf16
activations as the GEMM reads them, fp32 outputs)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_gate_up_draft_call_bytes():
    # N = 22016, K = 4096, M = 16, group 128
    packed = 22016 * 4096 // 2            # 45,088,768
    scales = 22016 * (4096 // 128) * 2    # 1,409,024
    acts = 16 * 4096                      # int8 activations: 65,536
    out = 16 * 22016 * 4                  # 1,409,024
    assert bench.gemm_bytes(16, 22016, 4096, "w4a4") == packed + scales + acts + out == 47_972_352


def test_verify_call_reads_bf16_activations():
    n, k = 4096, 11008
    w = n * k // 2 + n * (k // 128) * 2
    assert bench.gemm_bytes(80, n, k, "w4a16") == w + 80 * k * 2 + 80 * n * 4
    assert bench.packed_bytes(n, k) == w


def test_step_work_is_gamma_drafts_plus_one_verify_per_layer():
    b, ops = bench.step_work(1)
    want_b = sum(4 * bench.gemm_bytes(16, n, k, "w4a4") + bench.gemm_bytes(80, n, k, "w4a16")
                 for _, n, k in bench.LAYERS)
    want_ops = sum(4 * 2 * 16 * n * k + 2 * 80 * n * k for _, n, k in bench.LAYERS)
    assert (b, ops) == (want_b, want_ops)
    b32, ops32 = bench.step_work(32)
    assert (b32, ops32) == (32 * b, 32 * ops)
    # packed weights of one layer: QKV + o_proj + gate+up + down
    packed = sum(bench.packed_bytes(n, k) for _, n, k in bench.LAYERS)
    assert packed == (12288 * 4096 + 4096 * 4096 + 22016 * 4096 + 4096 * 11008) // 2 + \
        (12288 * 32 + 4096 * 32 + 22016 * 32 + 4096 * 86) * 2


@pytest.mark.parametrize("gamma,vocab", [(4, 32000), (5, 128256)])
def test_accept_bytes_closed_forms(gamma, vocab):
    out = (gamma + 2) * 4                 # accepted count + tokens row
    reject_first = 1 * 2 * 4 + 2 * vocab * 4 + out      # one tested position, p and q rows
    accept_all = gamma * 2 * 4 + vocab * 4 + out        # gamma tested, one p row (bonus)
    reject_last = gamma * 2 * 4 + 2 * vocab * 4 + out   # n = gamma - 1: all tested, p and q rows
    assert bench.accept_bytes([0], gamma, vocab) == reject_first
    assert bench.accept_bytes([gamma], gamma, vocab) == accept_all
    assert bench.accept_bytes([gamma - 1], gamma, vocab) == reject_last
    assert bench.accept_bytes([0, gamma], gamma, vocab) == reject_first + accept_all


@pytest.mark.parametrize("gamma,vocab", [(4, 32000), (5, 128256)])
def test_greedy_bytes_closed_forms(gamma, vocab):
    out = (gamma + 2) * 4
    first_mismatch = 1 * 4 + 1 * vocab * 4 + out          # draft 0 compared, row 0 read
    all_match = gamma * 4 + (gamma + 1) * vocab * 4 + out  # every draft compared, rows 0..gamma
    assert bench.greedy_bytes([0], gamma, vocab) == first_mismatch
    assert bench.greedy_bytes([gamma], gamma, vocab) == all_match
    assert bench.greedy_bytes([0, gamma], gamma, vocab) == first_mismatch + all_match


def test_job_throughput_is_whole_job():
    one = bench.job_throughput(1e9, 1, 10.0)
    assert one == pytest.approx(100.0)                  # 1 GB in 10 ms = 100 GB/s
    assert bench.job_throughput(1e9, 8, 10.0) == pytest.approx(8 * one)


def test_attention_bytes_closed_forms():
    import bench
    # batch 16 at length 1024, one new token, 32 heads of 128 (no grouping): 1025
    # keys and values of 256 bytes per head and sequence, plus fp32 query and output rows
    assert bench.attn_bytes([1024] * 16, 0, 1, 32, 32) == 16 * 1025 * 32 * 512 + 2 * 16 * 32 * 512
    # grouped: 8 KV heads serve 32 query heads; 5 new tokens at offset 2
    assert bench.attn_bytes([100, 200], 2, 5, 32, 8) == (107 + 207) * 8 * 512 + 2 * 2 * 5 * 32 * 512
    assert bench.append_bytes(16, 5, 32) == 16 * 5 * 2 * 32 * 128 * 6
