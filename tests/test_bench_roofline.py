"""bench.py's roofline arithmetic on CPU: the FFN's algorithmic bytes and flop at the bench shapes,
the choice of the binding roofline, and the whole-job throughput, checked against figures worked
out by hand from the shapes (no GPU)."""
import numpy as np
import pytest

import bench
import workloads as W

PEAKS = {"hbm_gbs": 6532.5, "bf16_tflops": 1625.3, "bf16_tflops_sustained": 1400.0, "source": "measured"}


@pytest.fixture(autouse=True)
def fixed_peaks(monkeypatch):
    monkeypatch.setattr(bench, "peaks_all", lambda: dict(PEAKS))


def _offsets(rows_per_expert):
    return np.concatenate([[0], np.cumsum(rows_per_expert)]).astype(np.int64)


def test_switch_ffn_bytes_and_hbm_bound():
    cfg = W.CONFIGS["switch"]
    rows = np.full(128, 63)
    rows[:75] += 1  # 8139 kept rows over 128 experts, as in the bench run
    off = _offsets(rows)
    assert off[-1] == 8139
    # per expert: W1 768 x 3072 + W2 3072 x 768 + b1 3072 + b2 768, bf16 -> 9,444,864 bytes;
    # xbuf read and y written once: 8139 rows x 768 x 2 bytes x 2
    assert bench.ffn_algorithmic_bytes(cfg, off) == 128 * 9_444_864 + 8139 * 768 * 2 * 2 == 1_233_945_600
    r = bench.ffn_roofline(cfg, off, 0.2125)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6532.5
    assert r["achieved"] == pytest.approx(1_233_945_600 / 0.2125e-3 / 1e9)
    assert r["frac"] == pytest.approx(0.8889, abs=1e-4)
    assert r["flop_per_launch"] == 4.0 * 8139 * 768 * 3072


def test_empty_experts_carry_no_weight_bytes():
    cfg = W.CONFIGS["switch"]
    rows = np.zeros(128, dtype=np.int64)
    rows[5] = 10
    off = _offsets(rows)
    assert bench.ffn_algorithmic_bytes(cfg, off) == 9_444_864 + 10 * 768 * 4


def test_lossfree_ffn_is_tensor_bound():
    cfg = W.CONFIGS["lossfree"]
    off = _offsets(np.full(64, 1536))  # no capacity drop: 16384 x 6 picks spread evenly
    flops = 4.0 * 98304 * 2048 * 1408
    r = bench.ffn_roofline(cfg, off, 1.0255)
    # tensor time 1.134e12 / 1.6253e15 = 698 us > HBM time (0.74 GB of weights + 0.8 GB of rows) / 6.5 TB/s;
    # the fraction is of the burst peak, the sustained one beside it
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1625.3
    assert r["achieved"] == pytest.approx(flops / 1.0255e-3 / 1e12)
    assert 0.67 < r["frac"] < 0.69
    assert 0.78 < r["frac_of_sustained"] < 0.80


def test_global_capacity_factor_and_tensor_bound():
    cfg = W.CONFIGS["global"]
    # capacity 256 per expert per 4096-token micro-batch with k = 2 over 64 experts: factor 2.0
    assert bench.capacity_factor(cfg) == 2.0
    off = _offsets(np.full(64, 1024))  # 65536 kept rows
    r = bench.ffn_roofline(cfg, off, 2.0)
    # 4 x 65536 x 4096 x 4096 = 4.40e12 flop: 2.7 ms at the burst peak, against 4.3 GB + 1.07 GB of bytes (0.8 ms)
    assert r["bound"] == "tensor" and r["flop_per_launch"] == 4.0 * 65536 * 4096 * 4096
    assert r["frac"] == pytest.approx(4.0 * 65536 * 4096 * 4096 / 2.0e-3 / 1e12 / 1625.3)


def test_stage_bytes_dispatch_reads_each_token_once():
    cfg = W.CONFIGS["switch"]
    off = _offsets(np.full(128, 64))
    b = bench.stage_bytes(cfg, off, src_tokens_read=8192)
    assert b["dispatch"] == (8192 + 8192) * 768 * 2 + 8192 * 1 * 4
    assert b["router"] == 8192 * 768 * 2 + 768 * 128 * 4 + 8192 * 128 * 4 + 8192 * 1 * 8


def test_whole_job_throughput_counts_every_rank():
    # 4 ranks x 8192 tokens x 50 steps in 12.5 ms of the slowest rank
    assert bench.whole_job_tokens_per_s(8192, 50, 4, 12.5) == pytest.approx(8192 * 50 * 4 / 12.5e-3)
