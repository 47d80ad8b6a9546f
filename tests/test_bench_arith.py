"""The bench's roofline arithmetic against per-step work worked out
independently from the workload definitions (CPU only)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from block_text_diffusion_b200 import inputs as I  # noqa: E402


def test_flops_per_round_match_the_workload_definitions():
    # 26B shape: 2T(QKV + O + router + k experts) per layer, 4T Hq hd (P + 256)
    # attention per layer, 2TVd LM head, 2TVd + 2Td^2 self-conditioning: 1.91 TFLOP
    _, f = bench.round_work(I.MOE26B_BF16, 1, 2048, [128] * 30)
    assert f == pytest.approx(1.907e12, rel=1e-3)
    _, f = bench.round_work(I.MID_BF16, 1, 1024, [32] * 8)          # 108 GFLOP
    assert f == pytest.approx(108.0e9, rel=1e-3)
    _, f = bench.round_work(I.LONG_CTX, 1, 32768, [32] * 8)         # 374 GFLOP, 277 of them attention
    assert f == pytest.approx(374.3e9, rel=1e-3)


def test_bytes_per_round_with_every_expert_touched():
    # weights alone: 49.70 GB for the 26B shape (experts 128 x 3 x d x ff per
    # layer, attention, router, E twice, W_sc); the round adds the KV cache and
    # three passes over the fp32 logits plus the probabilities
    b, _ = bench.round_work(I.MOE26B_BF16, 1, 2048, [128] * 30)
    kv = 30 * 2 * 8 * (2048 + 256) * 128 * 2
    logits = 256 * 262144 * 4
    assert b == pytest.approx(49.704e9 + kv + 2 * logits + 256 * 262144 * 2 * 2, rel=1e-4)


def test_touched_experts_and_fp8_scale_the_expert_bytes():
    w = I.MOE26B_BF16
    full, _ = bench.round_work(w, 1, 2048, [128] * 30)
    few, _ = bench.round_work(w, 1, 2048, [8] * 30)
    expert = 3 * 2816 * 704 * 2
    assert full - few == pytest.approx(30 * 120 * expert, rel=1e-9)
    f8, _ = bench.round_work(w.replace(expert_fp8=True), 1, 2048, [128] * 30)
    assert full - f8 == pytest.approx(30 * 128 * 3 * 2816 * 704 * (2 - 1 - 4 / 128), rel=1e-9)
    assert bench.gate_up_bytes(w, 1, [21] * 30) > bench.gate_up_bytes(w.replace(expert_fp8=True), 1, [21] * 30)
