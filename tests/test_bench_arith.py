"""The bench's roofline arithmetic against per-step work worked out
independently from the workload definitions (CPU only)."""
import os
import sys

import numpy as np
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


def test_clock_record_parsing_flags_throttling():
    # nvidia-smi CSV (index, sm, max sm, power, active, hw, hw thermal, sw thermal, sw power cap)
    c = bench.Clocks(0)
    c.out = "\n".join([
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1905, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 345, 1965, 120.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, 1965, 1965, 710.0, 0x0000000000000000, Not Active, Active, Not Active, Not Active",
    ])
    s = c.summary()
    assert s["samples"] == 4 and s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1965.0                      # median of the loaded samples (idle 345 dropped)
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    c.out = ""
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_measured_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    import hashlib
    src_dir = tmp_path / "block_text_diffusion_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (src_dir / "dg_gemm.cuh").write_bytes(b"kernel v1")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(b"kernel v1").hexdigest()
    (tmp_path / "profiles" / "expert_gemm_mid_ncu.md").write_text(
        f"# x\n- dg_gemm.cuh sha256: {sha}\n- DRAM bytes / algorithmic bytes: 0.9\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic(1000.0) == pytest.approx(900.0)
    (src_dir / "dg_gemm.cuh").write_bytes(b"kernel v2")      # the kernel changed since the capture
    assert bench.measured_traffic(1000.0) is None


def test_routing_bias_generator_contract():
    b = I.routing_bias(3, 2, 512, 32, 4, pool=12, beta=8.0)
    assert b.shape == (2, 512, 32) and b.dtype.name == "float32"
    assert set(np.unique(b).tolist()) == {0.0, 8.0}
    assert np.all((b > 0).sum(axis=2) == 4)                       # top_k preferred experts per token
    for l in range(2):
        assert len(np.unique(np.nonzero(b[l])[1])) == 12          # all from a pool of 12
    assert np.array_equal(b, I.routing_bias(3, 2, 512, 32, 4, pool=12, beta=8.0))   # seeded
    with pytest.raises(ValueError):
        I.routing_bias(3, 2, 512, 32, 4, pool=3)
