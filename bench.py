"""Benchmark of the denoising hot path on B200.

A bench "step" is one full block: dg_generate_block over B canvases (uniform
noise, denoising rounds on the device until every canvas stops or the round
budget ends), i.e. one pass of every hot-path stage.  The metric is denoise
rounds per second (and committed canvas tokens per second) of the whole job.

Default workload: the 26B-A4B-shaped MoE (30 layers, d 2816, 128 experts
top-8, vocab 262144) with one canvas and a 2048-token random prompt.
Multi-GPU (torchrun): every rank runs an independent replica on its own
canvases (no data-path collective); rank 0 reports the sum of rounds over
the max time.  `--impl reference` times the CPU oracle instead, on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "committed canvas tokens/s and denoise steps/s at 1 B200; % of step roofline"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="moe26b")
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-reps", type=int, default=3)
    ap.add_argument("--max-rounds", type=int, default=None,
                    help="override the round budget (short runs for profiler launch lists)")
    ap.add_argument("--no-fast-converging", action="store_true",
                    help="skip the committed-tokens measurement on the fast-converging workload")
    ap.add_argument("--expert-fp8", action="store_true",
                    help="expert weights as E4M3 codes with per-128-input power-of-two scales")
    ap.add_argument("--topk-study", action="store_true",
                    help="also compare exact and top-k-truncated sampling at batch 32 (mid workload)")
    ap.add_argument("--routing-study", action="store_true",
                    help="also sweep a structured router bias over expert-pool sizes (routing locality)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the throughput lines of the other workloads")
    return ap.parse_args()


def measured_traffic(algorithmic_bytes):
    """DRAM bytes per launch of the expert gate|up GEMM from the committed ncu
    summary (captured on the mid workload and scaled by its measured ratio of
    DRAM bytes to algorithmic bytes); None when the GEMM source changed since
    the capture."""
    import hashlib
    src = os.path.join(ROOT, "block_text_diffusion_b200", "csrc", "dg_gemm.cuh")
    summ = os.path.join(ROOT, "profiles", "expert_gemm_mid_ncu.md")
    try:
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        fields = {}
        with open(summ) as f:
            for line in f:
                if line.startswith("- ") and ": " in line:
                    k, v = line[2:].split(": ", 1)
                    fields[k.strip()] = v.strip()
        if fields.get("dg_gemm.cuh sha256") != sha:
            return None
        return algorithmic_bytes * float(fields["DRAM bytes / algorithmic bytes"])
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# --- algorithmic work of one round (bytes and FLOPs) ------------------------------------
def round_work(w, B, P, touched):
    """Bytes and FLOPs of one denoising round for B canvases.  `touched` is the
    list of distinct experts routed to in each layer (measured)."""
    esz = 2 if w.dtype == 1 else 4
    d, V, L, hd = w.d_model, w.vocab, w.n_layers, w.head_dim
    nq, nk = w.n_heads * hd, w.n_kv_heads * hd
    T = B * 256
    attn_w = (d * (nq + 2 * nk) + nq * d) * esz
    expert = 3 * d * w.d_ff * expert_weight_bytes(w)
    kv = 2 * B * w.n_kv_heads * (P + 256) * hd * esz
    per_layer = attn_w + w.n_experts * d * esz + kv
    logits = T * V * 4
    bytes_ = (L * per_layer + sum(touched) * expert + 2 * V * d * esz + d * d * esz + 2 * logits
              + T * V * esz * 2)
    flops = L * (2 * T * (d * (nq + 2 * nk) + nq * d + w.n_experts * d + w.top_k * 3 * d * w.d_ff)
                 + 4 * T * w.n_heads * hd * (P + 256)) + 2 * T * V * d * 2 + 2 * T * d * d
    return bytes_, flops


def expert_weight_bytes(w):
    """Bytes per expert weight: the storage dtype, or an E4M3 code plus its
    share of a 4-byte scale per 128 inputs."""
    if getattr(w, "expert_fp8", False):
        return 1.0 + 4.0 / 128.0
    return 2 if w.dtype == 1 else 4


def gate_up_bytes(w, B, touched):
    """Algorithmic bytes of one expert gate|up GEMM launch, averaged over the
    layers: touched experts' gate and up weights, the gathered rows read, and
    the method's output -- the SwiGLU activation, one value per (row, hidden
    unit) in the storage dtype."""
    esz = 2 if w.dtype == 1 else 4
    rows = B * 256 * w.top_k
    avg = sum(touched) / len(touched)
    return avg * 2 * w.d_ff * w.d_model * expert_weight_bytes(w) + rows * w.d_model * esz + rows * w.d_ff * esz


class Clocks:
    """nvidia-smi sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev):
        self.dev = dev
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.Q,
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.p:
            time.sleep(0.25)
            self.p.terminate()
            try:
                self.out, _ = self.p.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
                self.out = ""

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        load = [s for s in sm if mx and s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def reduce_over_ranks(times, work, world, device):
    """Whole-job numbers: the max of each time over ranks (the job ends when
    the slowest rank ends) and the sum of each work count."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(times, dtype=torch.float64, device=device)
    w = torch.tensor(work, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()], [int(x) for x in w.tolist()]


# --- our arm ------------------------------------------------------------------------------
def run_ours(a):
    import numpy as np
    import torch
    import torch.distributed as dist

    import block_text_diffusion_b200 as dg
    from block_text_diffusion_b200 import inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=600))
    w = I.WORKLOADS[a.workload]
    B = a.batch or w.batch
    P = w.prompt_len
    w = w.replace(sample_seed=w.sample_seed + 1000 * rank)
    if a.max_rounds:
        w = w.replace(max_steps=a.max_rounds)
    if a.expert_fp8:
        w = w.replace(name=w.name + "-fp8experts", expert_fp8=True)
    model = dg.Model(w, max_canvases=B, max_prompt=P)
    stream = torch.cuda.current_stream()
    prompt_h = torch.from_numpy(I.prompt_ids(w.sample_seed, B, P, w.vocab)).pin_memory()
    prompt_d = prompt_h.cuda()
    kv = model.new_kv(B, P)
    model.encode_prompt(prompt_d, kv)
    canvas = torch.zeros((B, 256), dtype=torch.int32, device="cuda")
    steps = torch.zeros(B, dtype=torch.int32, device="cuda")
    ncom = torch.zeros(B, dtype=torch.int32, device="cuda")

    def block():
        model.generate_block(kv, B, P, canvas, steps, ncom)

    for _ in range(a.warmup):
        block()
    model.sync_status()
    torch.cuda.synchronize()

    # timed region: device events, barrier on both sides
    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    rounds = torch.zeros((), dtype=torch.int64, device="cuda")
    loop_rounds = torch.zeros((), dtype=torch.int64, device="cuda")
    committed = torch.zeros((), dtype=torch.int64, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    model.reset_touched_experts()
    barrier()
    with Clocks(local) as clk:
        e0.record(stream)
        for _ in range(a.steps):
            block()
            rounds += steps.sum()
            loop_rounds += steps.max()
            committed += ncom.sum()
        e1.record(stream)
        barrier()
    ms = e0.elapsed_time(e1)
    model.sync_status()
    n_rounds, n_com = int(rounds.item()), int(committed.item())
    # distinct experts each layer streamed, averaged over every round of the
    # timed blocks (counted on the device)
    n_loop_rounds = int(loop_rounds.item())
    touched = [t / max(1, n_loop_rounds) for t in model.touched_experts_sum(reset=True)]

    # end to end through the public API with host buffers
    canvas_h = torch.zeros((B, 256), dtype=torch.int32).pin_memory()
    steps_h = torch.zeros(B, dtype=torch.int32).pin_memory()
    ncom_h = torch.zeros(B, dtype=torch.int32).pin_memory()
    e_rounds = 0
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    f0.record(stream)
    for _ in range(a.steps):
        prompt_d.copy_(prompt_h, non_blocking=True)
        model.encode_prompt(prompt_d, kv)
        block()
        canvas_h.copy_(canvas, non_blocking=True)
        steps_h.copy_(steps, non_blocking=True)
        ncom_h.copy_(ncom, non_blocking=True)
    f1.record(stream)
    barrier()
    e2e_ms = f0.elapsed_time(f1)
    e_rounds = int(steps_h.sum()) * a.steps

    # per-kernel timing (CUDA events around each launch of single rounds)
    prof = model.profile_step(kv, B, P, reps=a.profile_reps)

    study = None
    if a.routing_study:
        study = routing_study(dg, I, torch, model, w, kv, B, P, block, steps)
    topk = None
    if a.topk_study and world == 1:
        topk = topk_study(dg, I, torch)

    # throughput and roofline fraction of the other workloads: single-GPU runs only
    configs = None
    if world == 1 and not a.no_per_config:
        configs = per_config(dg, I, torch)

    # committed tokens on the fast-converging workload (logit scale 16), where
    # random-init weights still commit: single-GPU runs only
    fast = None
    if world == 1 and not a.no_fast_converging:
        fast = fast_converging(dg, I, torch)
        try:
            fast["block_autoregressive"] = block_autoregressive(dg, I, torch)
        except dg.DGError as e:   # reported, never fatal to the main line
            fast["block_autoregressive"] = {"error": str(e)}

    (ms, e2e_ms), (n_rounds, n_com, e_rounds) = reduce_over_ranks(
        [ms, e2e_ms], [n_rounds, n_com, e_rounds], world, "cuda")
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        model.close()
        return None

    hbm, tf, tf_sus, src = peaks()
    per_round_ms = ms / max(1, n_rounds / world)
    b_round, f_round = round_work(w, B, P, touched)
    step_roof_ms = max(b_round / (hbm * 1e9), f_round / (tf_sus * 1e12)) * 1e3
    gu_ms, gu_n = prof["expert_gate_up_gemm"]
    gu_avg = gu_ms / max(1, gu_n)
    gu_bytes = gate_up_bytes(w, B, touched)
    achieved = gu_bytes / (gu_avg * 1e-3) / 1e9
    # kernels of one captured round (counted at capture), and the loop-state
    # initialisation kernel launched before each block
    kper = model.launches_per_round()
    line = {
        "metric": METRIC,
        "value": n_rounds / (ms * 1e-3),
        "unit": "denoise steps/s",
        "n_gpus": world,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": ms / a.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == 1 else "f32",
        "data": "synthetic (random-init weights from Philox seed, random prompt ids)",
        "config": {"workload": w.name, "canvases_per_gpu": B, "prompt_len": P, "max_rounds": w.max_steps,
                   "rounds_per_step": n_rounds / world / a.steps,
                   "l2": "inputs larger than L2: every round streams all touched weights (%.1f GB)" % (b_round / 1e9),
                   "parallelism": "replicas" if world > 1 else "single"},
        "committed_tokens_per_s": n_com / (ms * 1e-3),
        "ms_per_round": per_round_ms,
        "step_roofline": {"bound": "hbm" if b_round / hbm > f_round / tf_sus / 1e3 else "tensor",
                          "roof_ms": step_roof_ms, "frac": step_roof_ms / per_round_ms,
                          "bytes": b_round, "flops": f_round,
                          "touched_experts_mean_over_timed_rounds": [round(t, 2) for t in touched]},
        "roofline": {"bound": "hbm", "kernel": "expert_gate_up_gemm", "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm,
                     # the committed capture is of the bf16 expert GEMM: no ratio for the FP8 kernel
                     "traffic": None if getattr(w, "expert_fp8", False) else measured_traffic(gu_bytes),
                     "peak_source": src, "avg_launch_ms": gu_avg, "algorithmic_bytes": gu_bytes},
        "phases_ms_per_round": {k: v[0] / a.profile_reps for k, v in prof.items() if v[1]},
        "e2e": {"value": e_rounds / (e2e_ms * 1e-3), "unit": "denoise steps/s",
                "h2d_bytes_per_step": B * P * 4 * world, "d2h_bytes_per_step": (B * 256 + 2 * B) * 4 * world,
                "includes": "prompt H2D, causal prompt encode, block loop, result D2H"},
        "per_config": configs,
        "fast_converging": fast,
        "routing_study": study,
        "topk_study": topk,
        "gpu_launches": int(n_loop_rounds * kper + a.steps) * world,
        "clocks": clk.summary(),
    }
    model.close()
    return line


def per_config(dg, I, torch, blocks=2):
    """Rounds per second, committed tokens per second and the step-roofline
    fraction of the workloads beside the headline one, each at its own bound
    (HBM copy peak, or the sustained bf16 tensor peak where the round's FLOPs
    dominate): the tiny fp32 decoder, the mid MoE, the Zipf-routed batch
    workload at 1, 4, 8 and 32 canvases (2048-token prompts each) and the
    long-context workload.  Device events around `blocks` full blocks after
    one warm-up block; touched experts counted on the device over the timed
    rounds."""
    hbm, _, tf_sus, _ = peaks()
    stream = torch.cuda.current_stream()
    cases = [("tiny", I.TINY_FP32, 1), ("mid", I.MID_BF16, 1)]
    cases += [("batch_B%d" % b, I.BATCH_ZIPF, b) for b in I.BATCH_SIZES]
    cases += [("long", I.LONG_CTX, 1)]
    out = {}
    for key, w, B in cases:
        P = w.prompt_len
        model = dg.Model(w, max_canvases=B, max_prompt=P)
        try:
            kv = model.new_kv(B, P)
            model.encode_prompt(torch.from_numpy(I.prompt_ids(w.sample_seed, B, P, w.vocab)).cuda(), kv)
            z = lambda *shape: torch.zeros(shape, dtype=torch.int32, device="cuda")
            canvas, steps, ncom = z(B, 256), z(B), z(B)
            model.generate_block(kv, B, P, canvas, steps, ncom)
            torch.cuda.synchronize()
            model.reset_touched_experts()
            rounds = torch.zeros((), dtype=torch.int64, device="cuda")
            loop_rounds = torch.zeros((), dtype=torch.int64, device="cuda")
            committed = torch.zeros((), dtype=torch.int64, device="cuda")
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(blocks):
                model.generate_block(kv, B, P, canvas, steps, ncom)
                rounds += steps.sum()
                loop_rounds += steps.max()
                committed += ncom.sum()
            e1.record(stream)
            torch.cuda.synchronize()
            model.sync_status()
            ms = e0.elapsed_time(e1)
            n_loop = max(1, int(loop_rounds.item()))
            touched = [t / n_loop for t in model.touched_experts_sum(reset=True)]
        finally:
            model.close()
        b_round, f_round = round_work(w, B, P, touched)
        t_hbm, t_tc = b_round / (hbm * 1e9) * 1e3, f_round / (tf_sus * 1e12) * 1e3
        ms_round = ms / n_loop
        out[key] = {"workload": w.name, "canvases": B, "prompt_len": P,
                    "denoise_steps_per_s": int(rounds.item()) / (ms * 1e-3),
                    "committed_tokens_per_s": int(committed.item()) / (ms * 1e-3),
                    "ms_per_round": ms_round, "rounds_per_block": n_loop / blocks,
                    "step_roofline": {"bound": "hbm" if t_hbm >= t_tc else "tensor", "roof_ms": max(t_hbm, t_tc),
                                      "frac": max(t_hbm, t_tc) / ms_round, "bytes": b_round, "flops": f_round,
                                      "touched_experts_mean": sum(touched) / len(touched)}}
    return out


def fast_converging(dg, I, torch, blocks=3):
    """Committed canvas tokens per second of full blocks on the long-context
    workload (32768-token prompt, logit scale 16), timed with device events."""
    w = I.LONG_CTX
    P = w.prompt_len
    model = dg.Model(w, max_canvases=1, max_prompt=P)
    stream = torch.cuda.current_stream()
    kv = model.new_kv(1, P)
    model.encode_prompt(torch.from_numpy(I.prompt_ids(w.sample_seed, 1, P, w.vocab)).cuda(), kv)
    canvas = torch.zeros((1, 256), dtype=torch.int32, device="cuda")
    steps = torch.zeros(1, dtype=torch.int32, device="cuda")
    ncom = torch.zeros(1, dtype=torch.int32, device="cuda")
    model.generate_block(kv, 1, P, canvas, steps, ncom)
    torch.cuda.synchronize()
    rounds = torch.zeros((), dtype=torch.int64, device="cuda")
    committed = torch.zeros((), dtype=torch.int64, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(blocks):
        model.generate_block(kv, 1, P, canvas, steps, ncom)
        rounds += steps.sum()
        committed += ncom.sum()
    e1.record(stream)
    torch.cuda.synchronize()
    model.sync_status()
    ms = e0.elapsed_time(e1)
    model.close()
    n_r, n_c = int(rounds.item()), int(committed.item())
    return {"workload": w.name, "prompt_len": P, "blocks": blocks, "committed_tokens_per_s": n_c / (ms * 1e-3),
            "committed_per_block": n_c / blocks, "rounds_per_block": n_r / blocks, "ms_per_block": ms / blocks}


def routing_study(dg, I, torch, model, w, kv, B, P, block, steps, pools=(8, 16, 32, 64, 84, 128), beta=8.0,
                  reps=2):
    """Routing locality: a structured per-token router bias confines each
    layer's canvas tokens to a pool of experts (each token prefers top_k of
    them, bias `beta`).  Per pool size: the distinct experts the layers
    touched, ms per round, the step roofline and its fraction, and the expert
    gate|up GEMM's achieved bandwidth."""
    stream = torch.cuda.current_stream()
    hbm, _, tf_sus, _ = peaks()
    out = []
    for pool in pools:
        if not w.top_k <= pool <= w.n_experts:
            continue
        bias = torch.from_numpy(I.routing_bias(7, w.n_layers, B * 256, w.n_experts, w.top_k, pool, beta)).cuda()
        model.set_routing_bias(bias)
        try:
            block()                                   # recapture + warm-up
            torch.cuda.synchronize()
            rounds = torch.zeros((), dtype=torch.int64, device="cuda")
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                block()
                rounds += steps.sum()
            e1.record(stream)
            torch.cuda.synchronize()
            ms_round = e0.elapsed_time(e1) / max(1, int(rounds.item()))
            prof = model.profile_step(kv, B, P, reps=2)
            touched = model.touched_experts()
        finally:
            model.set_routing_bias(None)
        model.sync_status()
        b_round, f_round = round_work(w, B, P, touched)
        roof = max(b_round / (hbm * 1e9), f_round / (tf_sus * 1e12)) * 1e3
        gu_ms, gu_n = prof["expert_gate_up_gemm"]
        dn_ms = prof["expert_down_gemm"][0]
        gu_gbs = gate_up_bytes(w, B, touched) / (gu_ms / max(1, gu_n) * 1e-3) / 1e9
        out.append({"pool": pool, "touched_mean": sum(touched) / len(touched), "ms_per_round": ms_round,
                    "roof_ms": roof, "frac": roof / ms_round, "expert_ms_per_round": (gu_ms + dn_ms) / 2,
                    "gate_up_gbs": gu_gbs, "gate_up_frac": gu_gbs / hbm})
    return out


def topk_study(dg, I, torch, K=64, B=32, reps=2):
    """Exact vs top-k-truncated sampling on the Zipf-routed batch workload
    (mid architecture, 2048-token prompts) at B canvases: ms per round of the
    device block loop, and the sampler and self-conditioning phases of single
    rounds (CUDA events around each launch)."""
    base = I.BATCH_ZIPF
    P = base.prompt_len
    stream = torch.cuda.current_stream()
    prompt = torch.from_numpy(I.prompt_ids(base.sample_seed, B, P, base.vocab)).cuda()
    out = {"workload": base.name, "canvases": B, "K": K}
    for name, w in (("exact", base), ("topk", base.replace(sample_topk=K))):
        model = dg.Model(w, max_canvases=B, max_prompt=P)
        kv = model.new_kv(B, P)
        model.encode_prompt(prompt, kv)
        z = lambda *shape: torch.zeros(shape, dtype=torch.int32, device="cuda")
        canvas, steps, ncom = z(B, 256), z(B), z(B)
        model.generate_block(kv, B, P, canvas, steps, ncom)
        torch.cuda.synchronize()
        rounds = torch.zeros((), dtype=torch.int64, device="cuda")
        committed = torch.zeros((), dtype=torch.int64, device="cuda")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            model.generate_block(kv, B, P, canvas, steps, ncom)
            rounds += steps.max()          # the loop runs until the last canvas stops
            committed += ncom.sum()
        e1.record(stream)
        torch.cuda.synchronize()
        model.sync_status()
        n_r = max(1, int(rounds.item()))
        prof = model.profile_step(kv, B, P, reps=2)
        ph = {k: v[0] / 2 for k, v in prof.items() if v[1]}
        out[name] = {"ms_per_round": e0.elapsed_time(e1) / n_r,
                     "committed_per_round": int(committed.item()) / n_r,
                     "sampler_ms": ph.get("sampler", 0.0),
                     "selfcond_ms": ph.get("selfcond_gemm", 0.0) + ph.get("selfcond_round", 0.0)}
        model.close()
    return out


def block_autoregressive(dg, I, torch, blocks=3):
    """Chained blocks through dg_generate on the long-context workload: each
    finished canvas is encoded causally into the cache and the next canvas
    starts after it.  A 1-block call and a (1 + blocks)-block call are timed;
    their difference is the cost of `blocks` continued blocks, append-encodes
    included, with the prompt encode cancelled out."""
    w = I.LONG_CTX
    P = w.prompt_len
    n_long = 1 + blocks
    model = dg.Model(w, max_canvases=1, max_prompt=P + 256 * (n_long - 1))
    stream = torch.cuda.current_stream()
    kv = model.new_kv(1, P + 256 * (n_long - 1))
    prompt = torch.from_numpy(I.prompt_ids(w.sample_seed, 1, P, w.vocab)).cuda()
    z = lambda *shape: torch.zeros(shape, dtype=torch.int32, device="cuda")
    toks, steps, ncom = z(1, n_long, 256), z(1, n_long), z(1, n_long)

    def timed(n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        model.generate(prompt, 1, P, n, kv, toks, steps, ncom)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    timed(n_long)                       # warm-up (graph captures, first touches)
    ms_short = timed(1)
    ms_long = timed(n_long)
    model.sync_status()
    n_c = int(ncom[0, 1:].sum().item())
    n_r = int(steps[0, 1:].sum().item())
    model.close()
    ms = max(ms_long - ms_short, 1e-6)
    return {"blocks_continued": blocks, "committed_tokens_per_s": n_c / (ms * 1e-3),
            "committed_per_block": n_c / blocks, "rounds_per_block": n_r / blocks, "ms_per_block": ms / blocks,
            "includes": "append-encode of each finished canvas (256 tokens, causal) and the next block's loop"}


# --- CPU oracle (bounded sample) ---------------------------------------------------------
def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_sample(w, P, budget_s=20.0):
    """Time the oracle on a bounded sample of one round of workload `w` and
    scale to a whole round.  Sample: one transformer layer (256 canvas tokens
    over a random P-token prompt cache, all experts), the LM head and self-
    conditioning on a 1/chunks slice of the vocabulary, and the sampler on
    rows/16 rows; costs are scaled by layers, chunks and 16."""
    import numpy as np
    from block_text_diffusion_b200 import inputs as I
    from oracle import model as om, sampler as sp, _native
    import threading
    bf = w.dtype == 1
    d, V = w.d_model, w.vocab
    s = w.weight_seed
    hq, hkv, hd = w.n_heads * w.head_dim, w.n_kv_heads * w.head_dim, w.head_dim
    E, ff = w.n_experts, w.d_ff
    t = lambda name: om.layer_tensor_id(0, name)
    layer = om.Layer(wq=om.weight_values(s, t("wq"), (hq, d), bf), wk=om.weight_values(s, t("wk"), (hkv, d), bf),
                     wv=om.weight_values(s, t("wv"), (hkv, d), bf), wo=om.weight_values(s, t("wo"), (d, hq), bf),
                     wr=om.weight_values(s, t("wr"), (E, d), bf), wg=om.weight_values(s, t("wg"), (E, ff, d), bf),
                     wu=om.weight_values(s, t("wu"), (E, ff, d), bf), wd=om.weight_values(s, t("wd"), (E, d, ff), bf))
    chunks = max(1, V // 16384)
    vs = V // chunks
    shell = om.Model.__new__(om.Model)
    shell.cfg = w
    shell.embed = om.weight_values(s, om.T_EMBED, (vs, d), bf)   # the first vocabulary slice
    shell.wsc = om.weight_values(s, om.T_WSC, (d, d), bf)
    K, Vv = I.prompt_kv(3, 1, 1, w.n_kv_heads, P, hd, bf16=bf)
    h = shell.embed[np.arange(256) % vs].astype(np.float64)
    t0 = time.perf_counter()
    h2, _, _ = om.block(shell, layer, h, P + np.arange(256), K[0, 0].transpose(1, 0, 2).astype(np.float64),
                        Vv[0, 0].transpose(1, 0, 2).astype(np.float64), causal=False)
    t_layer = time.perf_counter() - t0
    t0 = time.perf_counter()
    x = shell.store(om.rmsnorm(h2, w.rms_eps))
    lg = w.logit_scale * (x @ shell.embed.astype(np.float64).T)
    probs = np.abs(lg[:, :]).astype(np.float32)
    probs /= probs.sum(axis=1, keepdims=True)
    om.self_condition(shell, probs)
    t_head = time.perf_counter() - t0
    rows = 16
    l = I.logits(1, rows, V, "normal", 1.0)
    t0 = time.perf_counter()
    sp.sampler_rows(l, np.float32(1.25), w.sample_seed, 0, 0)
    t_samp = time.perf_counter() - t0
    per_round = w.n_layers * t_layer + chunks * t_head + (256 / rows) * t_samp
    threads = os.cpu_count() or 1
    sample = ("1 of %d layers (256 tokens, %d-token prompt cache, all %d experts), LM head + self-conditioning "
              "on 1/%d of the vocabulary, sampler on %d of 256 rows; scaled to one round"
              % (w.n_layers, P, E, chunks, rows))
    return 1.0 / per_round, threads, sample, t_layer + t_head + t_samp


def run_reference(a):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    from block_text_diffusion_b200 import inputs as I
    w = I.WORKLOADS[a.workload]
    vals = []
    for _ in range(a.warmup):
        oracle_sample(w, w.prompt_len)
    for _ in range(a.steps):
        v, cores, sample, _ = oracle_sample(w, w.prompt_len)
        vals.append(v)
    value = statistics.median(vals)
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "denoise steps/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 / value * w.max_steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (bf16 storage rounding)" if w.dtype == 1 else "f64",
            "data": "synthetic", "config": {"workload": w.name, "canvases_per_gpu": 1, "prompt_len": w.prompt_len},
            "cpu_baseline": {"value": value, "unit": "denoise steps/s", "cores": cores, "kind": "oracle",
                             "sample": sample, "cpu": cpu_model()},
            "e2e": {"value": value, "unit": "denoise steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    a = parse()
    if a.impl == "reference":
        line = run_reference(a)
        if line:
            print(json.dumps(line), flush=True)
        return
    line = run_ours(a)
    if line is None:
        return
    if not a.no_cpu_baseline and line["n_gpus"] == 1:
        from block_text_diffusion_b200 import inputs as I
        w = I.WORKLOADS[a.workload]
        v, cores, sample, secs = oracle_sample(w, w.prompt_len)
        line["cpu_baseline"] = {"value": v, "unit": "denoise steps/s", "cores": cores, "kind": "oracle",
                                "sample": sample, "cpu_seconds": secs, "cpu": cpu_model()}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
