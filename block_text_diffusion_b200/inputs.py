"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds workload descriptions and random inputs only.  It contains
none of the method's arithmetic: no normalisation, attention, routing,
sampling, entropy or rounding rule of the model lives here.  Every generator
is a pure function of its seed (numpy PCG64), so the CUDA path and the oracle
can be fed bit-identical inputs.

The five workloads mirror the shapes the DiffusionGemma pages describe: a
256-token canvas refined against a causally cached prompt, a 128-expert top-8
MoE with ~262 k vocabulary for the 26B-A4B-shaped model, multi-canvas batching
and a long-context case.  Weights themselves are not generated here: both
sides derive them from the counter-based generator each implements
independently (Philox4x32-10 + Box-Muller, keyed by the weight seed).
"""
from __future__ import annotations

import dataclasses
import numpy as np

CANVAS = 256

DTYPE_FP32 = 0
DTYPE_BF16 = 1

COMMIT_THRESH = 0   # commit where entropy < commit_bound (nats)
COMMIT_EB = 1       # entropy-bounded: cumulative sorted entropy <= commit_bound
STOP_MEAN = 0       # stop when all committed or mean entropy < stop_bound
STOP_EB = 1         # stop when mean entropy < stop_bound and argmax unchanged


@dataclasses.dataclass(frozen=True)
class Workload:
    """Architecture + sampler parameters of one synthetic workload."""
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    n_experts: int
    top_k: int
    d_ff: int
    vocab: int
    dtype: int
    logit_scale: float = 1.0
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    zipf_s: float = 0.0          # 0 = no router bias
    sample_topk: int = 0         # 0 = exact sampling; K = draw among the K largest logits
    expert_fp8: bool = False     # expert weights as E4M3 codes with power-of-two block scales
    temp_start: float = 0.8
    temp_end: float = 0.4
    max_steps: int = 48
    commit_mode: int = COMMIT_THRESH
    commit_bound: float = 0.5
    stop_mode: int = STOP_MEAN
    stop_bound: float = 0.1
    weight_seed: int = 0
    sample_seed: int = 0
    batch: int = 1
    prompt_len: int = 64

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def canvas_len(self) -> int:
        return CANVAS


# Tiny fp32 decoder (2 layers, d 256, 8 experts top-2, vocab 1024, 8 steps).
TINY_FP32 = Workload("tiny-fp32-L2-d256-E8k2-V1k", n_layers=2, d_model=256, n_heads=4,
                     n_kv_heads=4, head_dim=64, n_experts=8, top_k=2, d_ff=512,
                     vocab=1024, dtype=DTYPE_FP32, max_steps=8, weight_seed=0,
                     sample_seed=0, batch=1, prompt_len=64)
# Mid MoE decoder, bf16 (8 layers, d 1024, 32 experts top-4, vocab 32768).
MID_BF16 = Workload("mid-bf16-L8-d1024-E32k4-V32k", n_layers=8, d_model=1024, n_heads=8,
                    n_kv_heads=2, head_dim=128, n_experts=32, top_k=4, d_ff=1024,
                    vocab=32768, dtype=DTYPE_BF16, logit_scale=4.0, weight_seed=1,
                    sample_seed=1, batch=1, prompt_len=1024)
# 26B-A4B-shaped stand-in (30 layers, d 2816, 128 experts top-8, vocab 262144).
MOE26B_BF16 = Workload("moe26b-bf16-L30-d2816-E128k8-V262k", n_layers=30, d_model=2816,
                       n_heads=16, n_kv_heads=8, head_dim=128, n_experts=128, top_k=8,
                       d_ff=704, vocab=262144, dtype=DTYPE_BF16, weight_seed=2,
                       sample_seed=2, batch=1, prompt_len=2048)
# Multi-canvas batching on the mid architecture with a Zipf(1.1) router bias.
BATCH_ZIPF = MID_BF16.replace(name="mid-bf16-zipf-P2048", zipf_s=1.1,
                              weight_seed=3, sample_seed=3, batch=1, prompt_len=2048)
# Long-context, fast-converging canvas on the mid architecture.
LONG_CTX = MID_BF16.replace(name="mid-bf16-P32768-scale16", logit_scale=16.0,
                            weight_seed=4, sample_seed=4, batch=1, prompt_len=32768)

WORKLOADS = {
    "tiny": TINY_FP32,
    "mid": MID_BF16,
    "moe26b": MOE26B_BF16,
    "batch": BATCH_ZIPF,
    "long": LONG_CTX,
}
BATCH_SIZES = (1, 4, 8, 32)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed) & 0xFFFFFFFF, int(stream)]))


def prompt_ids(seed: int, batch: int, prompt_len: int, vocab: int) -> np.ndarray:
    """Uniform-random prompt token ids, int32 [batch, prompt_len]."""
    return _rng(seed, 101).integers(0, vocab, size=(batch, prompt_len), dtype=np.int32)


def canvas_ids(seed: int, batch: int, vocab: int) -> np.ndarray:
    """Uniform-random canvas token ids, int32 [batch, 256]."""
    return _rng(seed, 102).integers(0, vocab, size=(batch, CANVAS), dtype=np.int32)


def _bf16_grid(x: np.ndarray) -> np.ndarray:
    """Clear the low 16 bits so a float32 value is exactly representable in
    bfloat16 (a truncation used only to make random inputs representable)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def normal(seed: int, stream: int, shape, std: float = 1.0, bf16: bool = False) -> np.ndarray:
    x = (_rng(seed, stream).standard_normal(size=shape) * std).astype(np.float32)
    return _bf16_grid(x) if bf16 else x


def logits(seed: int, rows: int, vocab: int, kind: str = "normal", scale: float = 1.0) -> np.ndarray:
    """Synthetic fp32 logit rows [rows, vocab] with the structures the sampler
    meets: near-uniform (random-init model), peaked (converging canvas),
    ties, and exactly flat rows."""
    g = _rng(seed, 103)
    if kind == "normal":
        x = g.standard_normal(size=(rows, vocab)) * scale
    elif kind == "peaked":
        x = g.standard_normal(size=(rows, vocab)) * scale
        hot = g.integers(0, vocab, size=rows)
        gap = g.uniform(2.0, 40.0, size=rows)
        x[np.arange(rows), hot] += gap
    elif kind == "ties":
        x = g.integers(-3, 4, size=(rows, vocab)).astype(np.float64) * scale
    elif kind == "flat":
        x = np.full((rows, vocab), 0.25 * scale)
    elif kind == "mixed":
        x = g.standard_normal(size=(rows, vocab)) * scale
        n = rows // 4
        x[:n] *= 16.0
        hot = g.integers(0, vocab, size=n)
        x[np.arange(n), hot] += 60.0
        x[n:2 * n] = np.round(x[n:2 * n])
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(x, dtype=np.float32)


def entropies(seed: int, batch: int, low_frac: float = 0.5, ties: bool = False) -> np.ndarray:
    """Synthetic per-position entropies [batch, 256] in nats, a mix of values
    below and above the usual bounds (optionally with many exact ties)."""
    g = _rng(seed, 104)
    lo = g.uniform(0.0, 0.02, size=(batch, CANVAS))
    hi = g.uniform(0.0, 12.0, size=(batch, CANVAS))
    pick = g.random(size=(batch, CANVAS)) < low_frac
    h = np.where(pick, lo, hi).astype(np.float32)
    if ties:
        h = (np.round(h * 64.0) / 64.0).astype(np.float32)
    return h


def token_ids(seed: int, shape, vocab: int, stream: int = 105) -> np.ndarray:
    return _rng(seed, stream).integers(0, vocab, size=shape, dtype=np.int32)


def activations(seed: int, rows: int, cols: int, bf16: bool = True, std: float = 1.0) -> np.ndarray:
    return normal(seed, 106, (rows, cols), std=std, bf16=bf16)


def expert_choice(seed: int, tokens: int, n_experts: int, top_k: int, zipf_s: float = 0.0) -> np.ndarray:
    """Distinct expert ids per token [tokens, top_k], optionally Zipf-skewed."""
    g = _rng(seed, 107)
    w = 1.0 / np.power(np.arange(1, n_experts + 1, dtype=np.float64), zipf_s) if zipf_s else np.ones(n_experts)
    w = w / w.sum()
    out = np.empty((tokens, top_k), dtype=np.int32)
    for t in range(tokens):
        out[t] = g.choice(n_experts, size=top_k, replace=False, p=w)
    return out


def prompt_kv(seed: int, n_layers: int, batch: int, n_kv_heads: int, prompt_len: int,
              head_dim: int, bf16: bool) -> tuple[np.ndarray, np.ndarray]:
    """Synthetic prompt keys and values [L, B, Hkv, P, hd] (stand-in for an
    encoded prompt when the oracle cannot afford the causal encode)."""
    shape = (n_layers, batch, n_kv_heads, prompt_len, head_dim)
    k = normal(seed, 108, shape, std=1.0, bf16=bf16)
    v = normal(seed, 109, shape, std=1.0, bf16=bf16)
    return k, v


def routing_bias(seed: int, n_layers: int, tokens: int, n_experts: int, top_k: int, pool: int,
                 beta: float = 8.0) -> np.ndarray:
    """Structured per-token router bias [n_layers, tokens, n_experts] float32
    standing in for the expert locality of a trained router (the pages report
    about 84 of 128 experts touched per round).  In each layer a random pool
    of `pool` experts serves the canvas tokens and each token prefers top_k
    distinct experts of that pool: +beta on those, 0 elsewhere.  With beta
    well above the spread of the router logits every token picks its preferred
    experts, so a layer touches about `pool` distinct experts."""
    if not top_k <= pool <= n_experts:
        raise ValueError("pool must lie in [top_k, n_experts]")
    g = _rng(seed, 110)
    out = np.zeros((n_layers, tokens, n_experts), dtype=np.float32)
    for l in range(n_layers):
        members = g.permutation(n_experts)[:pool]
        for t in range(tokens):
            out[l, t, members[g.choice(pool, size=top_k, replace=False)]] = beta
    return out
