"""Oracle of FP8 expert weights: OCP E4M3 codes with power-of-two block scales.

TEST INFRASTRUCTURE ONLY: imported by the tests; shares no code with the CUDA
path.

What the pages fix: DiffusionGemma is deployed quantised to FP8 (release news
"速度数据": vLLM serves it with FP8 quantisation on H100/H200; "谷歌都下场了：
扩散语言模型的四倍速与六倍错" section 一: 1000+ tokens/s on an H100 in FP8).
They give no format detail.  Reading (the plainest one that keeps the
expert GEMM's arithmetic): the expert weights -- gate, up and down, the
bytes that dominate a round -- are stored as 8-bit E4M3 values (the OCP FP8
"E4M3FN" encoding: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
infinities, largest finite 448) with one scale per 128 consecutive inputs of
each output row; each scale is a power of two, s = 2^ceil(log2(amax / 448))
with amax the block's largest magnitude (s = 1 for an all-zero block), and
each code is round-to-nearest-even of w / s.  The value a GEMM uses is q s.
Because s is a power of two and q has a 3-bit mantissa, q s is exactly a
bfloat16 value: an FP8-weight model is the bf16 model run on the quantised
expert weights, with every other rule unchanged.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
E4M3_MAX = 448.0
BLOCK = 128


def e4m3_value(code: int) -> float:
    """Value of an E4M3FN byte (NaN for the two NaN codes S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9               # subnormal: m/8 * 2^(1-7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def _positive_table():
    """Non-negative finite E4M3FN values (codes 0x00..0x7E) in increasing order."""
    codes = np.arange(0x7F, dtype=np.uint8)
    return np.array([e4m3_value(int(c)) for c in codes]), codes


_VALS, _CODES = _positive_table()


def round_e4m3(x):
    """Round-to-nearest-even of float64 values onto E4M3FN, saturating at
    +-448 (only reached by the callers' own overflow checks).  The magnitude
    is rounded on the non-negative values ('even' = mantissa bit 0 clear) and
    the sign bit set from x, so negative values that round to zero give -0.
    Returns (codes uint8, values float64)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_VALS, a, side="left"), 0, _VALS.size - 1)
    lo = np.clip(hi - 1, 0, _VALS.size - 1)
    d_lo, d_hi = np.abs(a - _VALS[lo]), np.abs(_VALS[hi] - a)
    even_lo = (_CODES[lo] & 1) == 0
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~even_lo)
    idx = np.where(pick_hi, hi, lo)
    neg = np.signbit(x)
    codes = _CODES[idx] | np.where(neg, np.uint8(0x80), np.uint8(0))
    vals = np.where(neg, -_VALS[idx], _VALS[idx])
    return codes.astype(np.uint8), vals


def block_scales(w, block: int = BLOCK):
    """Power-of-two scale per (row, block of `block` inputs) of w [..., K]:
    2^ceil(log2(amax / 448)), 1 for an all-zero block.  Returns float64
    [..., ceil(K / block)]."""
    w = np.asarray(w, dtype=np.float64)
    K = w.shape[-1]
    nb = -(-K // block)
    pad = nb * block - K
    wp = np.concatenate([w, np.zeros(w.shape[:-1] + (pad,))], axis=-1) if pad else w
    amax = np.abs(wp.reshape(w.shape[:-1] + (nb, block))).max(axis=-1)
    e = np.ceil(np.log2(np.where(amax > 0, amax, 1.0) / E4M3_MAX))
    # log2 of a ratio can land a hair off an integer; settle the exponent exactly
    s = 2.0 ** e
    s = np.where(amax / s > E4M3_MAX, s * 2.0, s)
    s = np.where((amax > 0) & (amax / (s / 2.0) <= E4M3_MAX), s / 2.0, s)
    return np.where(amax > 0, s, 1.0)


def quantize(w, block: int = BLOCK):
    """E4M3 codes [..., K] (uint8), scales [..., K/block] and the dequantised
    values q s (float32, exact) of w [..., K]."""
    w = np.asarray(w, dtype=np.float64)
    s = block_scales(w, block)
    s_full = np.repeat(s, block, axis=-1)[..., :w.shape[-1]]
    codes, q = round_e4m3(w / s_full)
    return codes, s, (q * s_full).astype(F32)
