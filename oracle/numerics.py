"""Oracle numerics: counter-based random numbers and fixed fp32 op sequences.

TEST INFRASTRUCTURE ONLY.  Part of the CPU oracle; only the test-suite, the
smoke check and the bench's CPU-baseline leg may import it.  It shares no code
with the CUDA path.

Every function here is written from a published definition so that its
result is fixed bit-for-bit by the definition itself:

* Philox4x32-10 -- Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
  Easy as 1, 2, 3", SC'11, section 3.2 (the Philox S-box and key schedule).
* the fp32 natural log -- range reduction of the exponent, then
  ln m = 2 atanh(s), s = (m-1)/(m+1), by its odd Taylor series, with ln 2
  split in two parts (Cody & Waite, "Software Manual for the Elementary
  Functions", 1980).
* the fp32 exponential -- Cody-Waite reduction x = k ln2 + r, |r| <= ln2/2,
  then the Taylor series of e^r to degree 7.
* cos(2 pi u) -- octant reduction by the symmetries of cosine, then the
  Taylor series of cos / sin on [0, pi/4].

Each operation is one IEEE-754 binary32 operation with round-to-nearest-even
(numpy float32 arithmetic, no fused multiply-add), so any other faithful
implementation of the same operation sequence returns identical bits.  The
pages never fix these details: they only name Philox-counter sampling, and
this is how it is read -- the sampler's decisions (tokens, commit masks) must
come out the same on two implementations, so every draw is a Philox4x32-10
word turned into an exact binary32 uniform and passed through this fixed
operation sequence, never through a library log or exp.
"""
from __future__ import annotations

import math
import numpy as np

F32 = np.float32
U32 = np.uint32
U64 = np.uint64

# --- Philox4x32-10 (SC'11, section 3.2) ------------------------------------
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9   # golden ratio
PHILOX_W1 = 0xBB67AE85   # sqrt(3) - 1

MASK32 = U64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Ten Philox rounds over a 4x32-bit counter under a 2x32-bit key.

    Each round multiplies counter words 0 and 2 by the two round constants,
    keeps the high and low halves, and mixes the high halves with words 1 and
    3 and the key; the key is bumped by the Weyl constants between rounds.
    Arguments are broadcastable uint32 arrays; returns four uint32 arrays.
    """
    c0, c1, c2, c3 = (np.asarray(c, dtype=U32) for c in (c0, c1, c2, c3))
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    k0 = np.asarray(k0, dtype=U32)
    k1 = np.asarray(k1, dtype=U32)
    for rnd in range(10):
        if rnd:
            k0 = ((k0.astype(U64) + U64(PHILOX_W0)) & MASK32).astype(U32)
            k1 = ((k1.astype(U64) + U64(PHILOX_W1)) & MASK32).astype(U32)
        p0 = c0.astype(U64) * U64(PHILOX_M0)
        p1 = c2.astype(U64) * U64(PHILOX_M1)
        hi0 = (p0 >> U64(32)).astype(U32)
        lo0 = (p0 & MASK32).astype(U32)
        hi1 = (p1 >> U64(32)).astype(U32)
        lo1 = (p1 & MASK32).astype(U32)
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def seed_key(seed: int, canvas_id: int = 0):
    """Philox key of a seed and a canvas id: (seed_lo, seed_hi xor canvas)."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return U32(seed & 0xFFFFFFFF), U32(((seed >> 32) ^ int(canvas_id)) & 0xFFFFFFFF)


# Philox counter word 3 names the stream a random number belongs to.
STREAM_GUMBEL = 0
STREAM_RENOISE = 1
STREAM_INIT_CANVAS = 2
STREAM_WEIGHTS = 3


def uniform_open(x):
    """uint32 -> float32 in (0,1): ((x >> 9)*2 + 1) * 2^-24.

    The odd numerator has at most 24 bits, so the value is exact in binary32
    and lies in [2^-24, 1 - 2^-24]; 0 and 1 never occur.
    """
    n = ((np.asarray(x, dtype=U32) >> U32(9)) * U32(2) + U32(1)).astype(F32)
    return n * F32(2.0 ** -24)


def token_from_word(x, vocab: int):
    """Uniform token id in [0, vocab): floor(x * vocab / 2^32) in 64-bit integers."""
    return ((np.asarray(x, dtype=U32).astype(U64) * U64(vocab)) >> U64(32)).astype(np.int32)


# --- fp32 natural logarithm ---------------------------------------------------
_LN2 = math.log(2.0)
# ln 2 rounded to binary32, then cut to 16 significant bits so that k * LN2_HI
# is exact for every |k| < 2^8 (Cody-Waite split).
LN2_HI = (np.array([_LN2], dtype=F32).view(U32) & U32(0xFFFFFF00)).view(F32)[0]
LN2_LO = F32(_LN2 - float(LN2_HI))
INV_LN2 = F32(1.0 / _LN2)
# 2 atanh(s) = 2 s (1 + s^2/3 + s^4/5 + ... + s^10/11)
_ATANH_C = [F32(1.0 / n) for n in (11, 9, 7, 5, 3)]
_SQRT2_BITS = 0x3FB504F3      # largest binary32 below sqrt(2)


def log_f32(x):
    """Natural log of positive normal binary32 values (fixed op sequence).

    x = 2^e * m with m in [sqrt(1/2), sqrt(2)]; ln m = 2 s P(s^2) with
    s = (m-1)/(m+1) and P the atanh series through s^10/11 (|s| < 0.1716, so
    the first dropped term is below 2^-25 relative); ln x = e ln2 + ln m.
    """
    x = np.asarray(x, dtype=F32)
    b = x.view(U32)
    e = (b >> U32(23)).astype(np.int32) - 127
    mb = (b & U32(0x007FFFFF)) | U32(0x3F800000)
    big = mb > U32(_SQRT2_BITS)
    mb = np.where(big, mb - U32(0x00800000), mb).astype(U32)
    e = np.where(big, e + 1, e)
    m = mb.view(F32)
    s = (m - F32(1.0)) / (m + F32(1.0))
    z = s * s
    p = np.full_like(z, _ATANH_C[0])
    for c in _ATANH_C[1:]:
        p = p * z + c
    p = p * z + F32(1.0)
    lnm = (s + s) * p
    ef = e.astype(F32)
    return ef * LN2_HI + (ef * LN2_LO + lnm)


# --- fp32 exponential for x <= 0 ------------------------------------------------
_EXP_C = [F32(1.0 / math.factorial(n)) for n in (7, 6, 5, 4, 3, 2)]
EXP_FLUSH = F32(-86.0)   # below this, e^x < 2^-124 and is returned as 0


def exp_f32(x):
    """e^x for binary32 x <= 0 (fixed op sequence); 0 for x < -86.

    k = rint(x / ln2), r = (x - k LN2_HI) - k LN2_LO, e^r by its Taylor
    series through r^7/7! (|r| <= 0.347, first dropped term < 2^-27), then
    scaled by 2^k through the exponent field (k >= -124, result normal).
    """
    x = np.asarray(x, dtype=F32)
    xc = np.clip(x, F32(-87.0), F32(0.0)).astype(F32)
    t = xc * INV_LN2
    k = np.rint(t).astype(F32)
    r = (xc - k * LN2_HI) - k * LN2_LO
    p = np.full_like(r, _EXP_C[0])
    for c in _EXP_C[1:]:
        p = p * r + c
    p = p * r + F32(1.0)
    p = p * r + F32(1.0)
    ki = np.maximum(k.astype(np.int32), -126)
    scale = ((ki + 127).astype(U32) << U32(23)).view(F32)
    y = p * scale
    return np.where(x < EXP_FLUSH, F32(0.0), y).astype(F32)


# --- fp32 cos(2 pi u) for u in (0, 1) -------------------------------------------
TWO_PI = F32(2.0 * math.pi)
_COS_C = [F32(v) for v in (-1.0 / math.factorial(10), 1.0 / math.factorial(8), -1.0 / math.factorial(6),
                           1.0 / math.factorial(4), -0.5)]
_SIN_C = [F32(v) for v in (-1.0 / math.factorial(11), 1.0 / math.factorial(9), -1.0 / math.factorial(7),
                           1.0 / math.factorial(5), -1.0 / 6.0)]


def cos2pi_f32(u):
    """cos(2 pi u) for binary32 u in (0,1) (fixed op sequence).

    By symmetry the argument is folded to b in [0, 1/8]; the result is
    +-cos(2 pi b) or +-sin(2 pi b), each from its Taylor series on [0, pi/4]
    (cos through x^10, sin through x^11; dropped terms < 2^-32).
    """
    u = np.asarray(u, dtype=F32)
    a = np.where(u > F32(0.5), F32(1.0) - u, u).astype(F32)
    neg = a > F32(0.25)
    a = np.where(neg, F32(0.5) - a, a).astype(F32)
    use_sin = a > F32(0.125)
    b = np.where(use_sin, F32(0.25) - a, a).astype(F32)
    x = b * TWO_PI
    z = x * x
    pc = np.full_like(z, _COS_C[0])
    for c in _COS_C[1:]:
        pc = pc * z + c
    pc = pc * z + F32(1.0)
    ps = np.full_like(z, _SIN_C[0])
    for c in _SIN_C[1:]:
        ps = ps * z + c
    ps = ps * z + F32(1.0)
    ps = x * ps
    r = np.where(use_sin, ps, pc).astype(F32)
    return np.where(neg, -r, r).astype(F32)


# --- rounding to storage precision ---------------------------------------------
def round_bf16(x):
    """Round to the nearest bfloat16 (ties to even) directly from float64,
    returned as float32 holding the bf16 value."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                        # x = m 2^e, |m| in [0.5, 1)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # 8 significant bits, RNE
    return r.astype(np.float32)


def chunked(fn, *arrays, chunk: int = 1 << 15):
    """Apply an elementwise function over flattened arrays in small blocks.

    Pure evaluation-order bookkeeping: the result equals fn(*arrays); small
    blocks only keep numpy's temporaries in cache.
    """
    arrays = [np.ascontiguousarray(a) for a in np.broadcast_arrays(*arrays)]
    shape = arrays[0].shape
    flat = [a.reshape(-1) for a in arrays]
    n = flat[0].size
    first = fn(*[a[:min(chunk, n)] for a in flat])
    out = np.empty(n, dtype=first.dtype)
    out[:first.size] = first
    for i in range(chunk, n, chunk):
        out[i:i + chunk] = fn(*[a[i:i + chunk] for a in flat])
    return out.reshape(shape)


def round_bf16_from_f32(x):
    """Round binary32 values to bfloat16 (ties to even), as float32."""
    x = np.ascontiguousarray(x, dtype=F32)
    b = x.view(U32).astype(U64)
    lsb = (b >> U64(16)) & U64(1)
    b = (b + U64(0x7FFF) + lsb) & U64(0xFFFF0000)
    return b.astype(U32).view(F32)
