"""The storage-noise envelope helper (CPU): no noise reproduces the oracle's
rounding; a flip lands on the other bf16 neighbour of the exact value."""
import numpy as np

from block_text_diffusion_b200 import inputs as I
from oracle import model as om, numerics as nm
from storage_noise import NoisyStore, rms_ulps


def _values(n=20000, seed=5):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(n) * np.exp(rng.uniform(-20, 20, n))
    return np.concatenate([x, [0.0, -0.0, 1.0, -1.0]])


def test_zero_rate_is_the_oracle_store():
    w = I.TINY_FP32.replace(dtype=I.DTYPE_BF16, n_layers=1)
    x = _values()
    assert np.array_equal(NoisyStore(w, p=0.0).store(x), om.Model(w, layers=1).store(x))


def test_flip_is_the_other_neighbour():
    w = I.TINY_FP32.replace(dtype=I.DTYPE_BF16, n_layers=1)
    x = _values()
    r = nm.round_bf16(x).astype(np.float64)
    f = NoisyStore(w, p=1.0).store(x)
    moved = f != r
    # every finite nonzero value moved, zeros kept
    assert np.all(moved[r != 0]) and np.all(f[r == 0] == 0)
    # exactly one bf16 step apart, and x lies between the two neighbours
    b_r = (r.astype(np.float32).view(np.uint32) >> 16).astype(np.int64)
    b_f = (f.astype(np.float32).view(np.uint32) >> 16).astype(np.int64)
    assert np.all(np.abs(b_r - b_f)[moved] == 1)
    inexact = moved & (x != r)
    assert np.all((np.minimum(r, f) <= x)[inexact] & (x <= np.maximum(r, f))[inexact])


def test_flip_rate_and_rms_ulps():
    w = I.TINY_FP32.replace(dtype=I.DTYPE_BF16, n_layers=1)
    x = np.random.default_rng(2).standard_normal(200000)
    r = nm.round_bf16(x).astype(np.float64)
    f = NoisyStore(w, p=1 / 64, seed=3).store(x)
    rate = (f != r).mean()
    assert abs(rate - 1 / 64) < 5 * np.sqrt(1 / 64 / 200000)
    # a flip of a value below 2 in magnitude is at most one step of 2^-7
    m = (f != r) & (np.abs(r) < 2.0)
    d = rms_ulps(f, r)[m]
    assert np.all(d <= 1.0) and np.all(d > 0)
