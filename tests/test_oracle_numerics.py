"""Pins of the oracle's numerics against published vectors, float64 libm and
brute force (CPU only)."""
import math
import os

import numpy as np
import pytest
from scipy import stats

from oracle import _native, numerics as nm
from oracle import model as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _kat():
    rows = []
    for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([int(w, 16) for w in line.split()])
    return rows


def test_philox_known_answers():
    for r in _kat():
        out = nm.philox4x32_10(*[np.uint32(v) for v in r[:6]])
        assert [int(o) for o in out] == r[6:]


def test_uniform_open_interval_and_exactness():
    u = nm.uniform_open(np.array([0, 0x1FF, 0x200, 0xFFFFFFFF], dtype=np.uint32))
    assert u[0] == np.float32(2.0 ** -24) and u[1] == u[0]
    assert u[2] == np.float32(3 * 2.0 ** -24)
    assert u[3] == np.float32(1 - 2.0 ** -24) and u[3] < 1
    # exact: the odd numerator times 2^-24 equals the real quotient
    w = np.random.default_rng(0).integers(0, 2 ** 32, size=10000, dtype=np.uint64).astype(np.uint32)
    uu = nm.uniform_open(w).astype(np.float64)
    assert np.array_equal(uu, ((w >> 9).astype(np.float64) * 2 + 1) / 2 ** 24)


def test_token_from_word_range_and_uniformity():
    w = np.arange(0, 2 ** 32, 2 ** 20, dtype=np.uint64).astype(np.uint32)
    t = nm.token_from_word(w, 1000)
    assert t.min() == 0 and t.max() == 999
    assert np.array_equal(t, (w.astype(np.float64) * 1000 // 2 ** 32).astype(np.int32))


def _ulp_err(got, ref):
    got = np.asarray(got, np.float64)
    ulp = np.abs(np.spacing(np.asarray(ref, np.float32))).astype(np.float64)
    return np.abs(got - ref) / ulp


def test_log_f32_exhaustive_on_sampler_domain():
    # every uniform the sampler can draw, and every -ln(u) fed to the outer log
    n = np.arange(0, 2 ** 23, dtype=np.uint32)
    u = (n * 2 + 1).astype(np.float32) * np.float32(2.0 ** -24)
    lu = nm.chunked(nm.log_f32, u)
    assert _ulp_err(lu, np.log(u.astype(np.float64))).max() <= 3.0
    x = -lu
    lx = nm.chunked(nm.log_f32, x)
    assert _ulp_err(lx, np.log(x.astype(np.float64))).max() <= 3.0
    assert nm.log_f32(np.float32(1.0)) == 0.0


def test_log_f32_wide_range():
    g = np.random.default_rng(1)
    bits = g.integers(0x00800000, 0x7F800000, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    err = _ulp_err(nm.chunked(nm.log_f32, x), np.log(x.astype(np.float64)))
    assert err.max() <= 3.0
    # powers of two reduce to e*ln2
    for e in (-100, -1, 1, 10, 18, 100):
        assert abs(float(nm.log_f32(np.float32(2.0 ** e))) - e * math.log(2)) <= 1e-6 * max(1, abs(e))


def test_exp_f32_sweep():
    x = np.linspace(-86, 0, 1 << 22).astype(np.float32)
    e = nm.chunked(nm.exp_f32, x)
    assert _ulp_err(e, np.exp(x.astype(np.float64))).max() <= 2.0
    assert nm.exp_f32(np.float32(0.0)) == 1.0
    assert nm.exp_f32(np.float32(-86.5)) == 0.0 and nm.exp_f32(np.float32(-1e30)) == 0.0


def test_cos2pi_sweep_and_symmetries():
    n = np.arange(0, 2 ** 23, 7, dtype=np.uint32)
    u = (n * 2 + 1).astype(np.float32) * np.float32(2.0 ** -24)
    c = nm.chunked(nm.cos2pi_f32, u)
    assert np.abs(c - np.cos(2 * np.pi * u.astype(np.float64))).max() < 2.5e-7
    assert nm.cos2pi_f32(np.float32(0.5)) == -1.0
    assert abs(float(nm.cos2pi_f32(np.float32(0.25)))) < 1e-7
    assert abs(float(nm.cos2pi_f32(np.float32(1 / 3))) + 0.5) < 2e-7


def _bf16_brute(x):
    """Nearest bfloat16 by comparing the two neighbours (ties to even)."""
    out = []
    for v in np.asarray(x, np.float32):
        b = int(np.array([v]).view(np.uint32)[0])
        lo = b & 0xFFFF0000
        hi = lo + 0x10000
        flo = float(np.array([lo], np.uint32).view(np.float32)[0])
        fhi = float(np.array([hi], np.uint32).view(np.float32)[0])
        dl, dh = abs(float(v) - flo), abs(fhi - float(v))
        if dl < dh or (dl == dh and ((lo >> 16) & 1) == 0):
            out.append(flo)
        else:
            out.append(fhi)
    return np.array(out, np.float32)


def test_round_bf16_against_brute_force():
    g = np.random.default_rng(2)
    x = (g.standard_normal(4000) * 10).astype(np.float32)
    # force exact ties
    xb = x.view(np.uint32)
    xb[:500] = (xb[:500] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    ref = _bf16_brute(x)
    assert np.array_equal(nm.round_bf16_from_f32(x), ref)
    assert np.array_equal(nm.round_bf16(x.astype(np.float64)), ref)


def test_weights_box_muller_statistics():
    w = om.weight_values(11, 5, (1 << 20,), bf16=False)
    n = w.size
    assert abs(w.mean()) < 5 * 0.02 / math.sqrt(n)
    assert abs(w.std() / 0.02 - 1) < 0.01
    assert stats.kstest(w.astype(np.float64) / 0.02, stats.norm.cdf).pvalue > 1e-4
    # different tensors / seeds give different streams
    assert not np.array_equal(w[:64], om.weight_values(11, 6, (64,), bf16=False))
    assert not np.array_equal(w[:64], om.weight_values(12, 5, (64,), bf16=False))


@pytest.mark.skipif(_native.lib() is None, reason="no C compiler")
def test_c_twin_weights_bit_equal():
    for (seed, tid, start, count, bf) in [(0, 0, 0, 5000, True), (2, 471, 3 << 31, 3000, False),
                                          ((7 << 32) + 5, 17, 123456789, 2000, True)]:
        got = _native.weights(seed, tid, start, count, bf)
        ref = om._normal_weights(seed, tid, start, count, bf)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
