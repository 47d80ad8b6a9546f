"""Storage-noise envelope for bf16 parity (test helper, CPU only).

A bf16 implementation that accumulates in fp32 rounds some stored values to
the other bf16 neighbour of the exact result: whenever the exact value lies
within its fp32 error of a rounding midpoint.  Each such flip moves the value
by one bf16 step, the model propagates it, and RMSNorm's row-wide scale
spreads it over the whole row.  How far two correct implementations can end
up apart is therefore a property of the model, not of either implementation.

`NoisyStore` measures that property with the oracle itself: an oracle model
whose every storage rounding picks the other bf16 neighbour with probability
p (independent draws from a fixed seed).  The parity tests compare the CUDA
path's deviation from the oracle against the deviation of this perturbed
oracle from the plain one on the same inputs.
"""
import numpy as np

from oracle import model as om, numerics as nm

F32 = np.float32

# One stored value in 64 rounds the other way: the rate at which values
# computed with a relative error of about 3e-5 land on the far side of a bf16
# midpoint (2 * 3e-5 * 2^8 = 1.5%), above what fp32 accumulation over the
# model's reduction lengths (<= 2816 terms) produces for well-conditioned sums.
FLIP_RATE = 1.0 / 64


class NoisyStore(om.Model):
    """Oracle model whose bf16 storage rounds to the other neighbour with
    probability `p` (the weights are the oracle's own)."""

    def __init__(self, cfg, p=FLIP_RATE, seed=1):
        super().__init__(cfg)
        self.p = p
        self.rng = np.random.default_rng(seed)

    def store(self, x):
        x = np.asarray(x, dtype=np.float64)
        r = nm.round_bf16(x).astype(F32)
        if self.p <= 0.0:
            return r.astype(np.float64)
        flip = self.rng.random(r.shape) < self.p
        # direction of the other neighbour: towards x (exact hits go either way)
        toward = np.where(x > r, 1, np.where(x < r, -1, np.where(self.rng.random(r.shape) < 0.5, 1, -1)))
        # on the sign-magnitude bit pattern, +1 grows |r| and -1 shrinks it
        step = np.where(np.signbit(r), -toward, toward)
        bits = (r.view(np.uint32) >> 16).astype(np.int64)
        # never step across zero or into inf/nan: those values keep their rounding
        ok = flip & (bits & 0x7FFF != 0) & ((bits & 0x7F80) != 0x7F80) & \
            ~(((bits & 0x7FFF) == 0x7F7F) & (step > 0))
        bits = bits + np.where(ok, step, 0)
        return (bits.astype(np.uint32) << 16).view(F32).astype(np.float64)


def rms_ulps(a, b):
    """|a - b| in bf16 steps at the scale of a unit-rms row (2^-7)."""
    return np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)) / 2.0 ** -7


def quantiles(v, qs=(0.5, 0.99, 0.999)):
    v = np.asarray(v, dtype=np.float64).ravel()
    return {q: float(np.quantile(v, q)) for q in qs} | {"max": float(v.max()) if v.size else 0.0}
