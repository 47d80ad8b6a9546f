"""Pins of the FP8 expert-weight oracle (E4M3 codes, power-of-two block scales)."""
import numpy as np
import pytest

from block_text_diffusion_b200 import inputs as I
from oracle import fp8, model as om, numerics as nm

torch = pytest.importorskip("torch")
F32 = np.float32


def test_e4m3_code_table_closed_forms():
    vals = np.array([fp8.e4m3_value(c) for c in range(256)])
    assert np.isnan(vals).sum() == 2 and np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])
    fin = vals[~np.isnan(vals)]
    assert fin.max() == 448.0 and fin.min() == -448.0
    pos = np.unique(fin[fin > 0])
    assert pos[0] == 2.0 ** -9 and len(pos) == 126           # 7 subnormals + 15 binades x 8 - 1 (NaN)
    assert fp8.e4m3_value(0x08) == 2.0 ** -6                 # smallest normal
    assert fp8.e4m3_value(0x80) == 0.0 and np.signbit(fp8.e4m3_value(0x80))


def test_round_e4m3_matches_the_library_conversion():
    # torch's float8_e4m3fn conversion (round to nearest even) on binary32
    # inputs: the full range, ties, subnormals, signed zeros
    g = np.random.default_rng(0)
    mids = (fp8._VALS[:-1] + fp8._VALS[1:]) / 2              # exact ties
    x = np.concatenate([np.linspace(-448, 448, 100001), g.standard_normal(100000) * 3,
                        g.standard_normal(100000) * 1e-3, mids, -mids, mids * (1 + 2.0 ** -20),
                        [0.0, -0.0, 2.0 ** -10, -(2.0 ** -10), 3 * 2.0 ** -11]]).astype(F32)
    codes, vals = fp8.round_e4m3(x)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn)
    assert np.array_equal(t.view(torch.uint8).numpy(), codes)
    assert np.array_equal(t.to(torch.float64).numpy(), vals)


def test_block_scales_are_the_tight_power_of_two():
    g = np.random.default_rng(1)
    w = g.standard_normal((7, 300)) * np.exp(g.uniform(-20, 10, size=(7, 1)))
    w[3, 128:256] = 0.0
    s = fp8.block_scales(w)
    assert s.shape == (7, 3)
    assert np.all(np.log2(s) == np.round(np.log2(s)))
    amax = np.stack([np.abs(w[:, i * 128:(i + 1) * 128]).max(axis=1) for i in range(3)], axis=1)
    nz = amax > 0
    assert np.all(amax[nz] / s[nz] <= 448.0) and np.all(amax[nz] / s[nz] > 224.0)
    assert s[3, 1] == 1.0


def test_dequantised_expert_weights_are_bf16_values_close_to_the_originals():
    w = om.weight_values(3, om.layer_tensor_id(0, "wg"), (2, 704, 2816), True)
    codes, s, deq = fp8.quantize(w)
    assert codes.dtype == np.uint8 and s.shape == (2, 704, 22)
    assert np.array_equal(nm.round_bf16(deq.astype(np.float64)), deq.astype(np.float64))
    sf = np.repeat(s, 128, axis=-1)
    normal = np.abs(w) >= sf * 2.0 ** -6
    rel = np.abs(deq - w)[normal] / np.abs(w)[normal]
    assert rel.max() <= 2.0 ** -4
    assert np.all(np.abs(deq - w)[~normal] <= sf[~normal] * 2.0 ** -10)
    assert np.all(np.sign(deq)[deq != 0] == np.sign(w)[deq != 0])


def test_fp8_model_is_the_bf16_model_on_quantised_expert_weights():
    w = I.TINY_FP32.replace(n_layers=1, dtype=I.DTYPE_BF16)
    a, b = om.Model(w), om.Model(w.replace(expert_fp8=True))
    for name in ("wq", "wk", "wv", "wo", "wr"):
        assert np.array_equal(getattr(a.layers[0], name), getattr(b.layers[0], name))
    for name in ("wg", "wu", "wd"):
        assert np.array_equal(getattr(b.layers[0], name), fp8.quantize(getattr(a.layers[0], name))[2])
        assert not np.array_equal(getattr(b.layers[0], name), getattr(a.layers[0], name))
