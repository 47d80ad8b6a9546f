"""FP8 expert-weight kernels against the oracle and the bf16 GEMM (B200 only)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_text_diffusion_b200 as dg  # noqa: E402
from block_text_diffusion_b200 import inputs as I  # noqa: E402
from oracle import fp8, model as om  # noqa: E402

F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dg.lib()


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


@pytest.mark.parametrize("rows,K,tid", [(256, 2816, om.layer_tensor_id(0, "wg")), (300, 704, om.layer_tensor_id(1, "wd")),
                                        (64, 320, 7)])
def test_quant_fp8_bit_exact(rows, K, tid):
    w = om.weight_values(3, tid, (rows, K), True)
    w[5, :128] = 0.0                                   # an all-zero block: scale 1
    w[7, 3] = -1e-30 if K > 3 else w[7, 3]             # rounds to -0
    codes = torch.empty((rows, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, -(-K // 128)), dtype=torch.float32, device="cuda")
    dg.test_quant_fp8(cu(w).to(torch.bfloat16), codes, scales)
    c_ref, s_ref, _ = fp8.quantize(nm_bf16(w))
    assert np.array_equal(host(scales), s_ref.astype(F32))
    assert np.array_equal(host(codes), c_ref)


def nm_bf16(w):
    from oracle import numerics as nm
    return nm.round_bf16_from_f32(w)


@pytest.mark.parametrize("groups,M,K,bn,splits,counts_seed", [
    (4, 256, 1024, 64, 1, 1), (8, 1408, 2816, 256, 1, 2), (5, 2816, 704, 128, 1, 3),
    (3, 384, 2816, 32, 4, 4), (6, 200, 512, 256, 2, 5)])
def test_grouped_gemm_fp8_equals_bf16_gemm_on_dequantised_weights(groups, M, K, bn, splits, counts_seed):
    g = np.random.default_rng(counts_seed)
    counts = g.integers(0, 300, size=groups)
    counts[0] = max(counts[0], 1)
    rows = int(counts.sum())
    W = nm_bf16((0.02 * g.standard_normal((groups * M, K))).astype(F32))
    X = nm_bf16(g.standard_normal((rows, K)).astype(F32))
    codes, scales, deq = fp8.quantize(W)
    out8 = torch.zeros((splits, rows, M), dtype=torch.float32, device="cuda")
    dg.test_grouped_gemm_fp8(cu(codes), cu(scales.astype(F32)), cu(X).to(torch.bfloat16), counts, groups, M, out8,
                             bn=bn, k_splits=splits)
    got = host(out8).sum(axis=0, dtype=np.float64) if splits > 1 else host(out8)[0]
    # independent fp64 reference on the dequantised weights
    ref = np.empty((rows, M))
    r0 = 0
    for gi, c in enumerate(counts):
        ref[r0:r0 + c] = X[r0:r0 + c].astype(np.float64) @ deq[gi * M:(gi + 1) * M].astype(np.float64).T
        r0 += c
    bound = 4e-6 * (np.abs(X).astype(np.float64) @ np.abs(deq).astype(np.float64)[:M].T).max() + 1e-6
    assert np.abs(got - ref).max() <= max(bound, 1e-3 * np.abs(ref).max())
    if splits == 1:
        # bit-identical to the bf16 persistent GEMM on the same (dequantised) weights
        out16 = torch.zeros((rows, M), dtype=torch.float32, device="cuda")
        dg.test_grouped_gemm(cu(deq).to(torch.bfloat16), cu(X).to(torch.bfloat16), counts, groups, M, out16,
                             bn=bn, persistent=True)
        assert np.array_equal(host(out16).view(np.uint32), host(out8)[0].view(np.uint32))


def test_mid_fp8_expert_weights_read_back_equal_oracle():
    # the engine quantises the generated expert tensors at init: the
    # dequantised values it holds equal the oracle's FP8 model exactly
    w = I.MID_BF16.replace(n_layers=2, expert_fp8=True)
    gm = dg.Model(w)
    try:
        for l in range(w.n_layers):
            ref = om.layer_weights(w, l)
            for name in ("wg", "wu", "wd"):
                r = getattr(ref, name)
                out = torch.empty(r.shape, dtype=torch.bfloat16, device="cuda")
                gm.read_weight(om.layer_tensor_id(l, name), out)
                assert np.array_equal(host(out.float()).view(np.uint32), r.view(np.uint32)), (l, name)
    finally:
        gm.close()


@pytest.mark.slow
def test_mid_fp8_every_layer_matches_oracle():
    # every layer of the mid workload with E4M3 expert weights, from seeded
    # inputs, against the oracle's FP8 model under the per-layer bound
    import test_gpu_layers as tl
    w = I.MID_BF16.replace(expert_fp8=True, name="mid-bf16-fp8")
    tl.layer_sweep(w, w.prompt_len, 64, range(w.n_layers))
