"""The split-K GEMM entry point that allocates nothing (B200 only).

Some callers cannot allocate device memory -- serving loops that reserve all
device memory at start-up, or code that must never block other streams
(cudaMalloc/cudaFree can synchronise the device and fail under memory
pressure).  dg_gemm_splitk_noalloc keeps its partial sums in a fixed-size
array inside the library instead.  These tests call it through the C ABI and
check it against the existing GEMM entry point (dg_test_gemm) and against an
fp64 host product on calls in a row -- each later call reuses the array the
earlier, larger one filled -- and that it refuses a problem larger than the
array.  This file is collected last."""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_text_diffusion_b200 as dg  # noqa: E402
from block_text_diffusion_b200 import inputs as I  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dg.lib()


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda().to(torch.bfloat16)


# (M, N, K, k_splits): the larger problem first, so the second call runs on an
# array still holding the first call's bigger slabs; M and K tails (M not a
# multiple of 128, K not a multiple of 64) and a split count above the number
# of 64-wide K blocks (clamped to it).
CASES = ((4096, 200, 2816, 3), (1000, 77, 1000, 64), (1536, 256, 1024, 4))


def test_noalloc_gemm_matches_existing_entry_point_on_two_calls():
    for M, N, K, splits in CASES:
        g = np.random.default_rng(M + N + K)
        A = I._bf16_grid(g.standard_normal((M, K)).astype(np.float32))
        B = I._bf16_grid(g.standard_normal((N, K)).astype(np.float32))
        At, Bt = _bf16(A), _bf16(B)
        used = min(splits, -(-K // 64))
        ref = torch.zeros((used, N, M), dtype=torch.float32, device="cuda")
        dg.test_gemm(At, Bt, ref, alpha=1.0, k_splits=used, bn=256)
        out = torch.full((N, M), float("nan"), dtype=torch.float32, device="cuda")
        dg.gemm_splitk_noalloc(At, Bt, out, k_splits=splits)
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        want = ref.cpu().numpy().astype(np.float64).sum(axis=0)
        exact = B.astype(np.float64) @ A.astype(np.float64).T
        bound = np.abs(B.astype(np.float64)) @ np.abs(A.astype(np.float64)).T
        # against the existing entry point and against the fp64 product, with
        # the bound the GEMM parity tests use
        assert np.all(np.abs(got - want) <= 2e-6 * bound), (M, N, K, np.abs(got - want).max())
        assert np.all(np.abs(got - exact) <= 2e-6 * bound), (M, N, K, np.abs(got - exact).max())


def test_noalloc_gemm_rejects_problems_larger_than_its_array():
    A = torch.zeros((4096, 1024), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((2048, 1024), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((2048, 4096), dtype=torch.float32, device="cuda")
    with pytest.raises(dg.DGError) as e:
        dg.gemm_splitk_noalloc(A, B, out, k_splits=4)      # 4 x 2048 x 4096 > 16 Mi floats
    assert e.value.code == 1
