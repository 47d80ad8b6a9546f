"""The split-K GEMM entry point that allocates nothing (B200 only).

Some callers cannot allocate device memory -- serving loops that reserve all
device memory at start-up, or code that must never block other streams
(cudaMalloc/cudaFree can synchronise the device and fail under memory
pressure).  dg_gemm_splitk_noalloc keeps its partial sums in a fixed-size
array inside the library instead.  These tests call it through the C ABI and
check it against the existing GEMM entry point (dg_test_gemm) on two calls in
a row -- the second call reuses the array the first one filled -- and that
it refuses a problem larger than the array.  This file is collected last."""
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


def test_noalloc_gemm_matches_existing_entry_point_on_two_calls():
    for M, N, K, splits in ((1536, 256, 1024, 4), (4096, 200, 2816, 3)):
        g = np.random.default_rng(M + N + K)
        A = I._bf16_grid(g.standard_normal((M, K)).astype(np.float32))
        B = I._bf16_grid(g.standard_normal((N, K)).astype(np.float32))
        At, Bt = _bf16(A), _bf16(B)
        ref = torch.zeros((splits, N, M), dtype=torch.float32, device="cuda")
        dg.test_gemm(At, Bt, ref, alpha=1.0, k_splits=splits, bn=256)
        out = torch.full((N, M), float("nan"), dtype=torch.float32, device="cuda")
        dg.gemm_splitk_noalloc(At, Bt, out, k_splits=splits)
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        want = ref.cpu().numpy().astype(np.float64).sum(axis=0)
        bound = np.abs(B.astype(np.float64)) @ np.abs(A.astype(np.float64)).T
        assert np.all(np.abs(got - want) <= 2e-6 * bound), np.abs(got - want).max()


def test_noalloc_gemm_rejects_problems_larger_than_its_array():
    A = torch.zeros((4096, 1024), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((2048, 1024), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((2048, 4096), dtype=torch.float32, device="cuda")
    with pytest.raises(dg.DGError) as e:
        dg.gemm_splitk_noalloc(A, B, out, k_splits=4)      # 4 x 2048 x 4096 > 16 Mi floats
    assert e.value.code == 1
