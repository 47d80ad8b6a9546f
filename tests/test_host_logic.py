"""Host-side logic of the library that runs without a GPU: the attention
split plan, and the validation of configs and arguments that must reject bad
input before any device call."""
import ctypes

import pytest

import block_text_diffusion_b200 as dg
from block_text_diffusion_b200 import inputs as I

SMS = 148
BK = 64                      # keys per attention block


@pytest.fixture(scope="module")
def lib():
    from block_text_diffusion_b200 import build
    build.build()
    return dg.lib()


def plan(lib, n_q, G, Hkv, n_canvas, n_keys, cap=1 << 40):
    out = (ctypes.c_int32 * 5)()
    rows = n_q * G * Hkv * n_canvas
    assert lib.dg_test_attn_plan(n_q, G, Hkv, n_canvas, n_keys, rows, cap, out) == 0
    return list(out), rows


@pytest.mark.parametrize("n_q,G,Hkv,n_canvas,n_keys", [
    (256, 2, 8, 1, 2304),        # 26B shape, 2048-token prompt
    (256, 4, 2, 1, 1280),        # mid shape
    (256, 4, 2, 1, 33024),       # long context
    (256, 4, 2, 32, 2304),       # 32 canvases
    (64, 1, 4, 1, 320),          # tiny
    (256, 2, 8, 1, 1),           # a single key
    (1024, 4, 2, 1, 1024),       # causal encode chunk
])
def test_attention_plan_covers_every_key_block_once(lib, n_q, G, Hkv, n_canvas, n_keys):
    (q_tiles, n_splits, bps, ctas, cluster), rows = plan(lib, n_q, G, Hkv, n_canvas, n_keys)
    nblocks = -(-n_keys // BK)
    assert q_tiles * 128 >= n_q * G and (q_tiles - 1) * 128 < n_q * G
    assert 1 <= n_splits <= nblocks
    assert n_splits * bps >= nblocks and (n_splits - 1) * bps < nblocks      # no empty split
    base = -(-q_tiles // 2) * Hkv * n_canvas
    assert ctas == base * n_splits
    if base <= SMS:
        assert ctas <= SMS or n_splits == 1                                  # the grid fills the SMs once
    if cluster:
        assert n_splits <= 8                                                 # a portable cluster merges the splits


def test_attention_plan_respects_the_partial_buffer(lib):
    (_, n_splits, _, _, cluster), rows = plan(lib, 256, 4, 2, 1, 33024, cap=3 * 256 * 4 * 2)
    assert cluster or n_splits * rows <= 3 * 256 * 4 * 2
    (_, n_splits, _, _, cluster), _ = plan(lib, 256, 4, 2, 1, 33024, cap=1)
    assert cluster or n_splits == 1


def test_attention_plan_merges_short_key_ranges_in_the_kernel(lib):
    # the 26B-A4B canvas pass (2304 keys, 16 pairs x heads) and the mid one
    # merge their splits inside a cluster; the 33k-key long context splits
    # wider through the partial buffer
    assert plan(lib, 256, 2, 8, 1, 2304)[0][4] == 1
    assert plan(lib, 256, 4, 2, 1, 1280)[0][4] == 1
    assert plan(lib, 256, 4, 2, 1, 33024)[0][4] == 0


def _init_status(lib, w, **over):
    cfg = dg.make_config(w)
    for k, v in over.items():
        setattr(cfg, k, v)
    out = ctypes.c_void_p()
    return lib.dg_init_weights(ctypes.byref(cfg), 0, None, ctypes.byref(out))


@pytest.mark.parametrize("field,value", [
    ("canvas_len", 128), ("head_dim", 96), ("n_kv_heads", 3), ("d_model", 100), ("vocab", 1000),
    ("top_k", 0), ("max_steps", 0), ("commit_mode", 7), ("stop_mode", 7), ("max_canvases", 0),
    ("sample_topk", 257), ("sample_topk", -1), ("expert_fp8", 2),
])
def test_invalid_configs_are_rejected_before_any_device_call(lib, field, value):
    assert _init_status(lib, I.TINY_FP32, **{field: value}) == 1


def test_fp8_experts_need_bf16(lib):
    assert _init_status(lib, I.TINY_FP32, expert_fp8=1) == 1


def test_hook_arguments_are_checked_before_any_device_call(lib):
    P = ctypes.c_void_p(1)   # never dereferenced: the checks fail first
    # top-k sampler: K = 0, K > 256, vocab not a multiple of 32
    for K, V in ((0, 1024), (257, 1024), (16, 1000)):
        assert lib.dg_test_sampler_topk(P, 4, V, 4, 0, 0, 0.5, 0.8, 0.4, K, P, P, P, None, None, P, P, 0, None) == 1
    # FP8 GEMM: K not a multiple of 16, unsupported tile
    c = (ctypes.c_int32 * 1)(4)
    assert lib.dg_test_grouped_gemm_fp8(P, P, P, c, 1, 128, 100, 64, 1, P, None) == 1
    assert lib.dg_test_grouped_gemm_fp8(P, P, P, c, 1, 128, 128, 48, 1, P, None) == 1
    # routing bias: n_tok not a multiple of 256
    assert lib.dg_set_routing_bias(None, P, 100) == 1


@pytest.mark.parametrize("A,B,out", [
    ((256, 64, "bf16"), (32, 64, "bf16"), (32, 128, "f32")),   # out too small for [N, M]
    ((256, 64, "bf16"), (32, 48, "bf16"), (32, 256, "f32")),   # B's K differs from A's
    ((256, 64, "f32"), (32, 64, "bf16"), (32, 256, "f32")),    # A not bf16
    ((256, 64, "bf16"), (32, 64, "bf16"), (32, 256, "bf16")),  # out not fp32
])
def test_noalloc_binding_rejects_mismatched_tensors_before_any_call(A, B, out):
    # the allocation-free GEMM writes out[N][M] through a raw pointer: a
    # wrong shape or dtype must be refused on the host
    torch = pytest.importorskip("torch")
    dt = {"bf16": torch.bfloat16, "f32": torch.float32}
    mk = lambda r, c, t: torch.zeros((r, c), dtype=dt[t])
    with pytest.raises(ValueError):
        dg.gemm_splitk_noalloc(mk(*A), mk(*B), mk(*out))


def test_noalloc_binding_rejects_non_contiguous_operands():
    torch = pytest.importorskip("torch")
    A = torch.zeros((64, 256), dtype=torch.bfloat16).t()      # [256, 64], not contiguous
    B = torch.zeros((32, 64), dtype=torch.bfloat16)
    out = torch.zeros((32, 256), dtype=torch.float32)
    with pytest.raises(ValueError):
        dg.gemm_splitk_noalloc(A, B, out)


def launch_shape(lib, vocab, rows, n_experts, n_pairs):
    out = (ctypes.c_int32 * 2)()
    assert lib.dg_test_launch_shape(vocab, rows, n_experts, n_pairs, out) == 0
    return list(out)


@pytest.mark.parametrize("vocab,rows,want", [
    (262144, 256, 8),            # 26B vocabulary: 8 CTAs per row at every batch
    (262144, 8192, 8),
    (32768, 256, 2),             # one canvas: too few rows to give every SM four CTAs alone
    (32768, 1024, 1),            # four canvases and more: one CTA per row
    (32768, 8192, 1),
    (1024, 256, 2),
    (65536, 4 * SMS, 1),         # the boundaries
    (65536, 4 * SMS - 1, 2),
    (65600, 4 * SMS, 8),
])
def test_sampler_cluster_size_rule(lib, vocab, rows, want):
    assert launch_shape(lib, vocab, rows, 128, 2048)[0] == want


def test_permute_and_gather_fuse_while_the_permutation_fits_shared_memory(lib):
    # 1024 threads: 32 warp histograms of E ints, the offsets, then one int per pair
    def fits(E, n_pairs):
        return (32 * E + E + 1) * 4 + n_pairs * 4 <= 96 * 1024
    for E, k in ((128, 8), (32, 4), (8, 2)):
        for B in (1, 4, 8, 9, 10, 16, 22, 23, 32):
            n = B * 256 * k
            assert launch_shape(lib, 32768, 256, E, n)[1] == int(fits(E, n)), (E, k, B)
    assert launch_shape(lib, 32768, 256, 128, 9 * 256 * 8)[1] == 1    # 26B shape: up to 9 canvases
    assert launch_shape(lib, 32768, 256, 128, 10 * 256 * 8)[1] == 0


def test_launch_shape_rejects_bad_sizes(lib):
    out = (ctypes.c_int32 * 2)()
    assert lib.dg_test_launch_shape(0, 256, 128, 2048, out) != 0
    assert lib.dg_test_launch_shape(32768, 256, 128, 0, out) != 0
    assert lib.dg_test_launch_shape(32768, 256, 128, 2048, None) != 0
