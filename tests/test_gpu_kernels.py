"""Kernel-level parity of the CUDA library against the oracle (B200 only).

Integer and fixed-sequence work (Philox, the binary32 log/exp/cos, weight
values, sampled tokens, argmax, entropy, commit masks, stop flags) must be
bit-exact.  Tensor-core work is compared within tolerances derived from the
arithmetic: fp32 accumulation of bf16 products (GEMM) and bf16 rounding of
the softmax weights (attention)."""
import os

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_text_diffusion_b200 as dg  # noqa: E402
from block_text_diffusion_b200 import inputs as I  # noqa: E402
from oracle import _native, numerics as nm, sampler as sp, model as om  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
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


def bf16_tensor(a32):
    """float32 array holding bf16 values -> exact torch bf16 tensor."""
    return cu(a32.astype(np.float32)).to(torch.bfloat16)


# --- Philox and fixed-sequence math -------------------------------------------
def test_philox_known_answers_on_gpu():
    rows = []
    for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")):
        if line.strip() and not line.startswith("#"):
            rows.append([int(w, 16) for w in line.split()])
    g = np.random.default_rng(0)
    extra = g.integers(0, 2 ** 32, size=(4096, 6), dtype=np.uint64).astype(np.uint32)
    inp = np.concatenate([np.array([r[:6] for r in rows], np.uint32), extra])
    out = torch.empty((inp.shape[0], 4), dtype=torch.int32, device="cuda")
    dg.test_philox(cu(inp.view(np.int32)), out)
    got = host(out).view(np.uint32)
    for i, r in enumerate(rows):
        assert list(got[i]) == r[6:]
    ref = np.stack(nm.philox4x32_10(*[extra[:, j] for j in range(6)]), axis=1)
    assert np.array_equal(got[len(rows):], ref)


def _math(which, x):
    xt = cu(x)
    out = torch.empty(x.shape, dtype=torch.float32, device="cuda")
    dg.test_math(which, xt, out)
    return host(out)


def test_log_bit_exact_on_sampler_domain():
    n = np.arange(0, 2 ** 23, dtype=np.uint32)
    u = (n * 2 + 1).astype(F32) * F32(2.0 ** -24)
    ref = nm.chunked(nm.log_f32, u)
    assert np.array_equal(_math(0, u).view(np.uint32), ref.view(np.uint32))
    x = -ref
    assert np.array_equal(_math(0, x).view(np.uint32), nm.chunked(nm.log_f32, x).view(np.uint32))
    g = np.random.default_rng(1)
    w = g.integers(0x00800000, 0x7F800000, size=1 << 20, dtype=np.uint64).astype(np.uint32).view(F32)
    assert np.array_equal(_math(0, w).view(np.uint32), nm.chunked(nm.log_f32, w).view(np.uint32))


def test_exp_cos_gumbel_bit_exact():
    x = np.concatenate([np.linspace(-90, 0, 1 << 21).astype(F32), np.array([0.0, -86.0, -85.99, -1e-30], F32)])
    assert np.array_equal(_math(1, x).view(np.uint32), nm.chunked(nm.exp_f32, x).view(np.uint32))
    n = np.arange(0, 2 ** 23, 3, dtype=np.uint32)
    u = (n * 2 + 1).astype(F32) * F32(2.0 ** -24)
    assert np.array_equal(_math(2, u).view(np.uint32), nm.chunked(nm.cos2pi_f32, u).view(np.uint32))
    w = np.random.default_rng(2).integers(0, 2 ** 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    ref = nm.chunked(lambda a: -nm.log_f32(-nm.log_f32(nm.uniform_open(a))), w)
    assert np.array_equal(_math(3, w.view(np.int32)).view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("seed,tid", [(0, 0), (2, 16 + 16 * 29 + 5), ((5 << 32) + 7, 123)])
def test_weight_values_bit_exact(seed, tid):
    g = np.random.default_rng(3)
    idx = np.concatenate([np.arange(4096, dtype=np.uint64),
                          g.integers(0, 1 << 34, size=8192, dtype=np.uint64)])
    xt = cu(idx.view(np.int64))
    out = torch.empty(idx.shape, dtype=torch.float32, device="cuda")
    dg.test_math(4, xt, out, aux0=seed, aux1=tid)
    got = host(out)
    ref = np.concatenate([om._normal_weights(seed, tid, int(j), 1, False) for j in idx[4096:]])
    ref = np.concatenate([om._normal_weights(seed, tid, 0, 4096, False), ref])
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


# --- vocab sampler -----------------------------------------------------------------
def _oracle_rows(l, positions, seed, step, inv_t):
    R = l.shape[0]
    outs = {k: [] for k in ("H", "amax", "tokens", "S_q", "U_q", "p")}
    for c0 in range(0, R, positions):
        blk = l[c0:c0 + positions]
        r = _native.sampler_rows(blk, seed, c0 // positions, 0, step, inv_t, True) if _native.lib() else None
        if r is None:
            st = sp.row_stats(blk, want_probs=True)
            st["tokens"] = sp.sample_tokens(blk, inv_t, seed, c0 // positions, step)
            r = st
        for k in outs:
            outs[k].append(r[k])
    return {k: np.concatenate(v) for k, v in outs.items()}


@pytest.mark.parametrize("V,rows,positions,kind,scale,bf", [
    (1024, 256, 256, "normal", 1.0, False),
    (1024, 300, 256, "mixed", 3.0, False),      # ragged: a second canvas of 44 rows
    (32768, 64, 32, "peaked", 1.0, True),
    (32768, 16, 16, "ties", 1.0, True),
    (32768, 8, 8, "flat", 1.0, True),
    (262144, 12, 6, "normal", 4.0, True),
    (262144, 4, 4, "mixed", 16.0, True),
])
def test_sampler_bit_exact(V, rows, positions, kind, scale, bf):
    l = I.logits(V + rows, rows, V, kind, scale)
    step, t, seed = 5, 0.37, (3 << 32) + 11
    T = sp.temperature(F32(t))
    inv_t = F32(1.0) / T
    ref = _oracle_rows(l, positions, seed, step, inv_t)
    lt = cu(l)
    H = torch.empty(rows, dtype=torch.float32, device="cuda")
    tok = torch.empty(rows, dtype=torch.int32, device="cuda")
    am = torch.empty(rows, dtype=torch.int32, device="cuda")
    sq = torch.empty(rows, dtype=torch.int64, device="cuda")
    uq = torch.empty(rows, dtype=torch.int64, device="cuda")
    pr = torch.empty((rows, V), dtype=torch.bfloat16 if bf else torch.float32, device="cuda")
    dg.test_sampler(lt, positions, seed, step, t, 0.8, 0.4, H, tok, am, sq, uq, pr)
    assert np.array_equal(host(sq), ref["S_q"]) and np.array_equal(host(uq), ref["U_q"])
    assert np.array_equal(host(H).view(np.uint32), ref["H"].view(np.uint32))
    assert np.array_equal(host(am), ref["amax"])
    assert np.array_equal(host(tok), ref["tokens"])
    p = host(pr.float())
    pref = nm.round_bf16_from_f32(ref["p"]) if bf else ref["p"]
    assert np.array_equal(p.view(np.uint32), pref.view(np.uint32))


def test_sampler_uniform_entropy_is_log_v():
    V = 262144
    l = np.full((2, V), -1.25, F32)
    H = torch.empty(2, dtype=torch.float32, device="cuda")
    tok = torch.empty(2, dtype=torch.int32, device="cuda")
    am = torch.empty(2, dtype=torch.int32, device="cuda")
    dg.test_sampler(cu(l), 256, 1, 0, 1.0, 0.8, 0.4, H, tok, am)
    assert np.allclose(host(H), np.log(V), atol=2e-6)
    assert np.array_equal(host(am), [0, 0])


# --- top-k-truncated sampler -----------------------------------------------------------
@pytest.mark.parametrize("V,rows,positions,kind,scale,K,bf", [
    (1024, 256, 256, "normal", 1.0, 256, False),
    (1024, 300, 256, "mixed", 3.0, 64, False),     # ragged: a second canvas of 44 rows
    (32768, 64, 32, "peaked", 1.0, 64, True),
    (32768, 16, 16, "ties", 1.0, 200, True),       # many equal logits across the K-th place
    (32768, 8, 8, "flat", 1.0, 32, True),          # every logit equal: the K lowest ids
    (262144, 8, 8, "normal", 4.0, 64, True),
    (262144, 4, 4, "mixed", 16.0, 256, True),
    (4096, 16, 16, "normal", 1.0, 1, False),
])
def test_sampler_topk_bit_exact(V, rows, positions, kind, scale, K, bf):
    l = I.logits(V + rows + K, rows, V, kind, scale)
    step, t, seed = 3, 0.61, (7 << 32) + 5
    inv_t = F32(1.0) / sp.temperature(F32(t))
    ref = {k: [] for k in ("H", "amax", "tokens", "S_q", "U_q", "cand_ids", "cand_w")}
    for c0 in range(0, rows, positions):
        r = sp.sampler_rows_topk(l[c0:c0 + positions], K, inv_t, seed, c0 // positions, step)
        for k in ref:
            ref[k].append(r[k])
    ref = {k: np.concatenate(v) for k, v in ref.items()}
    z = lambda dt, *shape: torch.empty(shape, dtype=dt, device="cuda")
    H, tok, am = z(torch.float32, rows), z(torch.int32, rows), z(torch.int32, rows)
    sq, uq = z(torch.int64, rows), z(torch.int64, rows)
    ids, wts = z(torch.int32, rows, K), z(torch.bfloat16 if bf else torch.float32, rows, K)
    dg.test_sampler_topk(cu(l), positions, seed, step, t, 0.8, 0.4, K, H, tok, am, ids, wts, sq, uq)
    assert np.array_equal(host(sq), ref["S_q"]) and np.array_equal(host(uq), ref["U_q"])
    assert np.array_equal(host(H).view(np.uint32), ref["H"].view(np.uint32))
    assert np.array_equal(host(am), ref["amax"])
    assert np.array_equal(host(ids), ref["cand_ids"])
    assert np.array_equal(host(tok), ref["tokens"])
    wref = nm.round_bf16_from_f32(ref["cand_w"]) if bf else ref["cand_w"]
    assert np.array_equal(host(wts.float()).view(np.uint32), wref.view(np.uint32))


@pytest.mark.parametrize("rows,K,d,bf", [(256, 64, 2816, True), (300, 16, 256, False), (8, 256, 1024, True)])
def test_sc_gather(rows, K, d, bf):
    g = np.random.default_rng(rows + K)
    V = 4096
    emb = g.standard_normal((V, d)).astype(F32) * F32(0.02)
    ids = np.stack([g.choice(V, size=K, replace=False) for _ in range(rows)]).astype(np.int32)
    w = g.dirichlet(np.ones(K), size=rows).astype(F32)
    if bf:
        emb, w = nm.round_bf16_from_f32(emb), nm.round_bf16_from_f32(w)
    dt = torch.bfloat16 if bf else torch.float32
    u = torch.empty((rows, d), dtype=dt, device="cuda")
    dg.test_sc_gather(cu(ids), cu(w).to(dt), cu(emb).to(dt), u)
    ref = np.einsum("rk,rkd->rd", w.astype(np.float64), emb[ids].astype(np.float64))
    got = host(u.float())
    # fp32 accumulation of K products, then the storage rounding
    bound = (2.0 ** -8 if bf else 1e-6) * np.abs(ref) + K * 2e-7 * np.einsum(
        "rk,rkd->rd", np.abs(w.astype(np.float64)), np.abs(emb[ids].astype(np.float64)))
    assert np.all(np.abs(got - ref) <= bound + 1e-12)


# --- commit / stop -------------------------------------------------------------------
@pytest.mark.parametrize("mode,bound,stop_mode,stop_bound,step,ties,same", [
    (0, 0.5, 0, 0.1, 3, False, False),
    (0, 0.5, 0, 0.1, 47, False, False),     # last round always stops
    (1, 0.1, 1, 0.005, 4, False, True),
    (1, 0.1, 1, 0.005, 4, True, True),      # many exactly tied entropies
    (1, 0.1, 1, 0.005, 0, False, True),     # EB stop never at round 0
    (1, 0.1, 1, 0.005, 9, False, False),
    (1, 0.1, 0, 0.1, 2, True, False),
])
def test_commit_bit_exact(mode, bound, stop_mode, stop_bound, step, ties, same):
    B, V, seed, max_steps = 5, 4096, 77, 48
    H = I.entropies(step + 3, B, low_frac=0.9, ties=ties)
    H[1] = np.float32(0.001)                # a canvas under every bound
    H[2] = np.float32(3.0)                  # a canvas over every bound
    H[3, :7] = np.float32(0.0)
    tok = I.token_ids(1, (B, 256), V)
    amax = I.token_ids(2, (B, 256), V)
    prev = amax.copy() if same else I.token_ids(3, (B, 256), V)
    prev_t = cu(prev)
    commit = torch.empty((B, 256), dtype=torch.uint8, device="cuda")
    nxt = torch.empty((B, 256), dtype=torch.int32, device="cuda")
    stop = torch.empty(B, dtype=torch.int32, device="cuda")
    ncom = torch.empty(B, dtype=torch.int32, device="cuda")
    dg.test_commit(cu(H), cu(tok), cu(amax), prev_t, V, seed, step, max_steps, mode, bound, stop_mode,
                   stop_bound, commit, nxt, stop, ncom)
    gc, gn, gs, gk = host(commit), host(nxt), host(stop), host(ncom)
    for b in range(B):
        m = sp.commit_mask(H[b], mode, bound)
        assert np.array_equal(gc[b], m), b
        assert gk[b] == m.sum()
        assert np.array_equal(gn[b], sp.next_canvas(tok[b], m, seed, b, step, V))
        assert bool(gs[b]) == sp.stop_decision(H[b], m, amax[b], prev[b], step, max_steps, stop_mode, stop_bound)
    assert np.array_equal(host(prev_t), amax)


# --- GEMMs ----------------------------------------------------------------------------
def _bound(a, b):
    return np.abs(a.astype(np.float64)) @ np.abs(b.astype(np.float64)).T


@pytest.mark.parametrize("M,N,K,bn,splits", [
    (128, 16, 64, 32, 1), (256, 256, 512, 256, 1), (300, 200, 200, 256, 1), (1536, 256, 1024, 256, 4),
    (4096, 256, 2816, 256, 4), (1000, 40, 72, 64, 1), (640, 100, 4096, 128, 8), (128, 1, 64, 32, 1)])
@pytest.mark.parametrize("persistent", [False, True])
def test_gemm_bf16(M, N, K, bn, splits, persistent):
    g = np.random.default_rng(M + N + K)
    A = I._bf16_grid(g.standard_normal((M, K)).astype(F32))
    B = I._bf16_grid(g.standard_normal((N, K)).astype(F32))
    out = torch.zeros((splits, N, M), dtype=torch.float32, device="cuda")
    dg.test_gemm(bf16_tensor(A), bf16_tensor(B), out, alpha=0.5, k_splits=splits, bn=bn, persistent=persistent)
    got = host(out).astype(np.float64).sum(axis=0)
    ref = 0.5 * (B.astype(np.float64) @ A.astype(np.float64).T)
    err = np.abs(got - ref)
    assert np.all(err <= 2e-6 * 0.5 * _bound(B, A) + 1e-30), err.max()


@pytest.mark.parametrize("M,N,K,splits", [
    (256, 256, 512, 1), (300, 200, 200, 1), (785, 256, 1024, 3), (4096, 256, 2816, 4), (2000, 33, 4096, 16)])
def test_gemm_bf16_256_row_tiles(M, N, K, splits):
    # two accumulators per CTA sharing each B tile (the vocabulary GEMMs);
    # ragged M (a tile whose second half is partly or wholly outside M)
    g = np.random.default_rng(M * 7 + N + K)
    A = I._bf16_grid(g.standard_normal((M, K)).astype(F32))
    B = I._bf16_grid(g.standard_normal((N, K)).astype(F32))
    out = torch.zeros((splits, N, M), dtype=torch.float32, device="cuda")
    dg.test_gemm(bf16_tensor(A), bf16_tensor(B), out, alpha=0.5, k_splits=splits, bn=256, m256=True)
    got = host(out).astype(np.float64).sum(axis=0)
    ref = 0.5 * (B.astype(np.float64) @ A.astype(np.float64).T)
    assert np.all(np.abs(got - ref) <= 2e-6 * 0.5 * _bound(B, A) + 1e-30), np.abs(got - ref).max()


def test_gemm_f32():
    g = np.random.default_rng(5)
    M, N, K = 1000, 256, 300
    A = g.standard_normal((M, K)).astype(F32)
    B = g.standard_normal((N, K)).astype(F32)
    out = torch.zeros((2, N, M), dtype=torch.float32, device="cuda")
    dg.test_gemm(cu(A), cu(B), out, alpha=1.0, k_splits=2)
    got = host(out).astype(np.float64).sum(axis=0)
    ref = B.astype(np.float64) @ A.astype(np.float64).T
    assert np.all(np.abs(got - ref) <= 2e-6 * _bound(B, A))


@pytest.mark.parametrize("M,K,counts,bn,bf", [
    (1408, 256, [0, 1, 17, 64, 65, 300, 0, 3], 64, True),
    (512, 704, [16] * 20 + [0, 33, 2], 64, True),
    (2816, 128, [5, 0, 0, 130, 256, 257], 256, True),
    (1024, 128, [7, 0, 70, 1], 128, True),
    (1024, 256, [0, 9, 64, 65, 1], 64, False),
    (1408, 2816, [17, 3, 0, 31, 12, 1, 9, 20], 256, True),
])
@pytest.mark.parametrize("persistent", [False, True, "sized_ring", "m256"])
def test_grouped_gemm(M, K, counts, bn, bf, persistent):
    g = np.random.default_rng(sum(counts) + M)
    G = len(counts)
    rows = sum(counts)
    A = g.standard_normal((G * M, K)).astype(F32)
    B = g.standard_normal((rows, K)).astype(F32)
    if bf:
        A, B = I._bf16_grid(A), I._bf16_grid(B)
    At = bf16_tensor(A) if bf else cu(A)
    Bt = bf16_tensor(B) if bf else cu(B)
    out = torch.full((rows, M), float("nan"), dtype=torch.float32, device="cuda")
    # "sized_ring": the persistent kernel's ring stages shrink to the largest
    # item (more stages in flight), as the expert GEMMs run in the step
    # "m256": 256-row tiles (two accumulators), as the expert GEMMs run, with the
    # ring sized from the largest item
    dg.test_grouped_gemm(At, Bt, counts, G, M, out, bn=bn, persistent=bool(persistent) and bf,
                         sized_ring=persistent in ("sized_ring", "m256") and bf,
                         m256=persistent == "m256" and bf and bn == 256)
    got = host(out).astype(np.float64)
    r0 = 0
    for e, c in enumerate(counts):
        if c:
            Ae = A[e * M:(e + 1) * M]
            ref = B[r0:r0 + c].astype(np.float64) @ Ae.astype(np.float64).T
            assert np.all(np.abs(got[r0:r0 + c] - ref) <= 2e-6 * _bound(B[r0:r0 + c], Ae)), e
        r0 += c


@pytest.mark.parametrize("M,K,counts", [(1408, 2816, [17, 3, 0, 200, 12, 1, 256, 20]), (2048, 1024, [64, 65, 0, 9]),
                                         (1408, 2816, [300, 1, 0, 5]), (1408, 2816, [16] * 120 + [40])])
@pytest.mark.parametrize("m256", [False, True])
def test_grouped_gemm_fused_swiglu(M, K, counts, m256):
    # the unsplit gate|up GEMM writes round(silu(g) u) itself; A rows interleave
    # gate / up in blocks of 64
    g = np.random.default_rng(M + K + sum(counts))
    G, rows, ff = len(counts), sum(counts), M // 2
    A = I._bf16_grid((0.05 * g.standard_normal((G * M, K))).astype(F32))
    B = I._bf16_grid(g.standard_normal((rows, K)).astype(F32))
    out = torch.zeros((rows, M), dtype=torch.float32, device="cuda")
    dg.test_grouped_gemm(bf16_tensor(A), bf16_tensor(B), counts, G, M, out, bn=256, persistent=True,
                         sized_ring=True, swiglu=True, m256=m256)
    act = out.view(torch.bfloat16).reshape(-1)[:rows * ff].reshape(rows, ff)
    got = act.float().cpu().numpy().astype(np.float64)
    f = np.arange(ff)
    grow, urow = (f // 64) * 128 + f % 64, (f // 64) * 128 + 64 + f % 64
    r0 = 0
    for e, c in enumerate(counts):
        if c:
            Ae = A[e * M:(e + 1) * M].astype(np.float64)
            x = B[r0:r0 + c].astype(np.float64)
            gv, uv = x @ Ae[grow].T, x @ Ae[urow].T
            ref = gv / (1.0 + np.exp(-gv)) * uv
            sg, su = np.abs(x) @ np.abs(Ae[grow]).T, np.abs(x) @ np.abs(Ae[urow]).T
            tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * (sg * (np.abs(uv) + 1.0) + su * (np.abs(gv) + 1.0))
            assert np.all(np.abs(got[r0:r0 + c] - ref) <= tol), e
        r0 += c


# --- router -----------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,E,k,zipf,pool", [(256, 2816, 128, 8, 0.0, 0), (77, 1024, 32, 4, 0.0, 0),
                                               (1024, 1024, 32, 4, 1.1, 0), (40, 512, 100, 5, 0.0, 0),
                                               (256, 2816, 128, 8, 0.0, 84), (512, 1024, 32, 4, 1.1, 16)])
def test_router_kernel(T, d, E, k, zipf, pool):
    # top-k ids identical to the oracle's wherever the decision is farther
    # from a tie than the fp32 accumulation error can move it; gates within
    # 1e-4 of the fp64 softmax.  pool > 0 adds a per-token bias (beta 2, of
    # the order of the logit spread, so selection depends on both terms)
    g = np.random.default_rng(T + d + E)
    x = I._bf16_grid(g.standard_normal((T, d)).astype(F32))
    wr = I._bf16_grid((0.02 * g.standard_normal((E, d))).astype(F32))
    bias = None
    if zipf:
        bias = cu((-zipf * np.log(np.arange(E, dtype=np.float64) + 1.0)).astype(F32))
    tb = I.routing_bias(T, 1, T, E, k, pool, beta=2.0)[0] if pool else None
    ids = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    gate = torch.zeros((T, k), dtype=torch.float32, device="cuda")
    dg.test_router(bf16_tensor(x), bf16_tensor(wr), ids, gate, bias=bias, tok_bias=cu(tb) if pool else None)
    gi, gg = host(ids), host(gate)
    oi, ow = om.router(x, wr, k, zipf_s=zipf, extra=tb)
    r = om.router_logits(x, wr, zipf, tb)
    # fp32 accumulation error bound, plus the binary32 rounding of the biases
    err = 4e-6 * (np.abs(x.astype(np.float64)) @ np.abs(wr.astype(np.float64)).T).max(axis=1) + 1e-6 + 1e-5 * zipf
    srt = -np.sort(-r, axis=1)
    gaps = srt[:, :k] - srt[:, 1:k + 1]                       # adjacent gaps through the (k+1)-th
    safe_set = gaps[:, k - 1] > 2 * err
    safe_order = gaps.min(axis=1) > 2 * err
    assert safe_order.mean() > 0.5
    for t in range(T):
        if safe_order[t]:
            assert np.array_equal(gi[t], oi[t]), t
        elif safe_set[t]:
            assert set(gi[t]) == set(oi[t]), t
    assert np.allclose(gg[safe_order], ow[safe_order], atol=1e-4)
    assert np.allclose(gg.sum(axis=1), 1.0, atol=1e-5)


# --- attention --------------------------------------------------------------------------
def _attn_ref(q, k, v, n_canvas, n_q, q_pos0, causal, rows=None):
    out = []
    for b in range(n_canvas):
        qb = q[b * n_q:(b + 1) * n_q].astype(np.float64)
        kb = k[b].transpose(1, 0, 2).astype(np.float64)
        vb = v[b].transpose(1, 0, 2).astype(np.float64)
        out.append(om.attention(qb, kb, vb, causal_offset=q_pos0 if causal else None))
    return np.concatenate(out).reshape(n_canvas * n_q, -1)


@pytest.mark.parametrize("n_canvas,n_q,q_pos0,n_keys,causal,Hq,Hkv,bf", [
    (1, 256, 100, 356, False, 16, 8, True),
    (2, 256, 1024, 1280, False, 8, 2, True),
    (1, 256, 2048, 2304, False, 16, 8, True),
    (1, 200, 0, 200, True, 8, 2, True),          # causal, ragged query tile
    (1, 384, 128, 512, True, 16, 8, True),      # causal chunk after a prefix
    (1, 256, 64, 320, False, 4, 4, False),
    (1, 64, 0, 64, True, 4, 4, False),
])
@pytest.mark.parametrize("path", [0, 1, 2])
def test_attention(n_canvas, n_q, q_pos0, n_keys, causal, Hq, Hkv, bf, path):
    # path 0: the plan's choice; 1: split partials + combine kernel; 2: the
    # splits of a query-tile pair merged inside the kernel (thread-block cluster)
    if path and not bf:
        pytest.skip("the merge paths are the bf16 kernel's")
    g = np.random.default_rng(n_keys + Hq)
    hd = 128 if bf else 64
    q = g.standard_normal((n_canvas * n_q, Hq, hd)).astype(F32)
    k = g.standard_normal((n_canvas, Hkv, n_keys, hd)).astype(F32)
    v = g.standard_normal((n_canvas, Hkv, n_keys, hd)).astype(F32)
    if bf:
        q, k, v = I._bf16_grid(q), I._bf16_grid(k), I._bf16_grid(v)
    mk = bf16_tensor if bf else cu
    out = torch.empty((n_canvas * n_q, Hq * hd), dtype=torch.float32, device="cuda")
    took = dg.test_attention(mk(q), mk(k), mk(v), n_canvas, n_q, q_pos0, n_keys, causal, Hq, Hkv, out,
                             force_path=path)
    if path:
        assert took == path
    got = host(out)
    ref = _attn_ref(q, k, v, n_canvas, n_q, q_pos0, causal)
    tol = 1.2e-2 if bf else 1e-5
    assert np.abs(got - ref).max() <= tol, np.abs(got - ref).max()


@pytest.mark.parametrize("path", [0, 2])
def test_attention_long_context_sampled_rows(path):
    # 256 canvas queries over 32768 prompt + 256 canvas keys (split-KV path);
    # rows checked one by one against the definition.
    n_q, P, Hq, Hkv, hd = 256, 32768, 8, 2, 128
    n_keys = P + n_q
    g = np.random.default_rng(11)
    q = I._bf16_grid(g.standard_normal((n_q, Hq, hd)).astype(F32))
    k = I._bf16_grid(g.standard_normal((1, Hkv, n_keys, hd)).astype(F32))
    v = I._bf16_grid(g.standard_normal((1, Hkv, n_keys, hd)).astype(F32))
    out = torch.empty((n_q, Hq * hd), dtype=torch.float32, device="cuda")
    dg.test_attention(bf16_tensor(q), bf16_tensor(k), bf16_tensor(v), 1, n_q, P, n_keys, False, Hq, Hkv, out,
                      force_path=path)
    got = host(out).reshape(n_q, Hq, hd)
    for t in (0, 1, 77, 128, 255):
        for h in (0, 3, 7):
            kk = k[0, h // 4].astype(np.float64)
            s = kk @ q[t, h].astype(np.float64) / np.sqrt(hd)
            p = np.exp(s - s.max())
            ref = (p / p.sum()) @ v[0, h // 4].astype(np.float64)
            assert np.abs(got[t, h] - ref).max() <= 1.2e-2


@pytest.mark.parametrize("V,d,scale", [(262144, 2816, 1.0), (32768, 1024, 4.0), (32768, 1024, 16.0)])
def test_lm_head_within_2e2_given_same_inputs(V, d, scale):
    # The LM head's own arithmetic (tied embedding, fp32 accumulation, logit
    # scale) meets the 2e-2 absolute logit bound when both sides see the same
    # bf16 normalised states: unit-rms rows and N(0, 0.02) embeddings.
    g = np.random.default_rng(V + d)
    x = g.standard_normal((256, d))
    x /= np.sqrt((x ** 2).mean(axis=1, keepdims=True))
    x = I._bf16_grid(x.astype(F32))
    E = I._bf16_grid((g.standard_normal((V, d)) * 0.02).astype(F32))
    out = torch.zeros((1, 256, V), dtype=torch.float32, device="cuda")
    dg.test_gemm(bf16_tensor(E), bf16_tensor(x), out, alpha=scale, k_splits=1, bn=256)
    got = host(out)[0].astype(np.float64)
    ref = scale * (x.astype(np.float64) @ E.astype(np.float64).T)
    assert np.abs(got - ref).max() <= 2e-2
