"""Pins of the model oracle: a pure-Python brute-force forward on micro shapes
(explicit index loops, complex-number RoPE, Python sorting), plus invariants
the pages fix -- 256-wide canvas, bidirectional canvas attention, causal
prompt, top-k weights summing to 1, stop on low entropy (CPU only)."""
import cmath
import math

import numpy as np
import pytest

from block_text_diffusion_b200 import inputs as I
from oracle import model as om, sampler as sp

F32 = np.float32

MICRO = I.Workload("micro", n_layers=2, d_model=8, n_heads=2, n_kv_heads=1, head_dim=4,
                   n_experts=4, top_k=2, d_ff=6, vocab=16, dtype=I.DTYPE_FP32, logit_scale=2.0,
                   max_steps=4, weight_seed=21, sample_seed=5, prompt_len=5)


class BruteWeights:
    """Every weight fetched one by one by (tensor, row-major index)."""

    def __init__(self, cfg):
        self.cfg, self.cache = cfg, {}

    def __call__(self, tid, idx, shape):
        flat = 0
        for i, n in zip(idx, shape):
            assert 0 <= i < n
            flat = flat * n + i
        key = (tid, flat)
        if key not in self.cache:
            self.cache[key] = om.weight_element(self.cfg.weight_seed, tid, flat, bf16=False)
        return self.cache[key]


def r32(x):
    return float(np.float32(x))


def bf_block(cfg, W, l, h, positions, kpre, vpre, causal):
    d, H, G, hd, E, ff = cfg.d_model, cfg.n_heads, cfg.n_kv_heads, cfg.head_dim, cfg.n_experts, cfg.d_ff
    tid = lambda w: om.layer_tensor_id(l, w)
    n = len(h)

    def norm(v):
        ms = sum(a * a for a in v) / len(v)
        return [r32(a / math.sqrt(ms + cfg.rms_eps)) for a in v]

    def rot(vec, pos):
        out = list(vec)
        for c in range(hd // 2):
            z = complex(vec[c], vec[c + hd // 2]) * cmath.exp(1j * pos * cfg.rope_theta ** (-2 * c / hd))
            out[c], out[c + hd // 2] = z.real, z.imag
        return out

    x = [norm(v) for v in h]
    q = [[[r32(a) for a in rot([sum(W(tid("wq"), (hh * hd + c, i), (H * hd, d)) * x[t][i] for i in range(d))
                                 for c in range(hd)], positions[t])] for hh in range(H)] for t in range(n)]
    k = [[[r32(a) for a in rot([sum(W(tid("wk"), (g * hd + c, i), (G * hd, d)) * x[t][i] for i in range(d))
                                 for c in range(hd)], positions[t])] for g in range(G)] for t in range(n)]
    v = [[[r32(sum(W(tid("wv"), (g * hd + c, i), (G * hd, d)) * x[t][i] for i in range(d)))
           for c in range(hd)] for g in range(G)] for t in range(n)]
    keys = kpre + k
    vals = vpre + v
    o = []
    for t in range(n):
        row = []
        for hh in range(H):
            g = hh // (H // G)
            vis = [j for j in range(len(keys)) if not causal or j <= len(kpre) + t]
            sc = [sum(q[t][hh][c] * keys[j][g][c] for c in range(hd)) / math.sqrt(hd) for j in vis]
            mx = max(sc)
            ex = [math.exp(s - mx) for s in sc]
            z = sum(ex)
            row += [r32(sum(ex[a] / z * vals[j][g][c] for a, j in enumerate(vis))) for c in range(hd)]
        o.append(row)
    h = [[r32(h[t][i] + sum(W(tid("wo"), (i, c), (d, H * hd)) * o[t][c] for c in range(H * hd)))
          for i in range(d)] for t in range(n)]
    x2 = [norm(vv) for vv in h]
    out = []
    for t in range(n):
        logit = [sum(W(tid("wr"), (e, i), (E, d)) * x2[t][i] for i in range(d)) for e in range(E)]
        if cfg.zipf_s:
            logit = [a - cfg.zipf_s * math.log(e + 1) for e, a in enumerate(logit)]
        chosen = sorted(range(E), key=lambda e: (-logit[e], e))[:cfg.top_k]
        mx = max(logit[e] for e in chosen)
        gate = [math.exp(logit[e] - mx) for e in chosen]
        gate = [a / sum(gate) for a in gate]
        y = [0.0] * d
        for e, w in zip(chosen, gate):
            act = []
            for f in range(ff):
                gg = sum(W(tid("wg"), (e, f, i), (E, ff, d)) * x2[t][i] for i in range(d))
                uu = sum(W(tid("wu"), (e, f, i), (E, ff, d)) * x2[t][i] for i in range(d))
                act.append(r32(gg / (1 + math.exp(-gg)) * uu))
            for i in range(d):
                y[i] += w * sum(W(tid("wd"), (e, i, f), (E, d, ff)) * act[f] for f in range(ff))
        out.append([r32(h[t][i] + y[i]) for i in range(d)])
    return out, k, v


def bf_embed(cfg, W, ids):
    return [[W(om.T_EMBED, (int(t), i), (cfg.vocab, cfg.d_model)) for i in range(cfg.d_model)] for t in ids]


def bf_encode(cfg, W, prompt):
    h = bf_embed(cfg, W, prompt)
    K, V = [], []
    for l in range(cfg.n_layers):
        h, k, v = bf_block(cfg, W, l, h, list(range(len(prompt))), [], [], causal=True)
        K.append(k)
        V.append(v)
    return K, V


def bf_logits(cfg, W, K, V, canvas, selfcond=None):
    h = bf_embed(cfg, W, canvas)
    if selfcond is not None:
        h = [[r32(a + b) for a, b in zip(hr, sr)] for hr, sr in zip(h, selfcond)]
    P = len(K[0])
    for l in range(cfg.n_layers):
        h, _, _ = bf_block(cfg, W, l, h, [P + t for t in range(len(canvas))], K[l], V[l], causal=False)
    out = []
    for vec in h:
        ms = sum(a * a for a in vec) / len(vec)
        x = [r32(a / math.sqrt(ms + cfg.rms_eps)) for a in vec]
        out.append([cfg.logit_scale * sum(W(om.T_EMBED, (tok, i), (cfg.vocab, cfg.d_model)) * x[i]
                                          for i in range(cfg.d_model)) for tok in range(cfg.vocab)])
    return np.array(out)


@pytest.fixture(scope="module")
def micro():
    cfg = MICRO
    return cfg, om.Model(cfg), BruteWeights(cfg)


def _cache_to_lists(K):
    # oracle cache [L, Hkv, P, hd] -> brute [L][P][Hkv][hd]
    return [[[list(map(float, K[l, g, p])) for g in range(K.shape[1])] for p in range(K.shape[2])]
            for l in range(K.shape[0])]


@pytest.mark.parametrize("zipf", [0.0, 1.1])
def test_encode_and_canvas_forward_match_brute_force(micro, zipf):
    cfg, model, W = micro
    cfg = cfg.replace(zipf_s=zipf)
    model.cfg = cfg
    prompt = I.prompt_ids(1, 1, cfg.prompt_len, cfg.vocab)[0]
    K, V = om.encode_prompt(model, prompt)
    bK, bV = bf_encode(cfg, W, prompt)
    assert np.allclose(K, np.array(bK).transpose(0, 2, 1, 3), rtol=1e-6, atol=1e-7)
    assert np.allclose(V, np.array(bV).transpose(0, 2, 1, 3), rtol=1e-6, atol=1e-7)
    canvas = I.canvas_ids(2, 1, cfg.vocab)[0]
    sc = I.normal(3, 7, (256, cfg.d_model), std=0.05)
    logits, _ = om.forward_canvas(model, K, V, canvas, sc)
    ref = bf_logits(cfg, W, _cache_to_lists(K), _cache_to_lists(V), canvas, sc.tolist())
    assert logits.shape == (256, cfg.vocab)
    assert np.allclose(logits, ref, rtol=1e-5, atol=1e-6)
    model.cfg = MICRO


def test_self_conditioning_matches_brute_force(micro):
    cfg, model, W = micro
    p = np.abs(I.normal(4, 8, (256, cfg.vocab)))
    p = (p / p.sum(axis=1, keepdims=True)).astype(F32)
    s = om.self_condition(model, p)
    d = cfg.d_model
    for t in (0, 100, 255):
        u = [r32(sum(float(p[t, v]) * W(om.T_EMBED, (v, i), (cfg.vocab, d)) for v in range(cfg.vocab)))
             for i in range(d)]
        ref = [r32(sum(W(om.T_WSC, (o, i), (d, d)) * u[i] for i in range(d))) for o in range(d)]
        assert np.allclose(s[t], ref, rtol=1e-6, atol=1e-9)


def test_canvas_is_256_wide_and_bidirectional(micro):
    cfg, model, _ = micro
    K, V = I.prompt_kv(1, cfg.n_layers, 1, cfg.n_kv_heads, 7, cfg.head_dim, bf16=False)
    c = I.canvas_ids(3, 1, cfg.vocab)[0]
    a, _ = om.forward_canvas(model, K[:, 0], V[:, 0], c, None)
    c2 = c.copy()
    c2[255] = (c2[255] + 1) % cfg.vocab
    b, _ = om.forward_canvas(model, K[:, 0], V[:, 0], c2, None)
    assert a.shape[0] == 256
    # the first position sees the last one: bidirectional canvas attention
    assert np.abs(a[0] - b[0]).max() > 1e-6


def test_prompt_encode_is_causal(micro):
    cfg, model, _ = micro
    p = I.prompt_ids(5, 1, 9, cfg.vocab)[0]
    K1, V1 = om.encode_prompt(model, p)
    p2 = p.copy()
    p2[-1] = (p2[-1] + 3) % cfg.vocab
    K2, V2 = om.encode_prompt(model, p2)
    assert np.array_equal(K1[:, :, :-1], K2[:, :, :-1]) and np.array_equal(V1[:, :, :-1], V2[:, :, :-1])
    assert not np.array_equal(K1[:, :, -1], K2[:, :, -1])


def test_attention_special_cases():
    g = np.random.default_rng(0)
    q = g.standard_normal((3, 4, 8))
    k = g.standard_normal((1, 2, 8))
    v = g.standard_normal((1, 2, 8))
    o = om.attention(q, k, v)
    # one key: the output is that value, for every query and head
    assert np.allclose(o, np.repeat(v[:, [0, 0, 1, 1], :], 3, axis=0))
    k = g.standard_normal((6, 2, 8))
    v = g.standard_normal((6, 2, 8))
    # causal: query 0 with no prefix sees key 0 only
    oc = om.attention(q[:1], k, v, causal_offset=0)
    assert np.allclose(oc[0], v[0, [0, 0, 1, 1]])
    # bidirectional attention is invariant to permuting the keys with their values
    perm = g.permutation(6)
    assert np.allclose(om.attention(q, k, v), om.attention(q, k[perm], v[perm]))
    # identical keys: uniform weights -> mean of the values
    kk = np.repeat(k[:1], 6, axis=0)
    assert np.allclose(om.attention(q, kk, v), np.repeat(v.mean(axis=0)[[0, 0, 1, 1]][None], 3, axis=0))


def test_rope_rotation_properties():
    g = np.random.default_rng(1)
    x = g.standard_normal((5, 2, 16))
    pos = np.array([0, 1, 7, 100, 33000])
    r = om.rope(x, pos, 10000.0)
    assert np.allclose(r[0], x[0])
    assert np.allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(x, axis=-1))
    # relative position: <R_m q, R_n k> depends on m - n only
    q, k = x[:1], x[1:2]
    a = (om.rope(q, [10], 1e4) * om.rope(k, [3], 1e4)).sum()
    b = (om.rope(q, [1010], 1e4) * om.rope(k, [1003], 1e4)).sum()
    assert abs(a - b) < 1e-9


def test_rmsnorm_unit_rms():
    x = np.random.default_rng(2).standard_normal((4, 64)) * 7
    y = om.rmsnorm(x, 0.0)
    assert np.allclose(np.sqrt((y * y).mean(axis=1)), 1.0)


def test_router_topk_weights_sum_to_one_and_ties():
    g = np.random.default_rng(3)
    x = g.standard_normal((50, 16))
    wr = g.standard_normal((12, 16))
    ids, w = om.router(x, wr, 8)
    assert np.allclose(w.sum(axis=1), 1.0)
    r = x @ wr.T
    for t in range(50):
        assert list(ids[t]) == list(np.argsort(-r[t], kind="stable")[:8])
        assert np.all(np.diff(w[t]) <= 1e-15)
    # all-equal logits: ties go to the lower ids, equal weights
    ids, w = om.router(np.zeros((2, 16)), wr, 3)
    assert ids.tolist() == [[0, 1, 2]] * 2 and np.allclose(w, 1 / 3)
    # Zipf bias alone: experts 0..k-1, weights proportional to (e+1)^-s
    ids, w = om.router(np.zeros((1, 16)), wr, 4, zipf_s=1.1)
    ref = np.arange(1, 5) ** -1.1
    assert ids.tolist() == [[0, 1, 2, 3]] and np.allclose(w[0], ref / ref.sum())


def test_moe_all_experts_equal_gates_is_mean(micro):
    cfg, model, _ = micro
    layer = model.layers[0]
    x = np.random.default_rng(4).standard_normal((5, cfg.d_model))
    zero = om.Layer(**{**layer.__dict__, "wr": np.zeros_like(layer.wr)})
    model.cfg = cfg.replace(top_k=cfg.n_experts)
    y, ids, w = om.moe(model, zero, x)
    model.cfg = cfg
    ref = np.zeros_like(x)
    for e in range(cfg.n_experts):
        a = model.store(om.silu(x @ layer.wg[e].T.astype(np.float64)) * (x @ layer.wu[e].T.astype(np.float64)))
        ref += a @ layer.wd[e].T.astype(np.float64)
    assert np.allclose(y, ref / cfg.n_experts)


def test_low_entropy_canvas_stops_at_first_round(micro):
    # a huge logit scale makes every row one-hot: entropy ~0 -> all commit -> stop
    cfg, model, _ = micro
    model.cfg = cfg.replace(logit_scale=1e5)
    K, V = I.prompt_kv(2, cfg.n_layers, 1, cfg.n_kv_heads, 4, cfg.head_dim, bf16=False)
    r = om.generate_block(model, K[:, 0], V[:, 0])
    model.cfg = cfg
    assert r["steps_used"] == 1 and r["n_committed"] == 256
    assert np.array_equal(r["canvas"], r["trace"][0]["amax"])


def test_generate_runs_to_budget_when_uncertain(micro):
    cfg, model, _ = micro
    K, V = I.prompt_kv(2, cfg.n_layers, 1, cfg.n_kv_heads, 4, cfg.head_dim, bf16=False)
    r = om.generate_block(model, K[:, 0], V[:, 0])
    assert r["steps_used"] == cfg.max_steps
    assert np.array_equal(r["canvas"], r["trace"][-1]["tokens"])
    # round 0 used the uniform-noise canvas; later rounds the re-noised one
    t0 = r["trace"][0]
    assert np.array_equal(r["trace"][1]["canvas_next"].shape, (256,))
    assert np.array_equal(t0["canvas_next"][t0["commit"] == 1], t0["tokens"][t0["commit"] == 1])


def test_zero_selfcond_equals_none(micro):
    cfg, model, _ = micro
    K, V = I.prompt_kv(2, cfg.n_layers, 1, cfg.n_kv_heads, 4, cfg.head_dim, bf16=False)
    c = I.canvas_ids(9, 1, cfg.vocab)[0]
    a, _ = om.forward_canvas(model, K[:, 0], V[:, 0], c, None)
    b, _ = om.forward_canvas(model, K[:, 0], V[:, 0], c, np.zeros((256, cfg.d_model)))
    assert np.array_equal(a, b)


def test_bf16_storage_rounds_values(micro):
    cfg, _, _ = micro
    m = om.Model(cfg.replace(dtype=I.DTYPE_BF16), layers=1)
    w = m.layers[0].wg
    assert np.array_equal(w.view(np.uint32) & np.uint32(0xFFFF), np.zeros_like(w.view(np.uint32)))
    # bf16 spacing at 1 is 2^-7; exact ties go to the even mantissa
    x = np.array([1.0 + 2 ** -9, 1.0 + 3 * 2 ** -9, -3.14159, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8])
    assert np.array_equal(m.store(x), [1.0, 1.0 + 2 ** -7, -3.140625, 1.0, 1.0 + 2 ** -6])


def test_routing_alternatives_pins():
    g = np.random.default_rng(7)
    r = g.standard_normal(16)
    alts = om.routing_alternatives(r, 4, 1e-9)
    assert len(alts) == 1
    prim_ids, prim_w = alts[0]
    assert list(prim_ids) == list(np.argsort(-r, kind="stable")[:4]) and np.isclose(prim_w.sum(), 1.0)
    # construct a near tie at the boundary: 4th and 5th largest 1e-4 apart
    s = np.argsort(-r, kind="stable")
    r2 = r.copy()
    r2[s[4]] = r2[s[3]] - 1e-4
    alts = om.routing_alternatives(r2, 4, 1e-3)
    assert len(alts) == 2
    assert set(alts[1][0]) == (set(s[:3]) | {s[4]})
    assert np.isclose(alts[1][1].sum(), 1.0)


def test_token_logits_with_routing_reproduces_forward(micro):
    cfg, model, _ = micro
    one = om.Model.__new__(om.Model)
    one.cfg, one.embed, one.wsc, one.layers = cfg.replace(n_layers=1), model.embed, model.wsc, model.layers[:1]
    K, V = I.prompt_kv(4, 1, 1, cfg.n_kv_heads, 6, cfg.head_dim, bf16=False)
    c = I.canvas_ids(5, 1, cfg.vocab)[0]
    trace = []
    logits, _ = om.forward_canvas(one, K[:, 0], V[:, 0], c, None, trace=trace)
    for t in (0, 17, 255):
        ids, w = om.routing_alternatives(trace[0]["router"][t], cfg.top_k, 1e-12)[0]
        row = om.token_logits_with_routing(one, one.layers[0], trace[0]["h_attn"][t], ids, w)
        assert np.allclose(row, logits[t], rtol=1e-12, atol=1e-12)
        assert list(ids) == list(trace[0]["ids"][t])


# --- block-autoregressive continuation ------------------------------------------------------
def test_causal_encode_is_prefix_consistent():
    # a finished canvas joins the context by a causal encode: the cache of the
    # prompt part must not change when tokens are appended after it
    w = I.TINY_FP32.replace(n_layers=1, max_steps=2)
    m = om.Model(w)
    prompt = I.prompt_ids(w.sample_seed, 1, 24, w.vocab)[0]
    extra = I.prompt_ids(w.sample_seed + 1, 1, 40, w.vocab)[0]
    K0, V0 = om.encode_prompt(m, prompt)
    K1, V1 = om.encode_prompt(m, np.concatenate([prompt, extra]))
    assert np.array_equal(K1[:, :, :24], K0) and np.array_equal(V1[:, :, :24], V0)


def test_generate_chains_blocks_on_the_growing_context():
    w = I.TINY_FP32.replace(n_layers=1, max_steps=2)
    m = om.Model(w)
    prompt = I.prompt_ids(w.sample_seed, 1, 16, w.vocab)[0]
    blocks = om.generate(m, prompt, 2)
    # block 0 is exactly the single-block generation on the prompt
    K, V = om.encode_prompt(m, prompt)
    b0 = om.generate_block(m, K, V)
    assert np.array_equal(blocks[0]["canvas"], b0["canvas"]) and blocks[0]["steps_used"] == b0["steps_used"]
    # block 1 runs on [prompt ; block 0] with seed + 1
    K1, V1 = om.encode_prompt(m, np.concatenate([prompt, b0["canvas"]]))
    assert K1.shape[2] == 16 + 256
    import copy
    m1 = copy.copy(m)
    m1.cfg = w.replace(sample_seed=w.sample_seed + 1)
    b1 = om.generate_block(m1, K1, V1)
    assert np.array_equal(blocks[1]["canvas"], b1["canvas"])
    # the two blocks start from different noise
    assert not np.array_equal(sp.initial_canvas(w.sample_seed, 0, 256, w.vocab),
                              sp.initial_canvas(w.sample_seed + 1, 0, 256, w.vocab))


def test_route_bias_steers_selection_and_keeps_gate_softmax():
    # per-token router bias (routing-locality workloads): with a bias far above
    # the logit spread each token selects exactly its preferred experts; the
    # gates stay the softmax over the selected logits, which a constant shift
    # of the selected set leaves unchanged; the rows used are the canvas's own
    w = I.TINY_FP32.replace(n_layers=2)
    model = om.Model(w)
    E, k = w.n_experts, w.top_k
    pool = 4
    rb = I.routing_bias(5, w.n_layers, 2 * 256, E, k, pool, beta=1000.0)
    model.route_bias = rb
    K, V = om.encode_prompt(model, I.prompt_ids(w.sample_seed, 1, 16, w.vocab)[0])
    canvas = I.canvas_ids(9, 1, w.vocab)[0]
    for cid in (0, 1):
        trace = []
        om.forward_canvas(model, K, V, canvas, None, trace=trace, canvas_id=cid)
        for l in range(w.n_layers):
            ids = trace[l]["ids"]
            pref = rb[l, cid * 256:(cid + 1) * 256] > 0
            for t in range(256):
                assert set(ids[t].tolist()) == set(np.nonzero(pref[t])[0].tolist()), (cid, l, t)
            assert len(np.unique(ids)) == pool
            # gates (router on the biased logits r, identity weights) equal the
            # softmax of the unbiased logits over the selected experts
            r = trace[l]["router"]
            for t in (0, 100, 255):
                sel_ids, gates = om.router(r[t:t + 1], np.eye(E), k)
                base = r[t, sel_ids[0]] - rb[l, cid * 256 + t, sel_ids[0]]
                ex = np.exp(base - base.max())
                assert np.allclose(gates[0], ex / ex.sum(), rtol=1e-12)


def test_zero_route_bias_is_no_bias():
    w = I.TINY_FP32.replace(n_layers=1)
    model = om.Model(w)
    K, V = om.encode_prompt(model, I.prompt_ids(w.sample_seed, 1, 16, w.vocab)[0])
    canvas = I.canvas_ids(9, 1, w.vocab)[0]
    ref, _ = om.forward_canvas(model, K, V, canvas, None)
    model.route_bias = np.zeros((1, 256, w.n_experts), dtype=np.float32)
    got, _ = om.forward_canvas(model, K, V, canvas, None)
    assert np.array_equal(ref, got)


def test_topk_self_condition_is_dense_self_condition_of_the_sparse_distribution():
    # p E with p zero outside the candidates equals the weighted sum of the
    # candidates' embedding rows
    for w in (I.TINY_FP32.replace(n_layers=1), I.TINY_FP32.replace(n_layers=1, dtype=I.DTYPE_BF16)):
        model = om.Model(w)
        g = np.random.default_rng(3)
        K = 7
        ids = np.stack([g.choice(w.vocab, size=K, replace=False) for _ in range(256)]).astype(np.int32)
        wt = g.dirichlet(np.ones(K), size=256).astype(F32)
        dense = np.zeros((256, w.vocab), F32)
        dense[np.arange(256)[:, None], ids] = wt
        a = om.self_condition_topk(model, ids, wt)
        b = om.self_condition(model, dense)
        assert np.allclose(a, b, rtol=1e-6, atol=1e-9)


def test_router_bias_closed_form_with_zero_input():
    # x = 0: the logits are the bias alone, so the selection is the top-k of
    # the bias and the gates its softmax over the selected experts -- a bias
    # that reached only the selection (not the gates) gives equal gates
    E, k = 8, 2
    x = np.zeros((3, 16))
    wr = np.random.default_rng(0).standard_normal((E, 16))
    b = np.array([[0, 0, 3, 1, 0, 0, 0, 0], [2, 0, 0, 0, 0, 0, 0, 2], [0, -1, 0, 5, 4, 0, 0, 0]], dtype=np.float64)
    ids, gates = om.router(x, wr, k, extra=b)
    assert ids.tolist() == [[2, 3], [0, 7], [3, 4]]
    expect = [1 / (1 + math.exp(-2.0)), 0.5, 1 / (1 + math.exp(-1.0))]
    assert np.allclose(gates[:, 0], expect, rtol=1e-14) and np.allclose(gates.sum(axis=1), 1.0)


def test_lazy_expert_weights_equal_the_whole_tensor():
    # per-expert generation (used for single-layer checks of the large
    # workloads) is the same counter range of the same generator
    for w in (I.TINY_FP32, I.MID_BF16.replace(n_layers=1)):
        eager = om.layer_weights(w, 0)
        lazy = om.layer_weights(w, 0, lazy_experts=True)
        for name in ("wg", "wu", "wd"):
            full = getattr(eager, name)
            for e in (0, w.n_experts // 2, w.n_experts - 1):
                assert np.array_equal(lazy.__dict__[name][e].view(np.uint32), full[e].view(np.uint32)), (name, e)
