"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin
catches each one: a dropped term, a wrong sign, a transposed or misplaced
operand, an off-by-one in a rule.  Every planted mistake must make its pin
fail; the unmodified oracle passes the same pins (tests/test_oracle_*.py)."""
import math

import numpy as np
import pytest

from block_text_diffusion_b200 import inputs as I
from oracle import model as om, sampler as sp

import test_oracle_model as tm

F32 = np.float32


@pytest.fixture(scope="module")
def micro():
    cfg = tm.MICRO
    return cfg, om.Model(cfg), tm.BruteWeights(cfg)


def forward_matches_brute(cfg, model, W):
    prompt = I.prompt_ids(1, 1, cfg.prompt_len, cfg.vocab)[0]
    K, V = om.encode_prompt(model, prompt)
    bK, bV = tm.bf_encode(cfg, W, prompt)
    if not (np.allclose(K, np.array(bK).transpose(0, 2, 1, 3), rtol=1e-6, atol=1e-7)
            and np.allclose(V, np.array(bV).transpose(0, 2, 1, 3), rtol=1e-6, atol=1e-7)):
        return False
    canvas = I.canvas_ids(2, 1, cfg.vocab)[0]
    sc = I.normal(3, 7, (256, cfg.d_model), std=0.05)
    logits, _ = om.forward_canvas(model, K, V, canvas, sc)
    ref = tm.bf_logits(cfg, W, tm._cache_to_lists(K), tm._cache_to_lists(V), canvas, sc.tolist())
    return bool(np.allclose(logits, ref, rtol=1e-5, atol=1e-6))


def _rope_sign(x, positions, theta):
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-2.0 * np.arange(half) / hd)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c + b * s, -a * s + b * c], axis=-1)      # rotates the wrong way


def _attn_noscale(q, k, v, causal_offset=None):
    return om.attention.__wrapped__(q * math.sqrt(q.shape[-1]), k, v, causal_offset)


def _block_no_residual(model, layer, h, positions, kp, vp, causal):
    out, k, v = _ORIG_BLOCK(model, layer, h, positions, kp, vp, causal)
    return out - h, k, v


_ORIG_BLOCK = om.block


@pytest.mark.parametrize("name", ["rope_sign", "attention_scale", "residual", "moe_slot_weights",
                                  "rmsnorm_eps_inside", "logit_scale"])
def test_forward_mistakes_are_caught(micro, monkeypatch, name):
    cfg, model, W = micro
    if name == "rope_sign":
        monkeypatch.setattr(om, "rope", _rope_sign)
    elif name == "attention_scale":
        orig = om.attention
        monkeypatch.setattr(om, "attention",
                            lambda q, k, v, causal_offset=None: orig(q * math.sqrt(q.shape[-1]), k, v, causal_offset))
    elif name == "residual":
        monkeypatch.setattr(om, "block", _block_no_residual)
    elif name == "moe_slot_weights":
        orig = om.router
        monkeypatch.setattr(om, "router", lambda x, wr, k, z=0.0, extra=None: (orig(x, wr, k, z, extra)[0], orig(x, wr, k, z, extra)[1][:, ::-1]))
    elif name == "rmsnorm_eps_inside":
        monkeypatch.setattr(om, "rmsnorm", lambda h, eps: h / (np.sqrt(np.mean(h * h, -1, keepdims=True)) + 1e-2))
    elif name == "logit_scale":
        monkeypatch.setattr(model, "cfg", cfg.replace(logit_scale=1.0))
    assert not forward_matches_brute(cfg, model, W)


def test_selfcond_without_wsc_is_caught(micro, monkeypatch):
    cfg, model, W = micro
    p = np.abs(I.normal(4, 8, (256, cfg.vocab)))
    p = (p / p.sum(axis=1, keepdims=True)).astype(F32)
    monkeypatch.setattr(om, "_proj", lambda x, w: x)
    s = om.self_condition(model, p)
    d = cfg.d_model
    u = [tm.r32(sum(float(p[0, v]) * W(om.T_EMBED, (v, i), (cfg.vocab, d)) for v in range(cfg.vocab)))
         for i in range(d)]
    ref = [tm.r32(sum(W(om.T_WSC, (o, i), (d, d)) * u[i] for i in range(d))) for o in range(d)]
    assert not np.allclose(s[0], ref, rtol=1e-6, atol=1e-9)


def test_entropy_sign_mistake_is_caught(monkeypatch):
    V, k, a = 4096, 7, -2.5
    l = np.zeros((1, V), F32)
    l[0, :k] = a
    Z = k * math.exp(a) + V - k
    H = math.log(Z) - k * a * math.exp(a) / Z
    orig = sp.nm.log_f32
    # ln S + U/S instead of ln S - U/S
    st = sp.row_stats(l)
    wrong = float(orig(np.float32(st["S_q"][0] * 2.0 ** -40))) + float(st["U_q"][0]) / float(st["S_q"][0])
    assert abs(wrong - H) > 100 * 3e-6      # far outside the closed-form pin's tolerance
    assert abs(float(st["H"][0]) - H) < 3e-6


def test_gumbel_sign_mistake_is_caught(monkeypatch):
    from scipy import stats
    V = 8
    l = np.array([0.0, 1.0, -1.0, 0.5, 2.0, -3.0, 0.25, 1.5], F32)
    T = F32(0.7)
    inv_t = F32(1.0) / T
    monkeypatch.setattr(sp, "gumbel_noise", lambda *a: -_GUMBEL(*a))
    counts = np.zeros(V)
    for s in range(20):
        counts += np.bincount(sp.sample_tokens(np.broadcast_to(l, (256, V)), inv_t, 42, 3, s), minlength=V)
    lt = l.astype(np.float64) / float(T)
    p = np.exp(lt - lt.max())
    p /= p.sum()
    assert stats.chisquare(counts, p * counts.sum()).pvalue < 1e-6


_GUMBEL = sp.gumbel_noise


def test_temperature_endpoint_mistake_is_caught():
    wrong = lambda t: sp.temperature(1 - t)       # schedule reversed
    assert wrong(sp.schedule_t(0, 48)) != F32(0.8)


def test_eb_commit_off_by_one_is_caught():
    # committing the position that crosses the bound
    H = np.array([0.03, 0.04, 0.05, 0.2, 0.3, 1.0, 2.0, 0.01], F32)
    hq = sp.fixed_entropy(H)
    lim = sp.bound_fixed(0.1)
    order = sorted(range(8), key=lambda i: (int(hq[i]), i))
    acc, wrong = 0, np.zeros(8, np.uint8)
    for i in order:
        wrong[i] = 1
        acc += int(hq[i])
        if acc > lim:
            break
    n_star = max(tm_brute(hq, lim), 1)
    assert wrong.sum() != n_star
    assert sp.commit_mask(H, 1, 0.1).sum() == n_star


def tm_brute(h, lim):
    import test_oracle_sampler as ts
    return ts._eb_brute(h, lim)


def test_nonstrict_stop_is_caught():
    at = np.full(256, 0.1, F32)
    none = np.zeros(256, np.uint8)
    a = np.arange(256, dtype=np.int32)
    hq = sp.fixed_entropy(at)
    wrong = int(hq.sum()) <= 256 * sp.bound_fixed(0.1)
    assert wrong != sp.stop_decision(at, none, a, None, 1, 48, 0, 0.1)

def test_route_bias_missing_from_gates_is_caught(monkeypatch):
    # a router that selects with the per-token bias but forms the gates
    # without it: the zero-input closed form fails
    import test_oracle_model as tm
    orig_logits = om.router_logits

    def wrong_router(x, wr, top_k, zipf_s=0.0, extra=None):
        r = orig_logits(x, wr, zipf_s, extra)
        r0 = orig_logits(x, wr, zipf_s, None)
        ids = np.array([sorted(range(r.shape[1]), key=lambda e: (-r[t, e], e))[:top_k] for t in range(r.shape[0])],
                       dtype=np.int32)
        sel = np.take_along_axis(r0, ids, axis=1)
        ex = np.exp(sel - sel.max(axis=1, keepdims=True))
        return ids, ex / ex.sum(axis=1, keepdims=True)

    monkeypatch.setattr(om, "router", wrong_router)
    with pytest.raises(AssertionError):
        tm.test_router_bias_closed_form_with_zero_input()


def test_topk_ties_to_the_higher_index_are_caught(monkeypatch):
    import test_oracle_sampler as ts
    monkeypatch.setattr(sp, "topk_ids", lambda l, K: np.lexsort((-np.arange(np.asarray(l).size),
                                                                 -np.asarray(l, np.float64)))[:K].astype(np.int32))
    with pytest.raises(AssertionError):
        ts.test_topk_ids_brute_force("ties")
