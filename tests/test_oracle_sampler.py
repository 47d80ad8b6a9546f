"""Pins of the sampler oracle: entropy closed forms, temperature endpoints,
Gumbel-max distribution, commit rule brute force, stop rule (CPU only)."""
import itertools
import math

import numpy as np
import pytest
from scipy import stats

from block_text_diffusion_b200 import inputs as I
from oracle import _native, sampler as sp

F32 = np.float32


@pytest.mark.parametrize("V", [1024, 32768, 262144])
def test_entropy_of_uniform_logits_is_log_v(V):
    l = np.full((2, V), 0.37, dtype=F32)
    st = sp.row_stats(l) if V <= 32768 else _native.sampler_rows(l, 0, 0, 0, 0, F32(1.25), False)
    assert np.allclose(st["H"], math.log(V), rtol=0, atol=2e-6)
    assert np.allclose(sp.entropy_f64(l), math.log(V), atol=1e-12)


def test_entropy_closed_form_two_levels():
    # k entries at a, V-k at 0: Z = k e^a + V - k, H = ln Z - k a e^a / Z
    V = 4096
    for k, a in [(1, 3.0), (7, -2.5), (100, 0.75), (1, 30.0)]:
        l = np.zeros((1, V), F32)
        l[0, :k] = a
        Z = k * math.exp(a) + V - k
        H = math.log(Z) - k * a * math.exp(a) / Z
        assert abs(sp.entropy_f64(l)[0] - H) < 1e-12
        assert abs(float(sp.row_stats(l)["H"][0]) - H) < 3e-6


def test_entropy_one_hot_is_zero():
    l = I.logits(5, 4, 2048, "normal", 1.0)
    l[:, 17] += 120.0
    st = sp.row_stats(l)
    assert np.all(np.abs(st["H"]) < 1e-6)
    assert np.all(st["amax"] == 17)


@pytest.mark.parametrize("kind,scale", [("normal", 1.0), ("normal", 4.0), ("peaked", 1.0),
                                        ("mixed", 2.0), ("ties", 1.0)])
def test_decision_entropy_matches_definition(kind, scale):
    l = I.logits(9, 16, 8192, kind, scale)
    st = sp.row_stats(l, want_probs=True)
    ref = sp.entropy_f64(l)
    assert np.all(np.abs(st["H"] - ref) <= 4e-6 + 2e-6 * ref)
    # probabilities: p = softmax(l) within binary32 rounding, rows sum to 1
    p64 = np.exp(l.astype(np.float64) - l.max(axis=1, keepdims=True))
    p64 /= p64.sum(axis=1, keepdims=True)
    assert np.abs(st["p"] - p64).max() < 1e-6
    assert np.allclose(st["p"].astype(np.float64).sum(axis=1), 1.0, atol=1e-5)
    assert np.array_equal(st["amax"], l.argmax(axis=1))


def test_temperature_endpoints_and_linearity():
    assert sp.temperature(sp.schedule_t(0, 48)) == F32(0.8)
    assert sp.temperature(sp.schedule_t(47, 48)) == F32(0.4)
    assert sp.temperature(sp.schedule_t(0, 1)) == F32(0.8)
    Ts = [float(sp.temperature(sp.schedule_t(s, 48))) for s in range(48)]
    assert all(a > b for a, b in zip(Ts, Ts[1:]))
    # linear: constant decrement of 0.4/47 up to binary32 rounding
    d = np.diff(Ts)
    assert np.allclose(d, -0.4 / 47, atol=2e-7)
    assert abs(float(sp.temperature(F32(0.5))) - 0.6) < 1e-7


def test_gumbel_max_frequencies_match_softmax():
    # Gumbel-max draws from softmax(l/T); vary the (position, step) counter
    V = 8
    l = np.array([0.0, 1.0, -1.0, 0.5, 2.0, -3.0, 0.25, 1.5], F32)
    T = F32(0.7)
    inv_t = F32(1.0) / T
    n_pos, n_step = 512, 60
    counts = np.zeros(V)
    for s in range(n_step):
        rows = np.broadcast_to(l, (n_pos, V))
        toks = _native.sampler_rows(rows, 42, 3, 0, s, inv_t, False)["tokens"] if _native.lib() \
            else sp.sample_tokens(rows, inv_t, 42, 3, s)
        counts += np.bincount(toks, minlength=V)
    lt = l.astype(np.float64) / float(T)
    p = np.exp(lt - lt.max())
    p /= p.sum()
    assert stats.chisquare(counts, p * counts.sum()).pvalue > 1e-4


def test_gumbel_low_temperature_is_argmax():
    l = I.logits(3, 6, 512, "normal", 1.0)
    inv_t = F32(1e6)
    toks = sp.sample_tokens(l, inv_t, 1, 0, 0)
    assert np.array_equal(toks, l.argmax(axis=1))


def test_c_twin_sampler_bit_equal():
    if _native.lib() is None:
        pytest.skip("no C compiler")
    l = I.logits(4, 12, 4096, "mixed", 3.0)
    inv_t = F32(1.0) / F32(0.55)
    r = _native.sampler_rows(l, 99, 2, 0, 7, inv_t, True)
    st = sp.row_stats(l, want_probs=True)
    for k in ("H", "S_q", "U_q", "amax", "p"):
        assert np.array_equal(r[k], st[k]), k
    assert np.array_equal(r["tokens"], sp.sample_tokens(l, inv_t, 99, 2, 7))


def test_renoise_uniform():
    V = 16
    toks = np.concatenate([sp.renoise_tokens(5, 0, s, 256, V) for s in range(200)])
    cnt = np.bincount(toks, minlength=V)
    assert stats.chisquare(cnt).pvalue > 1e-4
    assert not np.array_equal(sp.renoise_tokens(5, 0, 1, 256, V), sp.renoise_tokens(5, 0, 2, 256, V))
    assert not np.array_equal(sp.initial_canvas(5, 0, 256, 1000), sp.renoise_tokens(5, 0, 0, 256, 1000))


def test_commit_threshold_rule():
    H = I.entropies(1, 1)[0]
    m = sp.commit_mask(H, 0, 0.5)
    assert np.array_equal(m.astype(bool), H < F32(0.5))


def _eb_brute(h_fixed, lim):
    """Largest committable count over all subsets, n* = max{|S|: sum_S h <= lim}."""
    n = len(h_fixed)
    best = 0
    for mask in range(1 << n):
        idx = [i for i in range(n) if mask >> i & 1]
        if sum(int(h_fixed[i]) for i in idx) <= lim:
            best = max(best, len(idx))
    return best


@pytest.mark.parametrize("seed", range(12))
def test_entropy_bounded_commit_matches_brute_force(seed):
    g = np.random.default_rng(seed)
    H = g.choice([0.0, 0.01, 0.02, 0.03, 0.05, 0.08, 0.2, 1.0], size=8).astype(F32)
    if seed % 3 == 0:
        H[:] = g.uniform(0.0, 0.05, size=8).astype(F32)
    mask = sp.commit_mask(H, 1, 0.1)
    hq = sp.fixed_entropy(H)
    lim = sp.bound_fixed(0.1)
    n_star = max(_eb_brute(hq, lim), 1)
    assert mask.sum() == n_star
    # committed ones are the most certain (ties broken by lower position)
    com = [(int(hq[i]), i) for i in range(8) if mask[i]]
    unc = [(int(hq[i]), i) for i in range(8) if not mask[i]]
    if com and unc:
        assert max(com) < min(unc)


def test_entropy_bounded_commits_at_least_one():
    H = np.full(256, 3.0, F32)
    H[77] = 2.0
    m = sp.commit_mask(H, 1, 0.1)
    assert m.sum() == 1 and m[77] == 1


def test_stop_rules():
    low = np.full(256, 0.05, F32)
    high = np.full(256, 5.0, F32)
    none = np.zeros(256, np.uint8)
    allm = np.ones(256, np.uint8)
    a = np.arange(256, dtype=np.int32)
    # mean mode: a canvas whose entropy sits below the bound stops
    assert sp.stop_decision(low, none, a, None, 0, 48, 0, 0.1)
    assert not sp.stop_decision(high, none, a, None, 3, 48, 0, 0.1)
    assert sp.stop_decision(high, allm, a, None, 3, 48, 0, 0.1)
    # the last round always stops
    assert sp.stop_decision(high, none, a, None, 47, 48, 0, 0.1)
    # EB mode: low mean entropy AND unchanged argmax, never at round 0
    tiny = np.full(256, 0.001, F32)
    assert not sp.stop_decision(tiny, allm, a, None, 0, 48, 1, 0.005)
    assert sp.stop_decision(tiny, allm, a, a.copy(), 5, 48, 1, 0.005)
    b = a.copy(); b[3] += 1
    assert not sp.stop_decision(tiny, allm, a, b, 5, 48, 1, 0.005)
    assert not sp.stop_decision(np.full(256, 0.006, F32), allm, a, a, 5, 48, 1, 0.005)
    # boundary: mean exactly at the bound does not stop (strict)
    at = np.full(256, 0.1, F32)
    assert not sp.stop_decision(at, none, a, None, 1, 48, 0, 0.1)


def test_next_canvas_keeps_committed_renoises_rest():
    tok = np.arange(256, dtype=np.int32) + 1000
    mask = (np.arange(256) % 3 == 0).astype(np.uint8)
    nxt = sp.next_canvas(tok, mask, 8, 1, 4, 5000)
    fresh = sp.renoise_tokens(8, 1, 4, 256, 5000)
    assert np.array_equal(nxt[mask == 1], tok[mask == 1])
    assert np.array_equal(nxt[mask == 0], fresh[mask == 0])


# --- top-k-truncated sampling ---------------------------------------------------------
@pytest.mark.parametrize("kind", ["normal", "ties", "flat", "peaked"])
def test_topk_ids_brute_force(kind):
    l = I.logits(11, 6, 64, kind, 2.0)
    for K in (1, 5, 17, 64, 100):
        for r in range(l.shape[0]):
            ref = sorted(range(64), key=lambda v: (-float(l[r, v]), v))[:K]
            assert sp.topk_ids(l[r], K).tolist() == ref


def test_topk_at_full_vocab_is_the_exact_sampler():
    for kind in ("normal", "ties", "flat", "mixed"):
        l = I.logits(12, 8, 512, kind, 3.0)
        inv_t = F32(1.0) / F32(0.65)
        for r in range(l.shape[0]):
            tok, _, _ = sp.topk_sample(l[r], 512, inv_t, 5, 1, r, 7)
            assert tok == sp.gumbel_argmax(l[r], inv_t, 5, 1, r, 7)


def test_topk_token_equals_exact_when_exact_winner_is_a_candidate():
    # Gumbel-max over a subset that holds the overall winner picks that winner;
    # otherwise the draw is still one of the candidates
    l = I.logits(13, 64, 2048, "normal", 1.0)
    inv_t = F32(1.0) / F32(0.8)
    hits = 0
    for r in range(l.shape[0]):
        exact = sp.gumbel_argmax(l[r], inv_t, 9, 0, r, 2)
        for K in (4, 32):
            tok, ids, _ = sp.topk_sample(l[r], K, inv_t, 9, 0, r, 2)
            assert tok in ids.tolist()
            if exact in ids.tolist():
                assert tok == exact
                hits += 1
    assert hits > 0


def test_topk_frequencies_match_truncated_softmax():
    # the truncated draw is softmax(l/T) renormalised over the K largest logits
    V, K = 8, 3
    l = np.array([0.0, 1.0, -1.0, 0.5, 2.0, -3.0, 0.25, 1.5], F32)
    T = F32(0.7)
    inv_t = F32(1.0) / T
    counts = np.zeros(V)
    for s in range(40):
        for pos in range(256):
            counts[sp.topk_sample(l, K, inv_t, 42, 3, pos, s)[0]] += 1
    ids = [4, 7, 1]
    assert counts.sum() == counts[ids].sum()
    lt = l[ids].astype(np.float64) / float(T)
    p = np.exp(lt - lt.max())
    p /= p.sum()
    assert stats.chisquare(counts[ids], p * counts.sum()).pvalue > 1e-4


def test_topk_weights_are_the_renormalised_untempered_softmax():
    l = I.logits(14, 5, 4096, "mixed", 4.0)
    for r in range(l.shape[0]):
        _, ids, w = sp.topk_sample(l[r], 50, F32(2.0), 1, 0, r, 0)
        x = l[r, ids].astype(np.float64)
        ref = np.exp(x - x.max())
        ref /= ref.sum()
        assert np.allclose(w, ref, rtol=2e-6, atol=1e-12)
        assert abs(float(w.astype(np.float64).sum()) - 1.0) < 50 * 2 ** -23
