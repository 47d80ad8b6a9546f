"""Step-level parity of the CUDA path against the oracle (B200 only).

Tolerances.  fp32 workload: logits and entropy within 1e-4 relative, tokens
and commit masks identical wherever the oracle's decision is not within
rounding of a tie, >= 99% agreement overall, full block runs agree on >= 99%
of tokens.  bf16 workloads: the LM head within 2e-2 absolute given the same
final normalised state; upstream of it, the deviation from the oracle must
stay within twice that of an oracle whose bf16 storage rounds one value in
64 to the other neighbour (see storage_noise.py for why no fixed absolute
bound can hold there); tokens identical wherever the Gumbel-max margin
exceeds twice the row's logit error."""
import copy

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_text_diffusion_b200 as dg  # noqa: E402
from block_text_diffusion_b200 import inputs as I  # noqa: E402
from oracle import model as om, sampler as sp, numerics as nm  # noqa: E402
from storage_noise import NoisyStore, quantiles, rms_ulps  # noqa: E402

F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dg.lib()


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch.cuda.synchronize()
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def read_kv(model, kv, B, P):
    """Decode the library's cache layout: K [L][B][Hkv][S][hd], V^T [L][B][Hkv][hd][S]."""
    w = model.w
    S = ((P + 256 + 63) // 64) * 64
    esz = 2 if w.dtype == I.DTYPE_BF16 else 4
    n = w.n_layers * B * w.n_kv_heads * S * w.head_dim
    raw = kv[: 2 * n * esz].view(torch.bfloat16 if esz == 2 else torch.float32)
    K = raw[:n].view(w.n_layers, B, w.n_kv_heads, S, w.head_dim)
    Vt = raw[n:].view(w.n_layers, B, w.n_kv_heads, w.head_dim, S)
    return host(K), host(Vt).transpose(0, 1, 2, 4, 3)


def step_buffers(w, B):
    dt = torch.bfloat16 if w.dtype == I.DTYPE_BF16 else torch.float32
    z = lambda shape, t: torch.zeros(shape, dtype=t, device="cuda")
    return dict(logits=z((B, 256, w.vocab), torch.float32), entropy=z((B, 256), torch.float32),
                tokens=z((B, 256), torch.int32), argmax=z((B, 256), torch.int32), commit=z((B, 256), torch.uint8),
                canvas_next=z((B, 256), torch.int32), selfcond_next=z((B, 256, w.d_model), dt),
                stop=z(B, torch.int32), n_committed=z(B, torch.int32))


def gumbel_margin(l32, inv_t, seed, canvas_id, step):
    """Gap between the best and second-best Gumbel key per row (oracle side)."""
    out = np.empty(l32.shape[0])
    for i in range(l32.shape[0]):
        g = sp.gumbel_noise(seed, canvas_id, i, step, l32.shape[1])
        key = np.sort(l32[i].astype(np.float64) * float(inv_t) + g)
        out[i] = key[-1] - key[-2]
    return out


def gumbel_margin_topk(l32, K, inv_t, seed, canvas_id, step):
    """Top-k-truncated draws: gap between the best and second-best key among
    the K candidates, capped by the gap between the K-th and (K+1)-th logit
    (scaled to key units) since a candidate set that rounding can change may
    change the draw."""
    out = np.empty(l32.shape[0])
    for i in range(l32.shape[0]):
        ids = sp.topk_ids(l32[i], K + 1)
        key = np.sort(l32[i, ids[:K]].astype(np.float64) * float(inv_t)
                      + sp.gumbel_noise_at(ids[:K], seed, canvas_id, i, step))
        gap = key[-1] - key[-2] if K > 1 else np.inf
        edge = (float(l32[i, ids[K - 1]]) - float(l32[i, ids[K]])) * float(inv_t) if K < l32.shape[1] else np.inf
        out[i] = min(gap, edge)
    return out


def check_logits(got, ref, fp32):
    if fp32:
        scale = np.maximum(np.abs(ref), np.sqrt((ref ** 2).mean(axis=-1, keepdims=True)))
        assert np.all(np.abs(got - ref) <= 1e-4 * scale), np.abs(got - ref).max()
    else:
        assert np.abs(got - ref).max() <= 2e-2, np.abs(got - ref).max()


def compare_round(r_gpu, r_ora, w, step, t, fp32, canvas_id=0, topk=0):
    check_logits(r_gpu["logits"], r_ora["logits64"], fp32)
    H_tol = 1e-4 * np.maximum(1.0, np.abs(r_ora["H"])) if fp32 else 2e-2
    assert np.all(np.abs(r_gpu["entropy"] - r_ora["H"]) <= H_tol)
    inv_t = F32(1.0) / sp.temperature(F32(t), w.temp_start, w.temp_end)
    margin = (gumbel_margin_topk(r_ora["logits"], topk, inv_t, w.sample_seed, canvas_id, step) if topk
              else gumbel_margin(r_ora["logits"], inv_t, w.sample_seed, canvas_id, step))
    err = np.abs(r_gpu["logits"] - r_ora["logits64"]).max(axis=1)
    safe = margin > 4 * err * float(inv_t) + 1e-6
    assert np.array_equal(r_gpu["tokens"][safe], r_ora["tokens"][safe])
    assert (r_gpu["tokens"] == r_ora["tokens"]).mean() >= 0.99
    Hb = w.commit_bound
    if w.commit_mode == 0:
        safe_c = np.abs(r_ora["H"] - Hb) > np.max(H_tol) * 2
        assert np.array_equal(r_gpu["commit"][safe_c], r_ora["commit"][safe_c])


# --- tiny fp32 workload: weights, encode, one round, full block ------------------------
@pytest.fixture(scope="module")
def tiny():
    w = I.TINY_FP32
    return w, dg.Model(w), om.Model(w)


def test_tiny_weights_bit_exact(tiny):
    w, gm, om_ = tiny
    shapes = {0: om_.embed, 1: om_.wsc}
    for l, L in enumerate(om_.layers):
        for j, name in enumerate(("wq", "wk", "wv", "wo", "wr", "wg", "wu", "wd")):
            shapes[om.layer_tensor_id(l, name)] = getattr(L, name)
    for tid, ref in shapes.items():
        out = torch.empty(ref.shape, dtype=torch.float32, device="cuda")
        gm.read_weight(tid, out)
        assert np.array_equal(host(out).view(np.uint32), ref.view(np.uint32)), tid


def test_tiny_encode_matches_oracle(tiny):
    w, gm, om_ = tiny
    P = w.prompt_len
    prompt = I.prompt_ids(w.sample_seed, 1, P, w.vocab)
    kv = gm.new_kv(1, P)
    gm.encode_prompt(cu(prompt), kv)
    K, V = read_kv(gm, kv, 1, P)
    Ko, Vo = om.encode_prompt(om_, prompt[0])
    assert np.allclose(K[:, 0, :, :P], Ko, rtol=1e-4, atol=1e-5)
    assert np.allclose(V[:, 0, :, :P], Vo, rtol=1e-4, atol=1e-5)


def test_tiny_round_and_block_match_oracle(tiny):
    w, gm, om_ = tiny
    P = w.prompt_len
    prompt = I.prompt_ids(w.sample_seed, 1, P, w.vocab)
    kv = gm.new_kv(1, P)
    gm.encode_prompt(cu(prompt), kv)
    Ko, Vo = om.encode_prompt(om_, prompt[0])
    canvas = sp.initial_canvas(w.sample_seed, 0, 256, w.vocab)
    out = step_buffers(w, 1)
    gm.denoise_step(kv, P, cu(canvas[None]), None, 0, 1.0, out)
    g = {k: host(v)[0] for k, v in out.items()}
    r = om.denoise_step(om_, Ko, Vo, canvas, None, 0, F32(1.0))
    compare_round(g, r, w, 0, 1.0, True)
    assert np.allclose(g["selfcond_next"], r["selfcond_next"], rtol=1e-4, atol=1e-6)
    # second round fed with the oracle's own self-conditioning and canvas
    gm.denoise_step(kv, P, cu(r["canvas_next"][None]), cu(r["selfcond_next"][None].astype(F32)), 1,
                    float(sp.schedule_t(1, w.max_steps)), out)
    g2 = {k: host(v)[0] for k, v in out.items()}
    r2 = om.denoise_step(om_, Ko, Vo, r["canvas_next"], r["selfcond_next"], 1, sp.schedule_t(1, w.max_steps),
                         prev_amax=r["amax"])
    compare_round(g2, r2, w, 1, float(sp.schedule_t(1, w.max_steps)), True)
    # full block on the device loop
    cout = torch.zeros((1, 256), dtype=torch.int32, device="cuda")
    su = torch.zeros(1, dtype=torch.int32, device="cuda")
    nc = torch.zeros(1, dtype=torch.int32, device="cuda")
    gm.encode_prompt(cu(prompt), kv)
    gm.generate_block(kv, 1, P, cout, su, nc)
    gm.sync_status()
    ref = om.generate_block(om_, Ko, Vo)
    assert int(host(su)[0]) == ref["steps_used"]
    assert (host(cout)[0] == ref["canvas"]).mean() >= 0.99
    assert abs(int(host(nc)[0]) - ref["n_committed"]) <= 2


def test_tiny_block_autoregressive_generation():
    # dg_generate: two blocks, the first joining the context before the second
    # (causal encode of its tokens after the prompt); against the oracle's chain
    w = I.TINY_FP32
    P, n_blocks = w.prompt_len, 2
    P_cap = P + 256 * (n_blocks - 1)
    gm = dg.Model(w, max_prompt=P_cap)
    prompt = I.prompt_ids(w.sample_seed, 1, P, w.vocab)
    kv = gm.new_kv(1, P_cap)
    toks = torch.zeros((1, n_blocks, 256), dtype=torch.int32, device="cuda")
    su = torch.zeros((1, n_blocks), dtype=torch.int32, device="cuda")
    nc = torch.zeros((1, n_blocks), dtype=torch.int32, device="cuda")
    gm.generate(cu(prompt), 1, P, n_blocks, kv, toks, su, nc)
    gm.sync_status()
    gt, gs, gn = host(toks)[0], host(su)[0], host(nc)[0]
    om_ = om.Model(w)
    refs = om.generate(om_, prompt[0], n_blocks)
    for i, ref in enumerate(refs):
        assert int(gs[i]) == ref["steps_used"], i
        assert (gt[i] == ref["canvas"]).mean() >= 0.99, i
        assert abs(int(gn[i]) - ref["n_committed"]) <= 2, i
    # the cache holds [prompt ; block 0] encoded causally (block 1's canvas after it)
    K, V = read_kv(gm, kv, 1, P_cap)
    Ko, Vo = om.encode_prompt(om_, np.concatenate([prompt[0], gt[0]]))
    assert np.allclose(K[:, 0, :, :P_cap], Ko, rtol=1e-4, atol=1e-5)
    assert np.allclose(V[:, 0, :, :P_cap], Vo, rtol=1e-4, atol=1e-5)
    gm.close()


def test_tiny_round_with_routing_bias(tiny):
    # structured per-token router bias (routing-locality workloads): the round
    # and the distinct experts each layer routed to match the oracle's
    w, gm, om_ = tiny
    P = w.prompt_len
    prompt = I.prompt_ids(w.sample_seed, 1, P, w.vocab)
    kv = gm.new_kv(1, P)
    gm.encode_prompt(cu(prompt), kv)
    Ko, Vo = om.encode_prompt(om_, prompt[0])
    rb = I.routing_bias(11, w.n_layers, 256, w.n_experts, w.top_k, pool=4, beta=2.0)
    gm.set_routing_bias(cu(rb))
    try:
        canvas = sp.initial_canvas(w.sample_seed, 0, 256, w.vocab)
        out = step_buffers(w, 1)
        gm.denoise_step(kv, P, cu(canvas[None]), None, 0, 1.0, out)
        g = {k: host(v)[0] for k, v in out.items()}
        touched = gm.touched_experts()
    finally:
        gm.set_routing_bias(None)
    biased = copy.copy(om_)
    biased.route_bias = rb
    trace = []
    r = om.denoise_step(biased, Ko, Vo, canvas, None, 0, F32(1.0), trace=trace)
    compare_round(g, r, w, 0, 1.0, True)
    assert touched == [len(np.unique(trace[l]["ids"])) for l in range(w.n_layers)]


def test_tiny_topk_sampler_round_and_block_match_oracle():
    # sampling truncated to the 16 largest logits: rounds (tokens, entropy,
    # commit, self-conditioning through the candidate gather) and a full block
    K = 16
    w = I.TINY_FP32.replace(sample_topk=K)
    gm, om_ = dg.Model(w), om.Model(w)
    P = w.prompt_len
    prompt = I.prompt_ids(w.sample_seed, 1, P, w.vocab)
    kv = gm.new_kv(1, P)
    gm.encode_prompt(cu(prompt), kv)
    Ko, Vo = om.encode_prompt(om_, prompt[0])
    canvas = sp.initial_canvas(w.sample_seed, 0, 256, w.vocab)
    out = step_buffers(w, 1)
    gm.denoise_step(kv, P, cu(canvas[None]), None, 0, 1.0, out)
    g = {k: host(v)[0] for k, v in out.items()}
    r = om.denoise_step(om_, Ko, Vo, canvas, None, 0, F32(1.0))
    compare_round(g, r, w, 0, 1.0, True, topk=K)
    assert np.allclose(g["selfcond_next"], r["selfcond_next"], rtol=1e-4, atol=1e-6)
    t1 = float(sp.schedule_t(1, w.max_steps))
    gm.denoise_step(kv, P, cu(r["canvas_next"][None]), cu(r["selfcond_next"][None].astype(F32)), 1, t1, out)
    g2 = {k: host(v)[0] for k, v in out.items()}
    r2 = om.denoise_step(om_, Ko, Vo, r["canvas_next"], r["selfcond_next"], 1, sp.schedule_t(1, w.max_steps),
                         prev_amax=r["amax"])
    compare_round(g2, r2, w, 1, t1, True, topk=K)
    cout = torch.zeros((1, 256), dtype=torch.int32, device="cuda")
    su = torch.zeros(1, dtype=torch.int32, device="cuda")
    nc = torch.zeros(1, dtype=torch.int32, device="cuda")
    gm.generate_block(kv, 1, P, cout, su, nc)
    gm.sync_status()
    ref = om.generate_block(om_, Ko, Vo)
    assert int(host(su)[0]) == ref["steps_used"]
    assert (host(cout)[0] == ref["canvas"]).mean() >= 0.99
    assert abs(int(host(nc)[0]) - ref["n_committed"]) <= 2
    gm.close()


# --- mid bf16 workload with a synthetic prompt cache -------------------------------------
@pytest.fixture(scope="module")
def mid():
    w = I.MID_BF16
    return w, dg.Model(w), om.Model(w)


def test_mid_weights_sampled_bit_exact(mid):
    w, gm, om_ = mid
    for tid, ref in ((0, om_.embed), (om.layer_tensor_id(3, "wg"), om_.layers[3].wg),
                     (om.layer_tensor_id(7, "wd"), om_.layers[7].wd), (om.layer_tensor_id(0, "wk"), om_.layers[0].wk)):
        out = torch.empty(ref.shape, dtype=torch.bfloat16, device="cuda")
        gm.read_weight(tid, out)
        assert np.array_equal(host(out).view(np.uint32), ref.view(np.uint32)), tid


DELTA = 0.005  # router-logit distance to a top-k tie below which a routing decision is ambiguous


def oracle_pair(w, K, V, canvas, canvas_id=0):
    """The oracle's round and the same round under storage noise (the
    envelope two correct bf16 implementations can differ by)."""
    trace, trace_n = [], []
    r = om.denoise_step(om.Model(w), K, V, canvas, None, 0, F32(1.0), canvas_id=canvas_id, trace=trace)
    rn = om.denoise_step(NoisyStore(w), K, V, canvas, None, 0, F32(1.0), canvas_id=canvas_id, trace=trace_n)
    return r, trace, rn, trace_n


def as_path_outputs(r):
    """An oracle round's outputs under the CUDA path's names."""
    return dict(logits=r["logits64"], entropy=r["H"], tokens=r["tokens"], selfcond_next=r["selfcond_next"])


def deviation(x_a, x_b, g_a, g_b, stable):
    """Deviation of one round from another on the routing-stable tokens:
    final normalised state in bf16 steps at unit scale, logits, entropy,
    self-conditioning (relative per row) and token agreement."""
    so = g_b["selfcond_next"][stable]
    rel = np.sqrt(((g_a["selfcond_next"][stable] - so) ** 2).mean(axis=1) /
                  np.maximum((so ** 2).mean(axis=1), 1e-30))
    return dict(x=quantiles(rms_ulps(x_a[stable], x_b[stable])),
                logit=quantiles(np.abs(g_a["logits"][stable] - g_b["logits64"][stable])),
                H=quantiles(np.abs(g_a["entropy"][stable] - g_b["H"][stable])),
                sc=quantiles(rel),
                tokens=float((g_a["tokens"][stable] == g_b["tokens"][stable]).mean()))


def within_envelope(dg_, dn, slack):
    """dg_ (CUDA path vs oracle) within twice dn (perturbed oracle vs oracle)
    plus `slack`, quantile by quantile."""
    for key, qs in (("x", (0.99, 0.999)), ("logit", (0.99, 0.999)), ("H", (0.99,)), ("sc", (0.99,))):
        for q in qs:
            assert dg_[key][q] <= 2 * dn[key][q] + slack[key], (key, q, dg_[key][q], dn[key][q])
    assert dg_["tokens"] >= dn["tokens"] - 0.02, (dg_["tokens"], dn["tokens"])


SLACK = dict(x=1.0, logit=2e-2, H=1e-3, sc=1e-2)


def compare_bf16_round(g, r, trace, om_model, w, gx_final, rn, trace_n, min_stable=0.9, canvas_id=0):
    """bf16 parity of one round against the oracle, assessed by the storage-noise
    envelope, plus the workload's 2e-2 on the LM head where it applies.

    * LM head: the logits equal logit_scale * x E^T of the path's own final
      normalised state x within 2e-2 absolute (the bf16 workloads' tolerance,
      which holds once both sides read the same x).
    * Upstream: every value is rounded to bf16 at the storage points, so an
      implementation that accumulates in fp32 rounds some of them to the
      other neighbour, and the model spreads each such step (RMSNorm scales
      the whole row).  The CUDA path's deviation from the oracle -- final
      normalised state, logits, entropy, self-conditioning -- must stay
      within twice the deviation of the storage-noise oracle, quantile by
      quantile, and agree on as many sampled tokens.
    * Tokens: identical wherever the Gumbel-max margin exceeds twice the row's
      logit error (the decision cannot move there).
    * Routing: a top-k decision within DELTA of a tie has more than one
      correct outcome; such tokens are left out, and in a single-layer model
      must match one of the selections the oracle enumerates as valid.
    Returns (n_stable, n_ambiguous)."""
    T = g["logits"].shape[0]
    layers = [tr for tr in trace if "margin" in tr]
    xo, xn = trace[-1]["x_final"], trace_n[-1]["x_final"]
    margin = np.min(np.stack([tr["margin"] for tr in layers]), axis=0)
    stable = margin >= DELTA
    assert stable.mean() >= min_stable, stable.mean()
    # LM head given the same normalised state
    lm = w.logit_scale * (gx_final.astype(np.float64) @ om_model.embed.astype(np.float64).T)
    lm_err = np.abs(g["logits"] - lm).max()
    assert lm_err <= 2e-2, lm_err
    dg_ = deviation(gx_final, xo, g, r, stable)
    dn = deviation(xn, xo, as_path_outputs(rn), r, stable)
    print(f"stable {stable.mean():.3f}; LM head err {lm_err:.2e}; path vs oracle {dg_}; noise envelope {dn}")
    within_envelope(dg_, dn, SLACK)
    dl = np.abs(g["logits"] - r["logits64"]).max(axis=1)
    Hs = r["H"][stable]
    assert np.all(np.abs(g["entropy"][stable] - Hs) <= 3 * np.maximum(Hs, 1.0) * dl[stable] + 1e-3)
    inv_t = F32(1.0) / sp.temperature(F32(1.0), w.temp_start, w.temp_end)
    gm_ = gumbel_margin(r["logits"], inv_t, w.sample_seed, canvas_id, 0)
    safe = gm_ > 2 * dl * float(inv_t)
    assert np.array_equal(g["tokens"][safe], r["tokens"][safe])
    if len(layers) == 1:
        layer = om_model.layers[0]
        tol = 2 * dn["logit"]["max"] + SLACK["logit"]
        for t in np.nonzero(~stable)[0]:
            alts = om.routing_alternatives(layers[0]["router"][t], w.top_k, DELTA)
            rows = [om.token_logits_with_routing(om_model, layer, layers[0]["h_attn"][t], ids, gt)
                    for ids, gt in alts]
            assert min(np.abs(g["logits"][t] - row).max() for row in rows) <= tol, t
    return int(stable.sum()), int(T - stable.sum())


def traced_round(gm, w, kv, B, P, canvas):
    """One GPU round with the diagnostic trace on; returns (outputs, x_final)."""
    T = B * 256
    htr = torch.zeros((2 * w.n_layers + 1, T, w.d_model), dtype=torch.float32, device="cuda")
    itr = torch.zeros((w.n_layers, T, w.top_k), dtype=torch.int32, device="cuda")
    gm.debug_trace(htr, itr)
    out = step_buffers(w, B)
    gm.denoise_step(kv, P, cu(canvas), None, 0, 1.0, out)
    gm.sync_status()
    gm.debug_trace(None, None)
    return {k: host(v) for k, v in out.items()}, host(htr)[2 * w.n_layers]


def run_bf16_round(w, P, kv_seed):
    gm = dg.Model(w)
    K, V = I.prompt_kv(kv_seed, w.n_layers, 1, w.n_kv_heads, P, w.head_dim, bf16=True)
    kv = gm.new_kv(1, P)
    gm.load_kv(kv, 1, P, cu(K).to(torch.bfloat16), cu(V).to(torch.bfloat16))
    canvas = sp.initial_canvas(w.sample_seed, 0, 256, w.vocab)
    gout, gx = traced_round(gm, w, kv, 1, P, canvas[None])
    g = {k: v[0] for k, v in gout.items()}
    gm.close()
    r, trace, rn, trace_n = oracle_pair(w, K[:, 0], V[:, 0], canvas)
    return g, r, trace, om.Model(w), gx, rn, trace_n


@pytest.mark.parametrize("layers", [1, 2])
def test_mid_round_matches_oracle(layers):
    w = I.MID_BF16.replace(n_layers=layers)
    g, r, trace, om_, gx, rn, trace_n = run_bf16_round(w, w.prompt_len, 9)
    compare_bf16_round(g, r, trace, om_, w, gx, rn, trace_n, min_stable=0.9 if layers == 1 else 0.8)


def test_mid_full_depth_round_statistics(mid):
    """All 8 layers: near-tie routing flips in early layers propagate through
    attention to every token, so no token set is routing-stable; the round is
    assessed by whole-round statistics against the storage-noise envelope, and
    the LM head by the workload's 2e-2 given the same normalised state."""
    w, gm, om_ = mid
    g, r, trace, _, gx, rn, trace_n = run_bf16_round(w, w.prompt_len, 9)
    lm = w.logit_scale * (gx.astype(np.float64) @ om_.embed.astype(np.float64).T)
    assert np.abs(g["logits"] - lm).max() <= 2e-2

    def stats(a, x_a):
        return dict(frac=float((np.abs(a["logits"] - r["logits64"]) <= 2e-2).mean()),
                    amax=float((a["argmax"] == r["amax"]).mean()),
                    tokens=float((a["tokens"] == r["tokens"]).mean()),
                    dH=float(np.median(np.abs(a["entropy"] - r["H"]))),
                    x50=float(np.median(rms_ulps(x_a, trace[-1]["x_final"]))))
    sg = stats(g, gx)
    sn = stats(dict(logits=rn["logits64"], argmax=rn["amax"], tokens=rn["tokens"], entropy=rn["H"]),
               trace_n[-1]["x_final"])
    print(f"full depth: path vs oracle {sg}; noise envelope {sn}")
    assert sg["frac"] >= sn["frac"] - 0.1 and sg["amax"] >= sn["amax"] - 0.1
    assert sg["tokens"] >= sn["tokens"] - 0.1
    assert sg["dH"] <= 2 * sn["dH"] + 1e-3 and sg["x50"] <= 2 * sn["x50"] + 1.0
