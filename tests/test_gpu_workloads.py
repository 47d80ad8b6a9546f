"""Parity and properties on the remaining workloads (B200 only).

* 26B-A4B shape: a 2-layer slice of the architecture (same d, heads,
  experts, vocab) against the oracle; the full 30-layer model at full size
  through properties that hold at any size (the oracle cannot afford it).
* multi-canvas batching with the Zipf-skewed router: per-canvas parity for
  B = 2, and B = 32 against single-canvas runs of the same canvases.
* long context: 32768-token prompt cache, logit scale 16 -- one round
  against the oracle and a full block loop (early stop exercised).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_text_diffusion_b200 as dg  # noqa: E402
from block_text_diffusion_b200 import inputs as I  # noqa: E402
from oracle import model as om, sampler as sp  # noqa: E402

import test_gpu_step as ts  # noqa: E402

F32 = np.float32


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dg.lib()


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def synthetic_kv(gm, w, B, P, seed):
    K, V = I.prompt_kv(seed, w.n_layers, B, w.n_kv_heads, P, w.head_dim, bf16=True)
    kv = gm.new_kv(B, P)
    gm.load_kv(kv, B, P, cu(K).to(torch.bfloat16), cu(V).to(torch.bfloat16))
    return kv, K, V


def run_round(gm, w, kv, B, P, canvas, selfcond=None, step=0, t=1.0):
    out = ts.step_buffers(w, B)
    gm.denoise_step(kv, P, cu(canvas), selfcond, step, t, out)
    gm.sync_status()
    return {k: ts.host(v) for k, v in out.items()}


# --- 26B-A4B shape ------------------------------------------------------------------------
@pytest.mark.slow
def test_moe26b_one_layer_slice_matches_oracle():
    # one layer of the 26B-A4B shape (d 2816, 16/8 heads, 128 experts top-8,
    # vocab 262144) with its 2048-token prompt cache, against the oracle
    w = I.MOE26B_BF16.replace(n_layers=1, name="moe26b-L1")
    g, r, trace, om_, gx, rn, trace_n = ts.run_bf16_round(w, w.prompt_len, 21)
    ts.compare_bf16_round(g, r, trace, om_, w, gx, rn, trace_n)


@pytest.mark.slow
def test_moe26b_full_size_properties():
    w = I.MOE26B_BF16
    P = w.prompt_len
    gm = dg.Model(w)
    prompt = I.prompt_ids(w.sample_seed, 1, P, w.vocab)
    kv = gm.new_kv(1, P)
    gm.encode_prompt(cu(prompt), kv)
    canvas = sp.initial_canvas(w.sample_seed, 0, 256, w.vocab)
    g = run_round(gm, w, kv, 1, P, canvas[None])
    counts = torch.zeros((w.n_layers, w.n_experts), dtype=torch.int32, device="cuda")
    cnt = ts.host(gm.expert_counts(counts))
    touched = gm.touched_experts()
    l = g["logits"][0]
    H = g["entropy"][0]
    assert np.isfinite(l).all() and np.isfinite(H).all()
    assert np.all(H >= -1e-6) and np.all(H <= np.log(w.vocab) + 1e-5)
    assert np.array_equal(g["argmax"][0], l.argmax(axis=1))
    assert np.all((g["tokens"][0] >= 0) & (g["tokens"][0] < w.vocab))
    assert np.array_equal(g["commit"][0].astype(bool), H < F32(w.commit_bound))
    assert g["n_committed"][0] == g["commit"][0].sum()
    # every layer routes all 256 x 8 (token, slot) pairs; the touched count is
    # the number of experts with rows (random-init hidden states are strongly
    # correlated across tokens, so far fewer than 128 experts are touched)
    assert np.all(cnt.sum(axis=1) == 256 * w.top_k)
    assert touched == list((cnt > 0).sum(axis=1))
    assert all(w.top_k <= t <= w.n_experts for t in touched)
    # the full block on the device loop runs to its budget (random weights never converge)
    out = torch.zeros((1, 256), dtype=torch.int32, device="cuda")
    su = torch.zeros(1, dtype=torch.int32, device="cuda")
    nc = torch.zeros(1, dtype=torch.int32, device="cuda")
    gm.generate_block(kv, 1, P, out, su, nc)
    gm.sync_status()
    assert int(ts.host(su)[0]) == w.max_steps
    gm.close()


# --- batching with a Zipf-skewed router ----------------------------------------------------
def test_batch_two_canvases_match_oracle():
    # one layer of the batching workload (Zipf-skewed router), two canvases,
    # each against its own oracle run
    w = I.BATCH_ZIPF.replace(n_layers=1)
    B, P = 2, 2048
    gm = dg.Model(w, max_canvases=B, max_prompt=P)
    kv, K, V = synthetic_kv(gm, w, B, P, 31)
    canvas = np.stack([sp.initial_canvas(w.sample_seed, b, 256, w.vocab) for b in range(B)])
    g, gx = ts.traced_round(gm, w, kv, B, P, canvas)
    counts = torch.zeros((w.n_layers, w.n_experts), dtype=torch.int32, device="cuda")
    cnt = ts.host(gm.expert_counts(counts)).sum(axis=0)
    gm.close()
    om_ = om.Model(w)
    for b in range(B):
        r, trace, rn, trace_n = ts.oracle_pair(w, K[:, b], V[:, b], canvas[b], canvas_id=b)
        gb = {k: v[b] for k, v in g.items() if v.ndim >= 1 and v.shape[0] == B}
        ts.compare_bf16_round(gb, r, trace, om_, w, gx[b * 256:(b + 1) * 256], rn, trace_n, canvas_id=b)
    # the Zipf bias skews the load: expert 0 gets far more rows than the last
    assert cnt[0] > 4 * max(1, cnt[-1])


def test_batch_32_equals_single_canvas_runs():
    # 32 canvases batched against the same canvases run one at a time (one
    # layer, so a routing tie moves only its own token): batching changes
    # only tile shapes and split-K orders, so the final normalised states
    # differ by no more than the storage-noise envelope of canvas 0
    w = I.BATCH_ZIPF.replace(n_layers=1)
    B, P = 32, 2048
    gm = dg.Model(w, max_canvases=B, max_prompt=P)
    kv, K, V = synthetic_kv(gm, w, B, P, 41)
    canvas = np.stack([sp.initial_canvas(w.sample_seed, b, 256, w.vocab) for b in range(B)])
    g, gx = ts.traced_round(gm, w, kv, B, P, canvas)
    _, trace, _, trace_n = ts.oracle_pair(w, K[:, 0], V[:, 0], canvas[0])
    env = ts.quantiles(ts.rms_ulps(trace_n[-1]["x_final"], trace[-1]["x_final"]))
    for b in (0, 7, 31):
        kv1 = gm.new_kv(1, P)
        gm.load_kv(kv1, 1, P, cu(K[:, b:b + 1]).to(torch.bfloat16), cu(V[:, b:b + 1]).to(torch.bfloat16))
        _, gx1 = ts.traced_round(gm, w, kv1, 1, P, canvas[b:b + 1])
        xb = gx[b * 256:(b + 1) * 256]
        du = ts.quantiles(ts.rms_ulps(gx1, xb))
        print(f"canvas {b}: batched vs single {du}; envelope {env}")
        assert du[0.5] <= 2 * env[0.5] + 1.0 and du[0.99] <= 2 * env[0.99] + 1.0
    gm.close()


# --- long context, fast-converging canvas -------------------------------------------------
@pytest.mark.slow
def test_long_context_round_matches_oracle():
    # one layer of the long-context workload: 32768-token prompt cache,
    # logit scale 16
    w = I.LONG_CTX.replace(n_layers=1)
    g, r, trace, om_, gx, rn, trace_n = ts.run_bf16_round(w, w.prompt_len, 51)
    ts.compare_bf16_round(g, r, trace, om_, w, gx, rn, trace_n)


@pytest.mark.slow
@pytest.mark.parametrize("layers", [1, 8])
def test_long_context_block_loop_matches_oracle(layers):
    # the full device block loop of the fast-converging workload (logit scale
    # 16) against the oracle's loop: rounds used, committed count, and the
    # committed tokens.  With one layer the loop converges in its first rounds
    # and the committed tokens must agree on >= 99% (the workload's
    # multi-round criterion).  With all 8 layers the random-init model does
    # not converge within the budget, and any storage-rounding difference
    # sends the sampled trajectory elsewhere; the oracle's own storage-noise
    # run measures how far, and the device loop must stay within that.
    w = I.LONG_CTX.replace(n_layers=layers)
    P = w.prompt_len
    gm = dg.Model(w)
    kv, K, V = synthetic_kv(gm, w, 1, P, 52)
    out = torch.zeros((1, 256), dtype=torch.int32, device="cuda")
    su = torch.zeros(1, dtype=torch.int32, device="cuda")
    nc = torch.zeros(1, dtype=torch.int32, device="cuda")
    gm.generate_block(kv, 1, P, out, su, nc)
    gm.sync_status()
    steps, ncom, canvas = int(ts.host(su)[0]), int(ts.host(nc)[0]), ts.host(out)[0]
    gm.close()
    ref = om.generate_block(om.Model(w), K[:, 0], V[:, 0])
    committed = ref["trace"][-1]["commit"] == 1

    def agreement(c):
        return float((c[committed] == ref["canvas"][committed]).mean()) if committed.any() else 1.0
    agree = agreement(canvas)
    print(f"long L{layers}: rounds gpu {steps} oracle {ref['steps_used']}; committed gpu {ncom} oracle "
          f"{ref['n_committed']}; committed-token agreement {agree:.4f}; all-token agreement "
          f"{(canvas == ref['canvas']).mean():.4f}")
    if layers == 1:
        assert steps == ref["steps_used"]
        assert abs(ncom - ref["n_committed"]) <= max(2, ref["n_committed"] // 50)
        assert agree >= 0.99
        return
    rn = om.generate_block(ts.NoisyStore(w), K[:, 0], V[:, 0])
    agree_n = agreement(rn["canvas"])
    print(f"  noise envelope: rounds {rn['steps_used']}; committed {rn['n_committed']}; "
          f"committed-token agreement {agree_n:.4f}")
    assert abs(steps - ref["steps_used"]) <= 2 * abs(rn["steps_used"] - ref["steps_used"]) + 1
    # once the trajectories have diverged, each position's final commit is an
    # independent draw: the committed count of another correct run scatters
    # binomially around the oracle's (three standard deviations allowed)
    p = ref["n_committed"] / 256.0
    sd = np.sqrt(256.0 * p * (1.0 - p))
    assert abs(ncom - ref["n_committed"]) <= max(2 * abs(rn["n_committed"] - ref["n_committed"]), 3.0 * sd) + 2
    assert agree >= agree_n - 0.05
