"""Layer-by-layer parity of the canvas pass on the bf16 workloads (B200 only).

Every layer of the 30-layer 26B-A4B-shaped model and of the 8-layer mid
model is run alone on the GPU (dg_test_layer) and in the oracle from the same
seeded inputs: a residual state h_in entering the layer, the prompt keys and
values of the cache, and (where used) a router bias.  No input of the oracle
comes from the CUDA path, and each layer is compared from identical inputs,
so rounding differences cannot compound across layers and a fixed bound
holds.

The bound.  Both sides round to bf16 at the
same storage points; the GPU accumulates in fp32 (and feeds the attention
probabilities to the tensor core in bf16), the oracle in fp64.  A value whose
exact result lies that close to a bf16 rounding midpoint lands on the other
neighbour, one bf16 step away.  Steps are counted at the bf16 spacing of
max(|value|, |residual it was added to|, rms of its row): the residual term
because a stored sum carries its addend's difference, measured at the
addend's own magnitude, and the row-rms floor so that elements cancelling to
near zero do not count an absolute error in their own tiny spacing.  Then:
  * keys, values: rounded once from GEMM outputs of identical normalised
    inputs, whose fp32-vs-fp64 error is a small fraction of a step: <= 1 step
    from the rounding, <= 2 allowed;
  * h after attention = round(h_in + O), h_in identical on both sides and O's
    error (bf16 P, fp32 sums) under a step: <= 2 steps;
  * h after the MoE, with the MoE half run again on the GPU from the oracle's
    h after attention (dg_test_moe): the GPU's fp32 gate and up sums flip the
    SwiGLU activation's rounding for a few elements and the down projection
    sums those one-step differences, plus the final rounding: <= 3 steps;
  * h after the MoE of the whole layer: RMSNorm(h after attention) carries
    that tensor's allowed deviation into the experts, SwiGLU (a product of two
    projections) doubles a relative deviation, and at random init the MoE
    output is larger than the residual: <= 8 steps and 2^-7 of the rms (a
    check for gross mistakes; the tight check is the MoE half's).
And the whole tensor's rms deviation must stay within 2^-8 of its rms (at
most about half the values one step off), except for the whole layer's h
after the MoE as stated.  tests/test_parity_bounds.py checks both MoE bounds
against the oracle's own deviation when its inputs move as each premise
allows.  A systematic mistake (a head rotated at the wrong position, a
missing residual, a wrong gate) moves many values by many steps and fails.

Compared per layer: the canvas keys (after RoPE) and values the layer writes
into the cache, h after the attention residual, h after the MoE, and the
routing.  Routing: the router reads RMSNorm(h after attention), which may
legitimately differ from the oracle's within the rms bound above (2^-8 of
its unit rms), and that moves the difference of two router logits by up to
sqrt(2) 2^-8 ||Wr_e|| rms.  A top-k decision closer to a tie than four times
that has more than one correct outcome: the GPU's selection must be a set of
k experts none of which lies more than that window below the best one left
out (slots in descending logit order, near-ties in either order), and that
token's h after the MoE is compared with the oracle's result for the GPU's
selection (gates the softmax of the oracle's logits of the selected
experts).

Workloads: the mid model with its own routing on all 8 layers; the 26B-A4B
shape with its own routing on its first and last layer, and on all 30 layers
with a seeded router bias that gives each layer a pool of 16 experts (the top
8 of the pool chosen by the router's own logits), so the oracle generates 16
of the 128 experts of each layer."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import block_text_diffusion_b200 as dg  # noqa: E402
from block_text_diffusion_b200 import inputs as I  # noqa: E402
from oracle import model as om  # noqa: E402

F32 = np.float32
REL_RMS = 2.0 ** -8     # rms deviation of a tensor relative to its rms
H_STD = 0.1             # scale of the seeded residual state entering a layer


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    dg.lib()


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16_steps(got, ref, addend=None):
    """|got - ref| in bf16 spacings at max(|ref|, |addend|, rms of the row)."""
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    mag = np.maximum(np.abs(ref), rms)
    if addend is not None:
        mag = np.maximum(mag, np.abs(np.asarray(addend, dtype=np.float64)))
    spacing = np.exp2(np.floor(np.log2(np.maximum(mag, 1e-30))) - 7.0)
    return np.abs(np.asarray(got, dtype=np.float64) - ref) / spacing


def worst(e, got, ref, n=6):
    """The n largest deviations: (row, column, reference, got, steps)."""
    flat = np.argsort(e.ravel())[::-1][:n]
    out = []
    for f in flat:
        i = np.unravel_index(f, e.shape)
        out.append((tuple(int(x) for x in i), float(np.asarray(ref)[i]), float(np.asarray(got)[i]), float(e[i])))
    return out


def check_close(name, got, ref, layer, max_steps, addend=None, extra="", rel_max=REL_RMS):
    e = bf16_steps(got, ref, addend)
    ref64 = np.asarray(ref, dtype=np.float64)
    rel = np.sqrt(np.mean((np.asarray(got, dtype=np.float64) - ref64) ** 2)) / np.sqrt(np.mean(ref64 ** 2))
    assert e.max() <= max_steps, (f"layer {layer} {name}: {e.max():.2f} bf16 steps (p99 {np.quantile(e, 0.99):.2f}, "
                                  f"rows over 2: {sorted(set(np.nonzero(e > 2)[0].tolist()))[:20]}) "
                                  f"worst {worst(e, got, ref)} {extra}")
    assert rel <= rel_max, f"layer {layer} {name}: rms deviation {rel:.2e} of rms"
    return float(e.max()), float(rel), float((e > 0).mean())


def pool_bias(seed, n_layers, n_experts, pool, beta=16.0):
    """Router bias [L, 256, E]: +beta on a seeded pool of experts per layer,
    the same for every token (the router's own logits pick top-k inside it)."""
    g = np.random.default_rng(seed)
    out = np.zeros((n_layers, 256, n_experts), dtype=F32)
    for l in range(n_layers):
        out[l, :, g.permutation(n_experts)[:pool]] = beta
    return out


def router_window(wr):
    """Four standard deviations of the difference of two router logits when the
    router's input deviates by the allowed rms (2^-8 of its unit rms)."""
    return 4.0 * np.sqrt(2.0) * REL_RMS * float(np.sqrt((np.asarray(wr, dtype=np.float64) ** 2).sum(axis=1)).max())


def moe_row_with(model, layer, x2_row, ids, gates):
    """sum_j g_j FFN_{e_j}(x) of one token for a given selection (oracle arithmetic)."""
    y = np.zeros(x2_row.shape[-1])
    for e, g in zip(ids, gates):
        a = model.store(om.silu(x2_row @ layer.wg[e].astype(np.float64).T) * (x2_row @ layer.wu[e].astype(np.float64).T))
        y += g * (a @ layer.wd[e].astype(np.float64).T)
    return y


def read_layer_kv(kv, w, P, layer):
    """Canvas keys/values of one layer from the cache: [256, Hkv, hd] each."""
    S = ((P + 256 + 63) // 64) * 64
    n = w.n_layers * w.n_kv_heads * S * w.head_dim
    raw = kv[: 2 * n * 2].view(torch.bfloat16)
    K = raw[:n].view(w.n_layers, w.n_kv_heads, S, w.head_dim)[layer, :, P:P + 256]
    Vt = raw[n:].view(w.n_layers, w.n_kv_heads, w.head_dim, S)[layer, :, :, P:P + 256]
    torch.cuda.synchronize()
    return (K.float().cpu().numpy().transpose(1, 0, 2), Vt.float().cpu().numpy().transpose(2, 0, 1))


def check_moe(name, model, lw, t, layer, g_out, g_ids, max_steps, rel_rms):
    """Routing valid within the router window, and h after the MoE against the
    oracle's (recomputed for the GPU's selection where that differs)."""
    k = model.cfg.top_k
    window = router_window(lw.wr)
    ref_out = t["h_out"].copy()
    x2 = model.store(om.rmsnorm(t["h_attn"], model.cfg.rms_eps))
    n_alt = 0
    for i in range(g_ids.shape[0]):
        if np.array_equal(g_ids[i], t["ids"][i]):
            continue
        r = t["router"][i]
        sel = g_ids[i]
        assert len(set(sel.tolist())) == k, f"layer {layer} {name} token {i}: repeated expert in {sel}"
        # slots run in descending logit order: two selected experts whose
        # logits lie within the window may come in either order
        assert all(r[a] >= r[b] - window for a, b in zip(sel[:-1], sel[1:])), \
            f"layer {layer} {name} token {i}: GPU slot order {sel} (logits {r[sel]})"
        rest = np.delete(r, sel)
        assert rest.size == 0 or r[sel].min() >= rest.max() - window, (
            f"layer {layer} {name} token {i}: GPU routing {sel} is not a top-{k} selection within {window:.4f} "
            f"(oracle {t['ids'][i]}, logits {np.sort(r)[::-1][:k + 2]})")
        if set(sel.tolist()) == set(t["ids"][i].tolist()):
            continue                      # the same experts and gates, slots in another order
        n_alt += 1
        ex = np.exp(r[sel] - r[sel].max())
        y = moe_row_with(model, lw, x2[i], sel, ex / ex.sum())
        ref_out[i] = model.store(t["h_attn"][i] + y)
    # a broken router would move most tokens; near-ties move a few
    assert n_alt <= 64, f"layer {layer} {name}: {n_alt} tokens routed differently"
    diff_rows = [i for i in range(g_ids.shape[0]) if not np.array_equal(g_ids[i], t["ids"][i])]
    extra = (f"| rows with other slot order or selection {diff_rows[:20]}; smallest router margins "
             f"{sorted((round(float(m), 5), i) for i, m in enumerate(t['margin']))[:6]}")
    st = check_close(name, g_out, ref_out, layer, max_steps, addend=t["h_attn"], extra=extra, rel_max=rel_rms)
    return st, n_alt, window


def check_layer(gm, w, kv, P, Kp, Vp, layer, h_in, bias):
    d, k = w.d_model, w.top_k
    trace = torch.zeros((3, 256, d), dtype=torch.float32, device="cuda")
    ids = torch.zeros((256, k), dtype=torch.int32, device="cuda")
    gm.run_layer(kv, 1, P, layer, cu(h_in).to(torch.bfloat16), trace, ids)
    torch.cuda.synchronize()
    g_tr = trace.cpu().numpy()
    g_ids = ids.cpu().numpy()
    g_k, g_v = read_layer_kv(kv, w, P, layer)

    model = om.Model(w, layers=0, with_embed=False)
    lw = om.layer_weights(w, layer, lazy_experts=True)
    tr = []
    _, k_new, v_new = om.block(model, lw, h_in.astype(np.float64), P + np.arange(256),
                               Kp[layer].transpose(1, 0, 2).astype(np.float64),
                               Vp[layer].transpose(1, 0, 2).astype(np.float64), causal=False, trace=tr,
                               route_bias=None if bias is None else bias[layer])
    t = tr[0]
    stats = {}
    stats["k"] = check_close("canvas keys", g_k, k_new, layer, 2)
    stats["v"] = check_close("canvas values", g_v, v_new, layer, 2)
    stats["h_attn"] = check_close("h after attention", g_tr[0], t["h_attn"], layer, 2, addend=h_in)
    stats["h_out_layer"], _, _ = check_moe("h after the MoE (whole layer)", model, lw, t, layer, g_tr[1], g_ids,
                                           8, 2 * REL_RMS)
    # the MoE half again, from the oracle's h after attention
    trace.zero_()
    gm.run_moe(1, layer, cu(t["h_attn"]).to(torch.bfloat16), trace, ids)
    torch.cuda.synchronize()
    g_tr = trace.cpu().numpy()
    g_ids = ids.cpu().numpy()
    stats["h_out"], stats["alt"], window = check_moe("h after the MoE", model, lw, t, layer, g_tr[1], g_ids,
                                                     3, REL_RMS)
    stats["window"] = round(window, 4)
    return stats


def layer_sweep(w, P, seed, layers, bias=None):
    gm = dg.Model(w, max_canvases=1, max_prompt=P)
    try:
        Kp, Vp = I.prompt_kv(seed, w.n_layers, 1, w.n_kv_heads, P, w.head_dim, bf16=True)
        kv = gm.new_kv(1, P)
        gm.load_kv(kv, 1, P, cu(Kp).to(torch.bfloat16), cu(Vp).to(torch.bfloat16))
        Kp, Vp = Kp[:, 0], Vp[:, 0]
        bias_t = None
        if bias is not None:
            bias_t = cu(bias)
            gm.set_routing_bias(bias_t)
        out = {}
        for l in layers:
            h_in = I.normal(seed + 1000 + l, 111, (256, w.d_model), std=H_STD, bf16=True)
            out[l] = check_layer(gm, w, kv, P, Kp, Vp, l, h_in, bias)
            print(f"layer {l}: " + ", ".join(f"{k} {v}" for k, v in out[l].items()))
        return out
    finally:
        gm.close()


@pytest.mark.slow
def test_mid_every_layer_matches_oracle():
    w = I.MID_BF16
    layer_sweep(w, w.prompt_len, 61, range(w.n_layers))


@pytest.mark.slow
def test_moe26b_first_and_last_layer_own_routing_match_oracle():
    w = I.MOE26B_BF16
    layer_sweep(w, w.prompt_len, 62, [0, w.n_layers - 1])


@pytest.mark.slow
def test_moe26b_every_layer_with_expert_pool_matches_oracle():
    w = I.MOE26B_BF16
    bias = pool_bias(63, w.n_layers, w.n_experts, 16)
    layer_sweep(w, w.prompt_len, 63, range(w.n_layers), bias=bias)
