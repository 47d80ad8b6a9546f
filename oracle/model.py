"""Oracle of the block-diffusion denoiser: weights, causal prompt encode, one
denoising step over a 256-token canvas, and the full block loop.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
bench's CPU-baseline leg; shares no code with the CUDA path.

What the pages fix (DiffusionGemma technical-report explainer, mlqm.cn,
section 二; "谷歌都下场了：扩散语言模型的四倍速与六倍错", bohuyeshan.top,
section 一):
  * one set of weights used two ways: the prompt is encoded with causal
    attention into a cached KV; the 256-token canvas is refined with
    bidirectional attention over [prompt KV ; canvas];
  * a Mixture-of-Experts FFN, each token routed to 8 of 128 experts in the
    26B-A4B model (top-k of E in the smaller workloads);
  * a self-conditioning input carrying the previous round's prediction.
The remaining architecture (pre-norm RMSNorm, rotate-half RoPE, SwiGLU
experts, tied LM head, logit scale) is the workload definition's.  Where
the pages are silent this oracle reads them so: no sqrt(d) embedding scale;
RoPE theta 10000 at absolute positions (prompt 0..P-1, canvas P..P+255);
RMSNorm eps 1e-6 with unit gains (random gains would scale the signal
away); the "logit scale" multiplies the final logits before temperature and
entropy; self-conditioning s = (softmax(l) E) W_sc^T with the tied embedding
E and a d x d W_sc (a linear V -> d map of about 7.8 M parameters at the
26B-A4B width, where a dense V x d matrix would hold 738 M), added to the
canvas token embeddings and zero at round 0; router softmax over the k
selected logits (plus a Zipf bias -s ln(e+1) when configured, in selection
and gates alike), ties to the lower expert id, slots in descending logit
order.

Arithmetic: float64 everywhere.  Values are rounded to the model's storage
dtype (bf16 round-to-nearest-even, or binary32) at the storage points of the
definition: the residual stream h, each RMSNorm output, q/k (after RoPE) and
v, the attention output, the SwiGLU activation, the softmax probabilities fed
to self-conditioning, and the self-conditioning vector and its intermediate.
Router logits and gate weights stay float64.  Expert outputs are summed in
slot order before the single rounding of h.

Weights: W = round(0.02 z), z = sqrt(-2 ln u1) cos(2 pi u2) (Box-Muller) with
u1, u2 the open-interval uniforms of words 0 and 1 of Philox4x32-10 keyed by
the weight seed, counter (index lo, index hi, tensor id, stream 3); every
linear weight is stored [out, in] and indexed row-major; expert tensors are
[E, out, in].  Norm gains are 1.
"""
from __future__ import annotations

import dataclasses
import numpy as np

from . import _native
from . import fp8 as f8
from . import numerics as nm
from . import sampler as sp

F32 = np.float32
CANVAS = 256
DTYPE_FP32 = 0
DTYPE_BF16 = 1

T_EMBED = 0
T_WSC = 1


def layer_tensor_id(layer: int, which: str) -> int:
    return 16 + 16 * layer + ("wq", "wk", "wv", "wo", "wr", "wg", "wu", "wd").index(which)


# --- weights --------------------------------------------------------------------
def _normal_weights(seed: int, tensor_id: int, start: int, count: int, bf16: bool) -> np.ndarray:
    j = np.arange(start, start + count, dtype=np.uint64)
    c0 = (j & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    c1 = (j >> np.uint64(32)).astype(np.uint32)
    k0, k1 = nm.seed_key(seed, 0)
    x0, x1, _, _ = nm.philox4x32_10(c0, c1, np.uint32(tensor_id), np.uint32(nm.STREAM_WEIGHTS), k0, k1)
    u1 = nm.uniform_open(x0)
    u2 = nm.uniform_open(x1)
    r = np.sqrt(nm.log_f32(u1) * F32(-2.0))
    z = r * nm.cos2pi_f32(u2)
    w = F32(0.02) * z
    return nm.round_bf16_from_f32(w) if bf16 else w.astype(F32)


def weight_values(seed: int, tensor_id: int, shape, bf16: bool) -> np.ndarray:
    """The whole tensor `tensor_id` (row-major `shape`) as float32 values
    (through the bit-identical C twin when it is built)."""
    n = int(np.prod(shape))
    if _native.lib() is not None:
        return _native.weights(seed, tensor_id, 0, n, bf16).reshape(shape)
    out = np.empty(n, dtype=F32)
    step = 1 << 15
    for s in range(0, n, step):
        c = min(step, n - s)
        out[s:s + c] = _normal_weights(seed, tensor_id, s, c, bf16)
    return out.reshape(shape)


def weight_element(seed: int, tensor_id: int, index: int, bf16: bool) -> float:
    """One weight by its row-major linear index (used by the one-by-one pins)."""
    return float(_normal_weights(seed, tensor_id, int(index), 1, bf16)[0])


@dataclasses.dataclass
class Layer:
    wq: np.ndarray
    wk: np.ndarray
    wv: np.ndarray
    wo: np.ndarray
    wr: np.ndarray
    wg: np.ndarray
    wu: np.ndarray
    wd: np.ndarray


class ExpertTensor:
    """An expert weight tensor [E, out, in] whose experts are generated one at
    a time on first use and kept (the per-layer checks of the large
    workloads touch a few experts of each layer).  Indexing by expert id
    gives the [out, in] matrix; FP8 workloads give the dequantised values."""

    def __init__(self, seed, tensor_id, shape, bf16, fp8=False):
        self.seed, self.tensor_id, self.shape, self.bf16, self.fp8 = seed, tensor_id, tuple(shape), bf16, fp8
        self._cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self._cache:
            _, o, i = self.shape
            n = o * i
            if _native.lib() is not None:
                w = _native.weights(self.seed, self.tensor_id, e * n, n, self.bf16)
            else:
                w = _normal_weights(self.seed, self.tensor_id, e * n, n, self.bf16)
            w = w.reshape(o, i)
            self._cache[e] = f8.quantize(w)[2] if self.fp8 else w
        return self._cache[e]


def layer_weights(cfg, l, lazy_experts=False) -> Layer:
    """Weights of layer l; with lazy_experts the expert tensors are
    ExpertTensor objects (generated per expert when first indexed)."""
    bf = cfg.dtype == DTYPE_BF16
    d, E, ff = cfg.d_model, cfg.n_experts, cfg.d_ff
    hq, hkv = cfg.n_heads * cfg.head_dim, cfg.n_kv_heads * cfg.head_dim
    s = cfg.weight_seed
    fp8 = bool(getattr(cfg, "expert_fp8", False))
    t = lambda w: layer_tensor_id(l, w)
    if lazy_experts:
        wg, wu, wd = (ExpertTensor(s, t("wg"), (E, ff, d), bf, fp8), ExpertTensor(s, t("wu"), (E, ff, d), bf, fp8),
                      ExpertTensor(s, t("wd"), (E, d, ff), bf, fp8))
    else:
        wg, wu, wd = (weight_values(s, t("wg"), (E, ff, d), bf), weight_values(s, t("wu"), (E, ff, d), bf),
                      weight_values(s, t("wd"), (E, d, ff), bf))
        if fp8:
            # FP8 expert weights: the GEMMs use the dequantised values q s
            # (exact in bf16), every other weight stays as generated
            wg, wu, wd = f8.quantize(wg)[2], f8.quantize(wu)[2], f8.quantize(wd)[2]
    return Layer(wq=weight_values(s, t("wq"), (hq, d), bf), wk=weight_values(s, t("wk"), (hkv, d), bf),
                 wv=weight_values(s, t("wv"), (hkv, d), bf), wo=weight_values(s, t("wo"), (d, hq), bf),
                 wr=weight_values(s, t("wr"), (E, d), bf), wg=wg, wu=wu, wd=wd)


class Model:
    """Weights of one workload (float32 arrays holding the stored values).
    `layers` limits how many layers are generated; with_embed=False skips the
    embedding and W_sc (for checks of single layers)."""

    def __init__(self, cfg, layers=None, with_embed=True):
        self.cfg = cfg
        bf = cfg.dtype == DTYPE_BF16
        d, V = cfg.d_model, cfg.vocab
        s = cfg.weight_seed
        self.embed = weight_values(s, T_EMBED, (V, d), bf) if with_embed else None
        self.wsc = weight_values(s, T_WSC, (d, d), bf) if with_embed else None
        # optional per-token router bias of the canvas pass, [L, 256 * canvases, E]
        # (a workload input that structures routing, standing in for the expert
        # locality of a trained router -- about 84 of 128 experts per round in
        # the explainer's section 五; None = no such term)
        self.route_bias = None
        self.layers = [layer_weights(cfg, l) for l in range(cfg.n_layers if layers is None else layers)]

    def store(self, x):
        """Round float64 values to the storage dtype (returned as float64)."""
        if self.cfg.dtype == DTYPE_BF16:
            return nm.round_bf16(x).astype(np.float64)
        return np.asarray(x, dtype=np.float64).astype(F32).astype(np.float64)


# --- building blocks --------------------------------------------------------------
def rmsnorm(h, eps):
    """x / sqrt(mean(x^2) + eps) (unit gain)."""
    h = np.asarray(h, dtype=np.float64)
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def rope(x, positions, theta):
    """Rotate-half RoPE on the last axis (head_dim): pair (i, i + hd/2) turns by
    angle pos * theta^(-2i/hd).  x: [..., n_pos, heads, hd]."""
    hd = x.shape[-1]
    half = hd // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / hd)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv[None, :]      # [n, half]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def attention(q, k, v, causal_offset=None):
    """softmax(q k^T / sqrt(hd)) v per head, float64.

    q: [nq, Hq, hd]; k, v: [nk, Hkv, hd]; query head h reads kv head
    h // (Hq/Hkv).  causal_offset=None: every query sees every key (canvas,
    bidirectional).  Otherwise query i sees keys j <= i + causal_offset
    (prompt encode, causal).
    """
    nq, hq, hd = q.shape
    nk, hkv, _ = k.shape
    g = hq // hkv
    out = np.empty((nq, hq, hd))
    for h in range(hq):
        kh, vh = k[:, h // g, :], v[:, h // g, :]
        s = (q[:, h, :] @ kh.T) / np.sqrt(hd)
        if causal_offset is not None:
            mask = np.arange(nk)[None, :] > (np.arange(nq)[:, None] + causal_offset)
            s = np.where(mask, -np.inf, s)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ vh
    return out


def router(x, wr, top_k, zipf_s=0.0, extra=None):
    """Top-k gating.  r = x Wr^T (+ b_e = -s ln(e+1)) (+ extra[t, e], a per-token
    bias given as input); the k largest logits (ties to the lower expert id) in
    descending order; gate weights are the softmax over those k logits, so they
    sum to 1.  Returns (ids [n,k] int32, weights [n,k] float64)."""
    r = router_logits(x, wr, zipf_s, extra)
    n, E = r.shape
    ids = np.empty((n, top_k), dtype=np.int32)
    w = np.empty((n, top_k))
    for t in range(n):
        order = sorted(range(E), key=lambda e: (-r[t, e], e))[:top_k]
        ids[t] = order
        sel = r[t, order]
        ex = np.exp(sel - sel.max())
        w[t] = ex / ex.sum()
    return ids, w


def silu(z):
    return z / (1.0 + np.exp(-z))


def moe(model, layer, x, extra=None):
    """sum over the k slots (in slot order) of gate_weight * expert FFN, with
    expert FFN(x) = (silu(x Wg^T) * (x Wu^T)) Wd^T and the SwiGLU activation
    rounded to the storage dtype.  `extra`: per-token router bias or None."""
    cfg = model.cfg
    ids, w = router(x, layer.wr, cfg.top_k, cfg.zipf_s, extra)
    y = np.zeros_like(x)
    for j in range(cfg.top_k):
        for e in np.unique(ids[:, j]):
            rows = np.nonzero(ids[:, j] == e)[0]
            xe = x[rows]
            a = model.store(silu(xe @ layer.wg[e].astype(np.float64).T) * (xe @ layer.wu[e].astype(np.float64).T))
            y[rows] += w[rows, j:j + 1] * (a @ layer.wd[e].astype(np.float64).T)
    return y, ids, w


def _proj(x, w):
    return x @ np.asarray(w, dtype=np.float64).T


def router_margin(x, wr, top_k, zipf_s=0.0, extra=None):
    """Gap between the k-th and (k+1)-th largest router logit per token (how
    close the top-k decision is to a tie; +inf when k = E).  Diagnostic only."""
    r = router_logits(x, wr, zipf_s, extra)
    if top_k >= r.shape[1]:
        return np.full(r.shape[0], np.inf)
    s = -np.sort(-r, axis=1)
    return s[:, top_k - 1] - s[:, top_k]


def routing_alternatives(r_row, top_k, delta):
    """Every top-k selection that is correct within `delta` of rounding.

    r_row: router logits of one token (bias included).  The primary selection
    is the k largest (ties to the lower id).  When the decision boundary is
    within delta -- a selected expert whose logit is less than delta above the
    best unselected one -- swapping that pair gives another selection that
    rounding of the inputs can legitimately produce.  Returns a list of
    (ids, gate weights) with the primary first; ids in descending-logit slot
    order, gate weights the softmax over the selected logits."""
    r = np.asarray(r_row, dtype=np.float64)
    E = r.size
    order = sorted(range(E), key=lambda e: (-r[e], e))
    sel, rest = order[:top_k], order[top_k:]
    sets = [sel]
    if rest:
        best_out = r[rest[0]]
        worst_in = r[sel[-1]]
        c_in = [e for e in sel if r[e] - best_out < delta]
        c_out = [e for e in rest if worst_in - r[e] < delta]
        for a in c_in:
            for b in c_out:
                alt = [e for e in sel if e != a] + [b]
                sets.append(sorted(alt, key=lambda e: (-r[e], e)))
    out = []
    for s in sets:
        v = r[s]
        ex = np.exp(v - v.max())
        out.append((np.array(s, dtype=np.int32), ex / ex.sum()))
    return out


def token_logits_with_routing(model, layer, h_attn_row, ids, gates):
    """Logits of one token of a single-layer model whose MoE uses the given
    selection: h = store(h_attn + sum_j g_j FFN_{e_j}(x)), x = store(RMSNorm(h_attn)),
    logits = logit_scale * store(RMSNorm(h)) E^T.  Diagnostic / parity helper."""
    cfg = model.cfg
    h = np.asarray(h_attn_row, dtype=np.float64)[None, :]
    x = model.store(rmsnorm(h, cfg.rms_eps))
    y = np.zeros_like(h)
    for e, g in zip(ids, gates):
        a = model.store(silu(x @ layer.wg[e].astype(np.float64).T) * (x @ layer.wu[e].astype(np.float64).T))
        y += g * (a @ layer.wd[e].astype(np.float64).T)
    h = model.store(h + y)
    xf = model.store(rmsnorm(h, cfg.rms_eps))
    return (cfg.logit_scale * _proj(xf, model.embed))[0]


def router_logits(x, wr, zipf_s=0.0, extra=None):
    """Router logits x Wr^T (+ Zipf bias) (+ per-token bias `extra` [n, E]), float64."""
    r = np.asarray(x, dtype=np.float64) @ np.asarray(wr, dtype=np.float64).T
    if zipf_s:
        r = r + (-zipf_s * np.log(np.arange(wr.shape[0], dtype=np.float64) + 1.0))[None, :]
    if extra is not None:
        r = r + np.asarray(extra, dtype=np.float64)
    return r


def block(model, layer, h, positions, k_prefix, v_prefix, causal, trace=None, route_bias=None):
    """One pre-norm transformer block over n tokens.  k_prefix/v_prefix are
    cached keys/values [n_prefix, Hkv, hd] the tokens also attend to.  Returns
    (h_out, k_new, v_new) with k_new/v_new the stored keys/values of the tokens.
    `trace` (a list) receives the intermediate states for diagnostics;
    `route_bias` [n, E] is added to the router logits (None: no term)."""
    cfg = model.cfg
    n = h.shape[0]
    hq, hkv, hd = cfg.n_heads, cfg.n_kv_heads, cfg.head_dim
    x = model.store(rmsnorm(h, cfg.rms_eps))
    q = model.store(rope(_proj(x, layer.wq).reshape(n, hq, hd), positions, cfg.rope_theta))
    k = model.store(rope(_proj(x, layer.wk).reshape(n, hkv, hd), positions, cfg.rope_theta))
    v = model.store(_proj(x, layer.wv).reshape(n, hkv, hd))
    kk = np.concatenate([k_prefix, k], axis=0)
    vv = np.concatenate([v_prefix, v], axis=0)
    o = model.store(attention(q, kk, vv, causal_offset=k_prefix.shape[0] if causal else None))
    h = model.store(h + _proj(o.reshape(n, hq * hd), layer.wo))
    x2 = model.store(rmsnorm(h, cfg.rms_eps))
    y, ids, w = moe(model, layer, x2, route_bias)
    if trace is not None:
        trace.append(dict(h_attn=h.copy(), ids=ids,
                          margin=router_margin(x2, layer.wr, cfg.top_k, cfg.zipf_s, route_bias),
                          router=router_logits(x2, layer.wr, cfg.zipf_s, route_bias)))
    h = model.store(h + y)
    if trace is not None:
        trace[-1]["h_out"] = h.copy()
    return h, k, v


# --- prompt encode (causal) ------------------------------------------------------
def encode_prompt(model, prompt):
    """Causal encode of one prompt [P] into its KV cache.  Returns (K, V), each
    [L, Hkv, P, hd] float32 (values in the storage dtype)."""
    cfg = model.cfg
    P = len(prompt)
    h = model.embed[np.asarray(prompt)].astype(np.float64)
    empty = np.zeros((0, cfg.n_kv_heads, cfg.head_dim))
    K, Vv = [], []
    for layer in model.layers:
        h, k, v = block(model, layer, h, np.arange(P), empty, empty, causal=True)
        K.append(k.transpose(1, 0, 2))
        Vv.append(v.transpose(1, 0, 2))
    return np.stack(K).astype(F32), np.stack(Vv).astype(F32)


# --- one denoising step ----------------------------------------------------------
def forward_canvas(model, K, V, canvas, selfcond, trace=None, canvas_id=0):
    """Bidirectional canvas pass.  K, V: prompt cache [L, Hkv, P, hd];
    canvas [256] ids; selfcond [256, d] or None.  Returns float64 logits
    [256, vocab] and the canvas keys/values written per layer.  A per-token
    router bias (model.route_bias) applies its rows of canvas `canvas_id`."""
    cfg = model.cfg
    P = K.shape[2]
    h = model.embed[np.asarray(canvas)].astype(np.float64)
    if selfcond is not None:
        h = model.store(h + np.asarray(selfcond, dtype=np.float64))
    pos = P + np.arange(CANVAS)
    kv_new = []
    for l, layer in enumerate(model.layers):
        kp = K[l].transpose(1, 0, 2).astype(np.float64)
        vp = V[l].transpose(1, 0, 2).astype(np.float64)
        rb = getattr(model, "route_bias", None)
        if rb is not None:
            rb = rb[l, canvas_id * CANVAS:(canvas_id + 1) * CANVAS]
        h, k, v = block(model, layer, h, pos, kp, vp, causal=False, trace=trace, route_bias=rb)
        kv_new.append((k, v))
    x = model.store(rmsnorm(h, cfg.rms_eps))
    if trace is not None:
        trace.append(dict(x_final=x.copy()))
    logits = cfg.logit_scale * _proj(x, model.embed)
    return logits, kv_new


def self_condition(model, probs):
    """Next round's self-conditioning vector s = (p E) W_sc^T from the binary32
    untempered probabilities p [256, V]; p, p E and s are stored values."""
    p = model.store(np.asarray(probs, dtype=np.float64))
    u = model.store(p @ model.embed.astype(np.float64))
    return model.store(_proj(u, model.wsc))


def self_condition_topk(model, ids, weights):
    """self_condition for a top-k-truncated distribution: p is zero outside
    the candidates ids [256, K] and holds the binary32 weights [256, K] on
    them, so p E is the weighted sum of K embedding rows per position."""
    p = model.store(np.asarray(weights, dtype=np.float64))
    n, K = p.shape
    u = np.zeros((n, model.cfg.d_model))
    for j in range(K):
        u += p[:, j:j + 1] * model.embed[np.asarray(ids)[:, j]].astype(np.float64)
    u = model.store(u)
    return model.store(_proj(u, model.wsc))


def denoise_step(model, K, V, canvas, selfcond, step, t, canvas_id=0, prev_amax=None, max_steps=None,
                 trace=None):
    """One round for one canvas.  Returns a dict with logits (float64 and the
    binary32 values the sampler reads), entropy, sampled tokens, argmax,
    commit mask, next canvas, next self-conditioning, stop flag and count."""
    cfg = model.cfg
    logits64, _ = forward_canvas(model, K, V, canvas, selfcond, trace=trace, canvas_id=canvas_id)
    l32 = logits64.astype(F32)
    T = sp.temperature(t, cfg.temp_start, cfg.temp_end)
    inv_t = F32(1.0) / T
    K = getattr(cfg, "sample_topk", 0)
    if K:
        st = sp.sampler_rows_topk(l32, K, inv_t, cfg.sample_seed, canvas_id, step)
    else:
        st = sp.sampler_rows(l32, inv_t, cfg.sample_seed, canvas_id, step)
    tok = st["tokens"]
    mask = sp.commit_mask(st["H"], cfg.commit_mode, cfg.commit_bound)
    nxt = sp.next_canvas(tok, mask, cfg.sample_seed, canvas_id, step, cfg.vocab)
    n_steps = cfg.max_steps if max_steps is None else max_steps
    stop = sp.stop_decision(st["H"], mask, st["amax"], prev_amax, step, n_steps,
                            cfg.stop_mode, cfg.stop_bound)
    s_next = self_condition_topk(model, st["cand_ids"], st["cand_w"]) if K else self_condition(model, st["p"])
    return dict(logits64=logits64, logits=l32, H=st["H"], tokens=tok, amax=st["amax"],
                commit=mask, canvas_next=nxt, selfcond_next=s_next, stop=stop,
                n_committed=int(mask.sum()), probs=st.get("p"), cand_ids=st.get("cand_ids"),
                cand_w=st.get("cand_w"))


def generate_block(model, K, V, canvas_id=0, max_steps=None):
    """Full block: uniform-noise canvas, rounds until the stop rule fires (or
    the budget ends).  Returns dict(canvas = sampled tokens of the stopping
    round, steps_used, n_committed, trace = per-round results)."""
    cfg = model.cfg
    n = cfg.max_steps if max_steps is None else max_steps
    canvas = sp.initial_canvas(cfg.sample_seed, canvas_id, CANVAS, cfg.vocab)
    selfcond, prev_amax, trace = None, None, []
    for s in range(n):
        t = sp.schedule_t(s, n)
        r = denoise_step(model, K, V, canvas, selfcond, s, t, canvas_id, prev_amax, n)
        trace.append(r)
        if r["stop"] or s == n - 1:
            return dict(canvas=r["tokens"], steps_used=s + 1, n_committed=r["n_committed"], trace=trace)
        canvas, selfcond, prev_amax = r["canvas_next"], r["selfcond_next"], r["amax"]
    raise AssertionError("unreachable")


def generate(model, prompt, n_blocks, canvas_id=0):
    """Block-autoregressive generation: canvases are produced one after another
    (release news "不是逐词写，而是整块去噪"; "谷歌都下场了：扩散语言模型的四倍速与六倍错"
    section 一: a finished canvas joins the context, then the next canvas
    starts).  Block i is generated against the causal KV of [prompt ; blocks
    0..i-1] (its canvas at positions P + 256 i) and samples with seed
    sample_seed + i.  Returns the list of generate_block results."""
    import copy
    context = [int(x) for x in prompt]
    blocks = []
    for i in range(n_blocks):
        K, V = encode_prompt(model, context)
        mi = copy.copy(model)
        mi.cfg = model.cfg.replace(sample_seed=model.cfg.sample_seed + i)
        ref = generate_block(mi, K, V, canvas_id)
        blocks.append(ref)
        context += [int(x) for x in ref["canvas"]]
    return blocks
