"""Oracle of the entropy-bounded sampler (per-position statistics, Gumbel-max
sampling at a linearly annealed temperature, commit / re-noise, adaptive stop).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
bench's CPU-baseline leg; shares no code with the CUDA path.

Method, as the DiffusionGemma technical-report explainer (mlqm.cn) states it in
its section 四 (the sampler):
  * each canvas position gets an entropy -- the model's uncertainty there;
  * positions are sorted by entropy, the most certain graduate first until the
    running entropy sum passes 0.1; the rest are re-randomised to fresh
    uniform tokens (multinomial noise, section 一) and revisited next round;
  * the temperature falls linearly from 0.8 to 0.4 over the rounds;
  * the loop stops once two rounds in a row barely change: mean entropy below
    0.005 and an identical most-likely token sequence; 48 rounds at most.
The workload definitions instead fix a simpler default rule: commit where the
entropy is below 0.5 nats, stop when every position is committed or the mean
entropy is below 0.1.  Both are implemented; `commit_mode` / `stop_mode`
choose.

Decision precision.  Tokens and commit masks are integers decided from
floating point, so they are taken in binary32 with the fixed op sequences of
`oracle.numerics` (own log/exp), and entropy sums are accumulated exactly in
64-bit fixed point.  `entropy_f64` is the plain definition the decision-
precision value is pinned against.
"""
from __future__ import annotations

import numpy as np

from . import numerics as nm

F32 = np.float32
FIX_S = F32(2.0 ** 40)      # fixed-point scale of the per-row softmax sums
FIX_H = F32(2.0 ** 32)      # fixed-point scale of per-position entropies


# --- temperature schedule (explainer section 四: 0.8 -> 0.4, linear) ---------
def schedule_t(step: int, n_steps: int) -> np.float32:
    """Diffusion time of round `step` of `n_steps`: 1 at the first round,
    0 at the last, linear in between: t = 1 - s/(N-1) in binary32."""
    if n_steps <= 1:
        return F32(1.0)
    return F32(1.0) - F32(step) / F32(n_steps - 1)


def temperature(t, temp_start=0.8, temp_end=0.4) -> np.float32:
    """T(t) = T_end + (T_start - T_end) t in binary32, so T(1) = T_start and
    T(0) = T_end exactly."""
    ts, te = F32(temp_start), F32(temp_end)
    return te + (ts - te) * F32(t)


# --- per-row statistics ----------------------------------------------------------
def entropy_f64(logits) -> np.ndarray:
    """Definition: H = -sum_v p_v ln p_v with p = softmax(l), in float64 (nats)."""
    l = np.asarray(logits, dtype=np.float64)
    l = l - l.max(axis=-1, keepdims=True)
    p = np.exp(l)
    p /= p.sum(axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(p > 0, p * np.log(p), 0.0)
    return -t.sum(axis=-1)


def _row_terms(d):
    e = nm.exp_f32(d)
    sq = (e * FIX_S).astype(np.int64)
    uq = ((e * d) * FIX_S).astype(np.int64)
    return e, sq, uq


def row_stats(logits, want_probs: bool = False, chunk: int = 1 << 15):
    """Per-row statistics of binary32 logits [R, V] in decision precision.

    m = max_v l_v;  e_v = exp(l_v - m) (own binary32 exp);
    S = sum_v e_v and U = sum_v e_v (l_v - m), each term truncated to 2^-40
    and summed exactly in int64;  H = ln(S) - U/S in binary32 (own log), which
    is -sum p ln p with p = e/S.  amax = argmax_v l_v (lowest index on ties).
    With want_probs, also p_v = e_v * (1/S) in binary32 (the untempered
    distribution fed to self-conditioning).
    Returns dict(m, S_q, U_q, H, amax[, p]).
    """
    l = np.ascontiguousarray(logits, dtype=F32)
    R, V = l.shape
    m = l.max(axis=1)
    amax = l.argmax(axis=1).astype(np.int32)
    Sq = np.zeros(R, dtype=np.int64)
    Uq = np.zeros(R, dtype=np.int64)
    P = np.empty_like(l) if want_probs else None
    for r in range(R):
        for c0 in range(0, V, chunk):
            d = l[r, c0:c0 + chunk] - m[r]
            e, sq, uq = _row_terms(d)
            Sq[r] += int(sq.sum())
            Uq[r] += int(uq.sum())
            if want_probs:
                P[r, c0:c0 + chunk] = e
    Sf = Sq.astype(F32)
    Uf = Uq.astype(F32)
    H = nm.log_f32(Sf * F32(2.0 ** -40)) - Uf / Sf
    out = dict(m=m, S_q=Sq, U_q=Uq, H=H.astype(F32), amax=amax)
    if want_probs:
        inv_s = F32(1.0) / (Sf * F32(2.0 ** -40))
        for r in range(R):
            P[r] = nm.chunked(lambda e: e * inv_s[r], P[r])
        out["p"] = P
    return out


# --- Gumbel-max sampling ---------------------------------------------------------
def gumbel_noise(seed: int, canvas_id: int, position: int, step: int, vocab: int) -> np.ndarray:
    """g_v = -ln(-ln u_v), u_v from Philox(key(seed, canvas), ctr = (v>>2,
    position, step, stream 0)) word v&3, in binary32 (own log)."""
    k0, k1 = nm.seed_key(seed, canvas_id)
    v4 = np.arange(vocab // 4, dtype=np.uint32)
    w = nm.philox4x32_10(v4, np.uint32(position), np.uint32(step), np.uint32(nm.STREAM_GUMBEL), k0, k1)
    words = np.stack(w, axis=1).reshape(-1)[:vocab]
    u = nm.uniform_open(words)
    return nm.chunked(lambda x: -nm.log_f32(-nm.log_f32(x)), u)


def gumbel_argmax(logits_row, inv_t, seed, canvas_id, position, step) -> int:
    """Sampled token = argmax_v (l_v * (1/T) + g_v), lowest index on ties
    (Gumbel-max trick: an exact draw from softmax(l/T))."""
    l = np.asarray(logits_row, dtype=F32)
    g = gumbel_noise(seed, canvas_id, position, step, l.size)
    key = nm.chunked(lambda a, b: a * F32(inv_t) + b, l, g)
    return int(np.argmax(key))


def sample_tokens(logits, inv_t, seed, canvas_id, step):
    """Sampled tokens of one canvas's rows [256, V] (row index = position)."""
    return np.array([gumbel_argmax(logits[i], inv_t, seed, canvas_id, i, step)
                     for i in range(logits.shape[0])], dtype=np.int32)


def renoise_tokens(seed, canvas_id, step, n_pos, vocab, stream=nm.STREAM_RENOISE):
    """Fresh uniform tokens for positions 0..n_pos-1 at a round (Philox word 0 of
    ctr = (0, position, step, stream))."""
    k0, k1 = nm.seed_key(seed, canvas_id)
    pos = np.arange(n_pos, dtype=np.uint32)
    w0, _, _, _ = nm.philox4x32_10(np.uint32(0), pos, np.uint32(step), np.uint32(stream), k0, k1)
    return nm.token_from_word(w0, vocab)


def initial_canvas(seed, canvas_id, n_pos, vocab):
    """Uniform-noise starting canvas (explainer section 一: start from 256 random
    tokens), Philox stream 2 at round 0."""
    return renoise_tokens(seed, canvas_id, 0, n_pos, vocab, stream=nm.STREAM_INIT_CANVAS)


def sampler_rows(logits, inv_t, seed, canvas_id, step):
    """row_stats (with probabilities) + sampled tokens for one canvas's rows
    (row i = position i), through the bit-identical C twin when it is built."""
    from . import _native
    if _native.lib() is not None:
        return _native.sampler_rows(logits, seed, canvas_id, 0, step, inv_t, True)
    st = row_stats(logits, want_probs=True)
    st["tokens"] = sample_tokens(logits, inv_t, seed, canvas_id, step)
    return st


# --- top-k-truncated sampling (explainer section 九) ---------------------------
# The explainer names top-k truncation as the sampler optimisation for large
# batches that the release lacks.  Reading: with truncation K, the token is the
# Gumbel-max draw restricted to the K largest logits (a draw from softmax(l/T)
# renormalised over them), each candidate keeping the noise g_v it has in the
# exact sampler; the self-conditioning input is the untempered distribution
# renormalised over the same candidates; entropy, argmax and the commit / stop
# decisions stay those of the full distribution.
def topk_ids(logits_row, K: int) -> np.ndarray:
    """Indices of the K largest binary32 logits of a row, by value descending,
    ties to the lower index (every index when K >= V)."""
    l = np.asarray(logits_row, dtype=F32)
    order = np.lexsort((np.arange(l.size), -l.astype(np.float64)))
    return order[:K].astype(np.int32)


def gumbel_noise_at(ids, seed: int, canvas_id: int, position: int, step: int) -> np.ndarray:
    """g_v of gumbel_noise at the given vocabulary ids only (same Philox
    counter (v>>2, position, step, stream 0) and word v&3)."""
    k0, k1 = nm.seed_key(seed, canvas_id)
    ids = np.asarray(ids, dtype=np.uint32)
    w = nm.philox4x32_10(ids >> np.uint32(2), np.uint32(position), np.uint32(step),
                         np.uint32(nm.STREAM_GUMBEL), k0, k1)
    words = np.stack(w, axis=1)[np.arange(ids.size), (ids & np.uint32(3)).astype(np.int64)]
    u = nm.uniform_open(words)
    return -nm.log_f32(-nm.log_f32(u))


def topk_sample(logits_row, K: int, inv_t, seed: int, canvas_id: int, position: int, step: int):
    """Top-k-truncated draw of one row.  Returns (token, ids, weights):
    ids = topk_ids(l, K); token = the id of the largest key l_v (1/T) + g_v
    among them (binary32, the lowest id on equal keys); weights = the
    untempered probabilities renormalised over the candidates, binary32:
    e_j = exp(l_j - m) (own exp, m the row maximum), s = e_0 + e_1 + ...
    accumulated in candidate order, w_j = e_j (1/s)."""
    l = np.asarray(logits_row, dtype=F32)
    ids = topk_ids(l, K)
    lc = l[ids]
    key = lc * F32(inv_t) + gumbel_noise_at(ids, seed, canvas_id, position, step)
    token = int(ids[key == key.max()].min())
    e = nm.exp_f32(lc - lc[0])
    s = F32(0.0)
    for x in e:
        s = F32(s + x)
    w = (e * (F32(1.0) / s)).astype(F32)
    return token, ids, w


def sampler_rows_topk(logits, K: int, inv_t, seed, canvas_id, step):
    """sampler_rows with top-k-truncated tokens: the full-distribution
    statistics (H, amax, S, U) plus tokens, candidate ids [R, K] and
    candidate weights [R, K] (no dense probabilities)."""
    st = sampler_rows(logits, inv_t, seed, canvas_id, step)
    st.pop("p", None)
    R = logits.shape[0]
    toks = np.empty(R, dtype=np.int32)
    ids, ws = [], []
    for i in range(R):
        toks[i], c, w = topk_sample(logits[i], K, inv_t, seed, canvas_id, i, step)
        ids.append(c)
        ws.append(w)
    st["tokens"] = toks
    st["cand_ids"] = np.stack(ids)
    st["cand_w"] = np.stack(ws)
    return st


# --- commit / re-noise / stop (explainer section 四) -----------------------------
def fixed_entropy(H) -> np.ndarray:
    """Per-position entropy in Q32 fixed point: trunc(H * 2^32) (exact
    binary32 scaling), so sums are exact in any order."""
    return (np.asarray(H, dtype=F32) * FIX_H).astype(np.int64)


def bound_fixed(bound) -> int:
    return int((np.asarray([bound], dtype=F32) * FIX_H).astype(np.int64)[0])


def commit_mask(H, commit_mode: int, commit_bound: float) -> np.ndarray:
    """Positions that graduate this round (uint8 [n_pos]).

    threshold mode: H_i < bound, compared in binary32.
    entropy-bounded mode: sort positions by (H_i, i) ascending and commit the
    longest prefix whose Q32 entropy sum stays <= bound; at least one
    position always commits (the most certain one).
    """
    H = np.asarray(H, dtype=F32)
    if commit_mode == 0:
        return (H < F32(commit_bound)).astype(np.uint8)
    hq = fixed_entropy(H)
    order = sorted(range(H.size), key=lambda i: (int(hq[i]), i))
    lim = bound_fixed(commit_bound)
    mask = np.zeros(H.size, dtype=np.uint8)
    acc = 0
    for n, i in enumerate(order):
        acc += int(hq[i])
        if n > 0 and acc > lim:
            break
        mask[i] = 1
    return mask


def stop_decision(H, mask, amax, prev_amax, step, max_steps, stop_mode, stop_bound) -> bool:
    """Adaptive stop of one canvas after round `step`.

    mean mode: every position committed, or mean entropy < bound.
    entropy-bounded mode: mean entropy < bound and the argmax sequence equals
    the previous round's (so never at round 0).
    The last round of the budget always stops.  Means compare Q32 sums:
    sum_i trunc(H_i 2^32) < n_pos * trunc(bound 2^32).
    """
    hq = fixed_entropy(H)
    n = hq.size
    low = int(hq.sum()) < n * bound_fixed(stop_bound)
    if step >= max_steps - 1:
        return True
    if stop_mode == 0:
        return bool(mask.all()) or low
    if step == 0 or prev_amax is None:
        return False
    return low and bool(np.array_equal(np.asarray(amax), np.asarray(prev_amax)))


def next_canvas(tokens, mask, seed, canvas_id, step, vocab):
    """Committed positions keep the sampled token; the others are re-noised to
    fresh uniform tokens (multinomial diffusion, explainer section 一)."""
    fresh = renoise_tokens(seed, canvas_id, step, tokens.size, vocab)
    return np.where(np.asarray(mask) != 0, tokens, fresh).astype(np.int32)
