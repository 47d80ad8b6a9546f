"""Python binding of the B200 block-text-diffusion denoising library.

Argument marshalling only: every step of the path runs in the CUDA kernels of
libdg.so (built in-tree by `block_text_diffusion_b200.build`).  PyTorch
provides device memory and streams; tensors are passed by data pointer.
There is no fallback: if the library is missing or no GPU is present the
calls raise.
"""
from __future__ import annotations

import ctypes
import os

from . import inputs  # noqa: F401  (seeded synthetic inputs)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")
_lib = None

DG_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "out of device memory", 3: "CUDA error",
          4: "device wait timed out", 5: "invalid state or device-side index error", 6: "unsupported"}


class DGError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} (status {code})")


class Config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("logit_scale", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("rms_eps", ctypes.c_float), ("zipf_s", ctypes.c_float), ("temp_start", ctypes.c_float),
                ("temp_end", ctypes.c_float), ("max_steps", ctypes.c_int32), ("commit_mode", ctypes.c_int32),
                ("commit_bound", ctypes.c_float), ("stop_mode", ctypes.c_int32), ("stop_bound", ctypes.c_float),
                ("canvas_len", ctypes.c_int32), ("max_canvases", ctypes.c_int32), ("max_prompt", ctypes.c_int32),
                ("sample_seed", ctypes.c_uint64), ("sample_topk", ctypes.c_int32), ("expert_fp8", ctypes.c_int32)]


class StepOut(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("entropy", ctypes.c_void_p), ("tokens", ctypes.c_void_p),
                ("argmax", ctypes.c_void_p), ("commit", ctypes.c_void_p), ("canvas_next", ctypes.c_void_p),
                ("selfcond_next", ctypes.c_void_p), ("stop", ctypes.c_void_p), ("n_committed", ctypes.c_void_p)]


def lib():
    """Load libdg.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m block_text_diffusion_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, U64, F, U32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                    ctypes.c_float, ctypes.c_uint32)
        sig = {
            "dg_init_weights": ([ctypes.POINTER(Config), U64, P, ctypes.POINTER(P)], I32),
            "dg_free": ([P], I32),
            "dg_kv_bytes": ([P, I32, I32], ctypes.c_size_t),
            "dg_encode_prompt": ([P, P, I32, I32, P, P], I32),
            "dg_denoise_step": ([P, P, I32, I32, P, P, I32, F, ctypes.POINTER(StepOut), P], I32),
            "dg_generate_block": ([P, P, I32, I32, P, P, P, P], I32),
            "dg_generate": ([P, P, I32, I32, I32, P, P, P, P, P], I32),
            "dg_sync_status": ([P, P], I32),
            "dg_status_string": ([I32], ctypes.c_char_p),
            "dg_kernels_per_step": ([P, I32, I32], I32),
            "dg_test_math": ([I32, P, P, I64, U64, U32, P], I32),
            "dg_test_philox": ([P, P, I64, P], I32),
            "dg_test_sampler": ([P, I32, I32, I32, U64, I32, F, F, F, P, P, P, P, P, P, I32, P], I32),
            "dg_test_sampler_topk": ([P, I32, I32, I32, U64, I32, F, F, F, I32, P, P, P, P, P, P, P, I32, P], I32),
            "dg_test_sc_gather": ([P, P, I32, I32, P, I32, I32, P, P], I32),
            "dg_test_quant_fp8": ([P, I64, I32, P, P, P], I32),
            "dg_test_attn_plan": ([I64, I32, I32, I32, I32, I64, I64, P], I32),
            "dg_test_grouped_gemm_fp8": ([P, P, P, P, I32, I32, I32, I32, I32, P, P], I32),
            "dg_test_commit": ([P, P, P, P, I32, I32, U64, I32, I32, I32, F, I32, F, P, P, P, P, P], I32),
            "dg_test_gemm": ([P, P, P, I32, I32, I32, I32, F, I32, I32, I32, P], I32),
            "dg_test_grouped_gemm": ([P, P, P, I32, I32, I32, I32, I32, I32, P, P], I32),
            "dg_test_router": ([P, P, P, P, I32, I32, I32, I32, P, P, P], I32),
            "dg_set_routing_bias": ([P, P, I32], I32),
            "dg_test_attention": ([P, P, P, I32, I32, I32, I32, I32, I32, I32, I32, I32, I32, P, P, P], I32),
            "dg_read_weight": ([P, I32, P, P], I32),
            "dg_load_kv": ([P, P, I32, I32, P, P, P], I32),
            "dg_profile_step": ([P, P, I32, I32, I32, P, P, I32, P], I32),
            "dg_phase_name": ([I32], ctypes.c_char_p),
            "dg_launches_per_round": ([P], I32),
            "dg_expert_counts": ([P, P, P], I32),
            "dg_debug_trace": ([P, P, P], I32),
            "dg_test_layer": ([P, P, I32, I32, I32, P, P, P, P], I32),
            "dg_test_moe": ([P, I32, I32, P, P, P, P], I32),
            "dg_test_attn_capacity": ([P], I32),
            "dg_test_launch_shape": ([I32, I64, I32, I32, P], I32),
            "dg_touched_experts_sum": ([P, P, I32, P], I32),
            "dg_gemm_splitk_noalloc": ([P, P, P, I32, I32, I32, I32, P], I32),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _check(code, where):
    if code != DG_OK:
        raise DGError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_config(w, max_canvases=None, max_prompt=None) -> Config:
    """dg_config of a workload description (block_text_diffusion_b200.inputs.Workload)."""
    return Config(w.n_layers, w.d_model, w.n_heads, w.n_kv_heads, w.head_dim, w.n_experts, w.top_k, w.d_ff,
                  w.vocab, w.dtype, w.logit_scale, w.rope_theta, w.rms_eps, w.zipf_s, w.temp_start, w.temp_end,
                  w.max_steps, w.commit_mode, w.commit_bound, w.stop_mode, w.stop_bound, 256,
                  max_canvases or w.batch, max_prompt or w.prompt_len, w.sample_seed, w.sample_topk,
                  int(w.expert_fp8))


class Model:
    """A dg_model: weights generated on the device from the weight seed."""

    def __init__(self, workload, max_canvases=None, max_prompt=None, stream=None):
        import torch
        self.w = workload
        self.cfg = make_config(workload, max_canvases, max_prompt)
        self.dtype = torch.bfloat16 if workload.dtype == inputs.DTYPE_BF16 else torch.float32
        h = ctypes.c_void_p()
        _check(lib().dg_init_weights(ctypes.byref(self.cfg), workload.weight_seed, _stream(stream),
                                     ctypes.byref(h)), "dg_init_weights")
        self.h = h

    def close(self):
        if self.h:
            lib().dg_free(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- main API ------------------------------------------------------------------
    def kv_bytes(self, B, P):
        return int(lib().dg_kv_bytes(self.h, B, P))

    def new_kv(self, B, P):
        import torch
        n = self.kv_bytes(B, P)
        if n == 0:
            raise DGError(1, "dg_kv_bytes")
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    def encode_prompt(self, prompt, kv, stream=None):
        B, P = prompt.shape
        _check(lib().dg_encode_prompt(self.h, _ptr(prompt), B, P, _ptr(kv), _stream(stream)), "dg_encode_prompt")

    def denoise_step(self, kv, P, canvas, selfcond, step, t, out: dict, stream=None):
        B = canvas.shape[0]
        so = StepOut(*[_ptr(out.get(k)) for k in ("logits", "entropy", "tokens", "argmax", "commit",
                                                  "canvas_next", "selfcond_next", "stop", "n_committed")])
        _check(lib().dg_denoise_step(self.h, _ptr(kv), B, P, _ptr(canvas), _ptr(selfcond), step, float(t),
                                     ctypes.byref(so), _stream(stream)), "dg_denoise_step")

    def generate_block(self, kv, B, P, canvas_out, steps_used, n_committed, stream=None):
        _check(lib().dg_generate_block(self.h, _ptr(kv), B, P, _ptr(canvas_out), _ptr(steps_used),
                                       _ptr(n_committed), _stream(stream)), "dg_generate_block")

    def generate(self, prompt, B, P, n_blocks, kv, tokens_out, steps_used, n_committed, stream=None):
        """Block-autoregressive generation of n_blocks canvases (see dg_generate)."""
        _check(lib().dg_generate(self.h, _ptr(prompt), B, P, n_blocks, _ptr(kv), _ptr(tokens_out),
                                 _ptr(steps_used), _ptr(n_committed), _stream(stream)), "dg_generate")

    def sync_status(self, stream=None):
        _check(lib().dg_sync_status(self.h, _stream(stream)), "device status")

    def kernels_per_step(self, B, P):
        return int(lib().dg_kernels_per_step(self.h, B, P))

    def launches_per_round(self):
        return int(lib().dg_launches_per_round(self.h))

    # -- test / bench hooks --------------------------------------------------------
    def read_weight(self, tensor_id, out, stream=None):
        _check(lib().dg_read_weight(self.h, tensor_id, _ptr(out), _stream(stream)), "dg_read_weight")

    def load_kv(self, kv, B, P, k, v, stream=None):
        _check(lib().dg_load_kv(self.h, _ptr(kv), B, P, _ptr(k), _ptr(v), _stream(stream)), "dg_load_kv")

    def debug_trace(self, h_trace=None, ids_trace=None):
        """Record per-layer hidden states and routing of later eager calls."""
        _check(lib().dg_debug_trace(self.h, _ptr(h_trace), _ptr(ids_trace)), "dg_debug_trace")

    def run_layer(self, kv, B, P, layer, h_in, h_trace, ids, stream=None):
        """Layer `layer` of the canvas pass from the residual state h_in
        [B*256, d] (model dtype): h_trace fp32 [3, B*256, d] receives h after
        the attention residual, after the MoE and RMSNorm of the latter; ids
        int32 [B*256, top_k] the routing; the canvas keys/values go into kv."""
        _check(lib().dg_test_layer(self.h, _ptr(kv), B, P, layer, _ptr(h_in), _ptr(h_trace), _ptr(ids),
                                   _stream(stream)), "dg_test_layer")

    def run_moe(self, B, layer, h_attn, h_trace, ids, stream=None):
        """The MoE half of layer `layer` from the residual state h_attn
        [B*256, d] (model dtype) after its attention: h_trace fp32
        [3, B*256, d] receives h after the MoE in row 1 and its RMSNorm in
        row 2; ids int32 [B*256, top_k] the routing."""
        _check(lib().dg_test_moe(self.h, B, layer, _ptr(h_attn), _ptr(h_trace), _ptr(ids), _stream(stream)),
               "dg_test_moe")

    def expert_counts(self, counts, stream=None):
        """Per-layer expert row counts [n_layers, n_experts] of the most recent call."""
        _check(lib().dg_expert_counts(self.h, _ptr(counts), _stream(stream)), "dg_expert_counts")
        return counts

    def set_routing_bias(self, bias, n_tok=None):
        """Per-token router bias of the canvas passes, device fp32 [L, n_tok, E]
        (None removes it); the caller keeps the tensor alive while in use."""
        if bias is None:
            _check(lib().dg_set_routing_bias(self.h, None, 0), "dg_set_routing_bias")
            self._routing_bias = None
            return
        n = bias.shape[1] if n_tok is None else n_tok
        _check(lib().dg_set_routing_bias(self.h, _ptr(bias), n), "dg_set_routing_bias")
        self._routing_bias = bias

    def touched_experts_sum(self, reset=False, stream=None):
        """Per layer, the distinct experts streamed summed over every canvas
        pass since creation or the last reset (list of ints)."""
        out = (ctypes.c_uint64 * self.w.n_layers)()
        _check(lib().dg_touched_experts_sum(self.h, out, int(reset), _stream(stream)), "dg_touched_experts_sum")
        return [int(x) for x in out]

    def reset_touched_experts(self, stream=None):
        _check(lib().dg_touched_experts_sum(self.h, None, 1, _stream(stream)), "dg_touched_experts_sum")

    def touched_experts(self, stream=None):
        """Distinct experts each layer of the most recent call routed to (list)."""
        import torch
        c = torch.zeros((self.w.n_layers, self.w.n_experts), dtype=torch.int32, device="cuda")
        self.expert_counts(c, stream)
        return [int(x) for x in (c > 0).sum(dim=1).tolist()]

    def profile_step(self, kv, B, P, reps=3, stream=None):
        n = 32
        ms = (ctypes.c_float * n)()
        cnt = (ctypes.c_int32 * n)()
        _check(lib().dg_profile_step(self.h, _ptr(kv), B, P, reps, ms, cnt, n, _stream(stream)), "dg_profile_step")
        out = {}
        for i in range(n):
            name = lib().dg_phase_name(i)
            if name is None:
                break
            out[name.decode()] = (ms[i], cnt[i])
        return out


def test_math(which, x, out, aux0=0, aux1=0, stream=None):
    _check(lib().dg_test_math(which, _ptr(x), _ptr(out), x.numel(), aux0, aux1, _stream(stream)), "dg_test_math")


def test_philox(inp, out, stream=None):
    _check(lib().dg_test_philox(_ptr(inp), _ptr(out), inp.shape[0], _stream(stream)), "dg_test_philox")


def test_sampler(logits, positions, seed, step, t, temp_start, temp_end, H, tok, amax, s_q=None, u_q=None,
                 probs=None, stream=None):
    import torch
    rows, vocab = logits.shape
    bf = 1 if (probs is not None and probs.dtype == torch.bfloat16) else 0
    _check(lib().dg_test_sampler(_ptr(logits), rows, vocab, positions, seed, step, float(t), float(temp_start),
                                 float(temp_end), _ptr(H), _ptr(tok), _ptr(amax), _ptr(s_q), _ptr(u_q),
                                 _ptr(probs), bf, _stream(stream)), "dg_test_sampler")


def test_sampler_topk(logits, positions, seed, step, t, temp_start, temp_end, K, H, tok, amax, cand_ids, cand_w,
                      s_q=None, u_q=None, stream=None):
    import torch
    rows, vocab = logits.shape
    bf = 1 if cand_w.dtype == torch.bfloat16 else 0
    _check(lib().dg_test_sampler_topk(_ptr(logits), rows, vocab, positions, seed, step, float(t), float(temp_start),
                                      float(temp_end), K, _ptr(H), _ptr(tok), _ptr(amax), _ptr(s_q), _ptr(u_q),
                                      _ptr(cand_ids), _ptr(cand_w), bf, _stream(stream)), "dg_test_sampler_topk")


def test_sc_gather(cand_ids, cand_w, emb, u, stream=None):
    import torch
    rows, K = cand_ids.shape
    d = emb.shape[1]
    _check(lib().dg_test_sc_gather(_ptr(cand_ids), _ptr(cand_w), rows, K, _ptr(emb), d,
                                   1 if emb.dtype == torch.bfloat16 else 0, _ptr(u), _stream(stream)),
           "dg_test_sc_gather")


def test_quant_fp8(w, codes, scales, stream=None):
    rows, K = w.shape
    _check(lib().dg_test_quant_fp8(_ptr(w), rows, K, _ptr(codes), _ptr(scales), _stream(stream)), "dg_test_quant_fp8")


def test_grouped_gemm_fp8(codes, scales, B, counts, groups, M, out, bn=64, k_splits=1, stream=None):
    K = codes.shape[-1]
    c = (ctypes.c_int32 * groups)(*[int(x) for x in counts])
    _check(lib().dg_test_grouped_gemm_fp8(_ptr(codes), _ptr(scales), _ptr(B), c, groups, M, K, bn, k_splits,
                                          _ptr(out), _stream(stream)), "dg_test_grouped_gemm_fp8")


def test_commit(H, tok, amax, prev_amax, vocab, seed, step, max_steps, commit_mode, commit_bound, stop_mode,
                stop_bound, commit, canvas_next, stop, n_committed, stream=None):
    B = H.shape[0]
    _check(lib().dg_test_commit(_ptr(H), _ptr(tok), _ptr(amax), _ptr(prev_amax), B, vocab, seed, step, max_steps,
                                commit_mode, float(commit_bound), stop_mode, float(stop_bound), _ptr(commit),
                                _ptr(canvas_next), _ptr(stop), _ptr(n_committed), _stream(stream)), "dg_test_commit")


def test_gemm(A, B, out, alpha=1.0, k_splits=1, bn=256, persistent=False, m256=False, stream=None):
    import torch
    M, K = A.shape
    N = B.shape[0]
    flags = int(persistent) | (2 if m256 else 0)
    _check(lib().dg_test_gemm(_ptr(A), _ptr(B), _ptr(out), M, N, K, 1 if A.dtype == torch.bfloat16 else 0,
                              float(alpha), k_splits, bn, flags, _stream(stream)), "dg_test_gemm")


def test_router(x, wr, ids, gate, bias=None, tok_bias=None, stream=None):
    T, d = x.shape
    E = wr.shape[0]
    k = ids.shape[1]
    _check(lib().dg_test_router(_ptr(x), _ptr(wr), _ptr(bias) if bias is not None else None,
                                _ptr(tok_bias) if tok_bias is not None else None, T, d, E, k,
                                _ptr(ids), _ptr(gate), _stream(stream)), "dg_test_router")


def test_grouped_gemm(A, B, counts, groups, M, out, bn=64, persistent=False, sized_ring=False, swiglu=False,
                      m256=False, stream=None):
    import torch
    K = A.shape[-1]
    c = (ctypes.c_int32 * groups)(*[int(x) for x in counts])
    flags = int(persistent) | (2 if sized_ring else 0) | (4 if swiglu else 0) | (8 if m256 else 0)
    _check(lib().dg_test_grouped_gemm(_ptr(A), _ptr(B), c, groups, M, K, 1 if A.dtype == torch.bfloat16 else 0,
                                      bn, flags, _ptr(out), _stream(stream)), "dg_test_grouped_gemm")


def test_attention(q, k, v, n_canvas, n_q, q_pos0, n_keys, causal, Hq, Hkv, out, force_path=0, stream=None):
    """Returns the merge path taken: 1 = split partials + combine kernel,
    2 = in-kernel cluster merge."""
    import torch
    hd = q.shape[-1]
    path = ctypes.c_int32(0)
    _check(lib().dg_test_attention(_ptr(q), _ptr(k), _ptr(v), n_canvas, n_q, q_pos0, n_keys, int(causal), Hq,
                                   Hkv, hd, 1 if q.dtype == torch.bfloat16 else 0, int(force_path),
                                   ctypes.byref(path), _ptr(out), _stream(stream)), "dg_test_attention")
    return path.value


def attn_cluster_capacity():
    """Resident thread-block clusters of the bf16 attention kernel per cluster
    size 1..8 (index 0 unused), as the device reports them."""
    out = (ctypes.c_int32 * 9)()
    _check(lib().dg_test_attn_capacity(out), "dg_test_attn_capacity")
    return list(out)


def gemm_splitk_noalloc(A, B, out, k_splits=1, stream=None):
    """out[n][m] = sum_k A[m][k] B[n][k] (bf16 in, fp32 out) through the
    entry point that allocates no device memory (its split-K partial sums
    live in a fixed-size array inside the library).  For callers that must
    not call cudaMalloc: see dg_gemm_splitk_noalloc in include/dg.h."""
    import torch
    for name, t, dt in (("A", A, torch.bfloat16), ("B", B, torch.bfloat16), ("out", out, torch.float32)):
        if t.dtype != dt or t.dim() != 2 or not t.is_contiguous() or t.device != A.device:
            raise ValueError(f"gemm_splitk_noalloc: {name} must be a contiguous 2-D {dt} tensor on {A.device}")
    M, K = A.shape
    N = B.shape[0]
    if B.shape[1] != K:
        raise ValueError(f"gemm_splitk_noalloc: B has {B.shape[1]} columns, A has {K}")
    if tuple(out.shape) != (N, M):
        raise ValueError(f"gemm_splitk_noalloc: out must be [{N}, {M}], got {list(out.shape)}")
    _check(lib().dg_gemm_splitk_noalloc(_ptr(A), _ptr(B), _ptr(out), M, N, K, k_splits, _stream(stream)),
           "dg_gemm_splitk_noalloc")
