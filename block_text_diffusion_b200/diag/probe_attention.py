"""Timeline of the attention kernel (diagnostics).

Runs the canvas attention of the 26B-A4B shape (256 canvas queries, 16 query
/ 8 KV heads, 2048 + 256 keys) through libdg_probe.so (see
`python -m block_text_diffusion_b200.build --probe`) and prints CTA 0's
stamps: start, prologue done, Q landed, per K/V block of tile A the QK^T issue,
the softmax start and the P hand-off, the epilogue and the exit.  Usage:
python -m block_text_diffusion_b200.diag.probe_attention
"""
import ctypes
import os

import numpy as np
import torch

import block_text_diffusion_b200 as dg

dg.LIB_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "libdg_probe.so")
L = dg.lib()
L.dg_probe_read.argtypes = [ctypes.c_void_p]
L.dg_probe_read.restype = ctypes.c_int


def run(n_q, n_prefix, Hq, Hkv):
    n_keys = n_prefix + n_q
    g = torch.Generator(device="cuda").manual_seed(1)
    q = torch.randn((n_q, Hq, 128), device="cuda", generator=g).to(torch.bfloat16)
    k = torch.randn((1, Hkv, n_keys, 128), device="cuda", generator=g).to(torch.bfloat16)
    v = torch.randn((1, Hkv, n_keys, 128), device="cuda", generator=g).to(torch.bfloat16)
    out = torch.zeros((n_q, Hq, 128), dtype=torch.float32, device="cuda")
    for _ in range(3):
        dg.test_attention(q, k, v, 1, n_q, n_prefix, n_keys, False, Hq, Hkv, out)
    buf = (ctypes.c_longlong * 4096)()
    L.dg_probe_read(buf)
    a = np.array(buf[:], dtype=np.int64)
    t0 = a[2000]
    rel = lambda x: (x - t0) / 1000.0 if x > t0 else float("nan")
    print(f"== attention n_q {n_q} keys {n_keys} Hq {Hq} Hkv {Hkv}")
    print(f"  prologue done {rel(a[2001]):.2f} us, Q landed {rel(a[2002]):.2f} us")
    for j in range(32):
        if a[2050 + j] > t0:
            print(f"  block {j}: S issued {rel(a[2010 + j]):7.2f}  softmax start {rel(a[2050 + j]):7.2f}  "
                  f"P handed {rel(a[2090 + j]):7.2f}")
    print(f"  epilogue start {rel(a[2130]):.2f}, end {rel(a[2131]):.2f}, exit {rel(a[2140]):.2f} us")


run(256, 2048, 16, 8)
run(256, 1024, 8, 2)
