"""Timeline of the persistent expert GEMM (diagnostics).

Runs grouped GEMMs shaped like the expert layers of the 26B-A4B-shaped
model through libdg_probe.so (the library built with -DDG_PROBE, see
`python -m block_text_diffusion_b200.build --probe`) and prints, for CTA 0,
when each K block's loads were issued and landed, and when each tile's
accumulator completed and its epilogue finished.  Usage:
python -m block_text_diffusion_b200.diag.probe_gemm [all]
"""
import ctypes
import os
import sys

import numpy as np
import torch

import block_text_diffusion_b200 as dg

dg.LIB_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "libdg_probe.so")
L = dg.lib()
L.dg_probe_read.argtypes = [ctypes.c_void_p]
L.dg_probe_read.restype = ctypes.c_int

def run(name, M, K, counts, swiglu, m256=False):
    g = torch.Generator(device="cuda").manual_seed(1)
    G, rows = len(counts), sum(counts)
    A = (0.02 * torch.randn((G * M, K), device="cuda", generator=g)).to(torch.bfloat16)
    B = torch.randn((rows, K), device="cuda", generator=g).to(torch.bfloat16)
    out = torch.zeros((rows, M), dtype=torch.float32, device="cuda")
    for _ in range(3):
        dg.test_grouped_gemm(A, B, counts, G, M, out, bn=256, persistent=True, sized_ring=True, swiglu=swiglu,
                             m256=m256)
    buf = (ctypes.c_longlong * 4096)()
    L.dg_probe_read(buf)
    a = np.array(buf[:], dtype=np.int64)
    t0 = a[1000]
    rel = lambda x: (x - t0) / 1000.0
    issue = [rel(a[i]) for i in range(256) if a[i] > t0]
    land = [rel(a[256 + i]) for i in range(256) if a[256 + i] > t0]
    print(f"== {name}: M {M} K {K} experts {G} rows {rows}; stamps issue {len(issue)} land {len(land)}")
    n = min(len(issue), len(land), 60)
    for i in range(0, n, max(1, n // 20)):
        print(f"  kb {i:3d}: issue {issue[i]:8.2f} us  land {land[i]:8.2f} us  lat {land[i]-issue[i]:6.2f}")
    if len(land) > 4:
        d = np.diff(land[:n])
        print(f"  land interval median {np.median(d):.3f} us, mean {np.mean(d):.3f}")
    for t in range(8):
        af, ae, ed = a[512 + t], a[576 + t], a[640 + t]
        if ae > t0:
            print(f"  tile {t}: acc free {rel(af):8.2f}  acc complete {rel(ae):8.2f}  epilogue done {rel(ed) if ed > t0 else -1:8.2f}")

which = sys.argv[1] if len(sys.argv) > 1 else "all"
run("gate|up 10x256", 1408, 2816, [256] * 8 + [128, 128], False)
if which == "all":
    run("gate|up 10x256 fused", 1408, 2816, [256] * 8 + [128, 128], True)
    run("gate|up 120x17", 1408, 2816, [17] * 120, False)
    run("down 10x256", 2816, 704, [256] * 8 + [128, 128], False)
    run("gate|up 10x256 m256", 1408, 2816, [256] * 8 + [128, 128], False, True)
    run("gate|up 10x256 m256 fused", 1408, 2816, [256] * 8 + [128, 128], True, True)
    run("gate|up 120x17 m256", 1408, 2816, [17] * 120, False, True)
    run("down 10x256 m256", 2816, 704, [256] * 8 + [128, 128], False, True)
