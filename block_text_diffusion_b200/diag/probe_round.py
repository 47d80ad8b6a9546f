"""Per-kernel timeline of denoising rounds inside the captured block loop
(diagnostics).

Runs one block of the chosen workload through libdg_probe.so (built with
`python -m block_text_diffusion_b200.build --probe`), in which a one-thread
stamp kernel follows every phase launch and records the global time once the
launch before it has completed.  The interval between consecutive stamps is
attributed to the phase of the later one; intervals include the stamp
kernels' own launch latency (a few microseconds each), so compare phases
with each other rather than with the plain build.  Usage:
python -m block_text_diffusion_b200.diag.probe_round [workload] [rounds]
"""
import ctypes
import os
import sys
from collections import defaultdict

import numpy as np
import torch

import block_text_diffusion_b200 as dg
from block_text_diffusion_b200 import inputs as I

dg.LIB_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "libdg_probe.so")
L = dg.lib()
L.dg_timeline_read.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int]
L.dg_timeline_read.restype = ctypes.c_int


def main():
    name = sys.argv[1] if len(sys.argv) > 1 else "moe26b"
    rounds = int(sys.argv[2]) if len(sys.argv) > 2 else 3
    w = I.WORKLOADS[name].replace(max_steps=rounds)
    P = w.prompt_len
    model = dg.Model(w, max_canvases=1, max_prompt=P)
    kv = model.new_kv(1, P)
    model.encode_prompt(torch.from_numpy(I.prompt_ids(w.sample_seed, 1, P, w.vocab)).cuda(), kv)
    z = lambda *s: torch.zeros(s, dtype=torch.int32, device="cuda")
    canvas, steps, ncom = z(1, 256), z(1), z(1)
    model.generate_block(kv, 1, P, canvas, steps, ncom)       # capture + warm-up
    cap = 8192
    t = (ctypes.c_longlong * cap)()
    ph = (ctypes.c_int * cap)()
    L.dg_timeline_read(t, ph, cap, 1)                          # drop the warm-up records
    model.generate_block(kv, 1, P, canvas, steps, ncom)
    n = L.dg_timeline_read(t, ph, cap, 1)
    model.sync_status()
    ts = np.array(t[:n], dtype=np.int64)
    phs = np.array(ph[:n], dtype=np.int32)
    names = {i: L.dg_phase_name(i).decode() for i in range(32) if L.dg_phase_name(i)}
    per = defaultdict(float)
    count = defaultdict(int)
    for i in range(1, n):
        per[phs[i]] += (ts[i] - ts[i - 1]) / 1000.0
        count[phs[i]] += 1
    total = (ts[-1] - ts[0]) / 1000.0
    r = int(steps[0].item())
    print(f"{w.name}: {r} rounds, {n} stamps, {total / 1000.0:.3f} ms from first to last stamp "
          f"({total / 1000.0 / max(1, r):.3f} ms per round)")
    print(f"{'phase':24s} {'us/round':>10s} {'launches/round':>15s} {'us/launch':>10s} {'share':>7s}")
    for p in sorted(per, key=lambda k: -per[k]):
        print(f"{names.get(p, str(p)):24s} {per[p] / r:10.1f} {count[p] / r:15.1f} {per[p] / count[p]:10.2f} "
              f"{per[p] / total:7.1%}")
    model.close()


if __name__ == "__main__":
    main()
