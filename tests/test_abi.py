"""The C-ABI library loads and exports every symbol its headers declare (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("dg.h", "dg_test.h")]


def declared():
    names = []
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(dg_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def libpath():
    from block_text_diffusion_b200 import build
    return build.build()


def test_headers_declare_the_api():
    names = declared()
    for n in ("dg_init_weights", "dg_encode_prompt", "dg_denoise_step", "dg_generate_block", "dg_free",
              "dg_kv_bytes", "dg_status_string", "dg_sync_status"):
        assert n in names


def test_library_exports_every_declared_symbol(libpath):
    out = subprocess.check_output(["nm", "-D", "--defined-only", libpath], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in declared() if n not in exported]
    assert not missing, missing


def test_library_loads_and_answers_without_a_gpu(libpath):
    L = ctypes.CDLL(libpath)
    L.dg_status_string.restype = ctypes.c_char_p
    L.dg_status_string.argtypes = [ctypes.c_int]
    assert L.dg_status_string(0) == b"ok"
    assert L.dg_status_string(1) == b"invalid argument"
    # argument validation happens before any device work
    L.dg_init_weights.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
    assert L.dg_init_weights(None, 0, None, None) == 1
    L.dg_kv_bytes.restype = ctypes.c_size_t
    L.dg_kv_bytes.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32]
    assert L.dg_kv_bytes(None, 1, 1) == 0


def test_bad_config_rejected_on_host(libpath):
    import block_text_diffusion_b200 as dg
    from block_text_diffusion_b200 import inputs as I
    L = dg.lib()
    h = ctypes.c_void_p()
    for bad in (dict(d_model=100), dict(head_dim=96), dict(n_heads=6, n_kv_heads=4), dict(top_k=9),
                dict(vocab=1000), dict(max_steps=0)):
        cfg = dg.make_config(I.TINY_FP32.replace(**bad))
        assert L.dg_init_weights(ctypes.byref(cfg), 0, None, ctypes.byref(h)) == 1
    cfg = dg.make_config(I.TINY_FP32)
    cfg.canvas_len = 128
    assert L.dg_init_weights(ctypes.byref(cfg), 0, None, ctypes.byref(h)) == 1


def test_product_path_refuses_without_library(tmp_path, monkeypatch):
    import block_text_diffusion_b200 as dg
    monkeypatch.setattr(dg, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(dg, "_lib", None)
    with pytest.raises(RuntimeError):
        dg.lib()


def test_binding_structs_match_the_header_layout(tmp_path):
    # the ctypes mirrors of dg_config and dg_step_out have the C layout
    # (size and every field offset), compiled from the header with the host C compiler
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    import block_text_diffusion_b200 as dg
    structs = {"dg_config": dg.Config, "dg_step_out": dg.StepOut}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "dg.h"', 'int main(void) {']
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'  printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call([cc, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = {}
    for line in subprocess.check_output([str(exe)], text=True).splitlines():
        cname, field, val = line.split()
        got[(cname, field)] = int(val)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)
