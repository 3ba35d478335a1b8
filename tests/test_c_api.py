"""The C ABI is usable from plain C: tests/c_api_example.c compiles against
include/ssd.h and links against the in-tree libssd.so (no GPU needed to build), and on a GPU
its scan and decode step (fp32) match the fp64 oracle within 1e-4 (1 + |ref|)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "state_space_model_07_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


needs_build = pytest.mark.skipif(
    shutil.which("gcc") is None or not os.path.exists(os.path.join(LIB_DIR, "libssd.so")),
    reason="needs gcc and the built library")


def _build(tmp_path):
    exe = tmp_path / "c_api_example"
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_api_example.c"),
           "-L", LIB_DIR, "-lssd", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + LIB_DIR, "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@needs_build
def test_c_example_compiles_and_links(tmp_path):
    assert _build(tmp_path).exists()


@needs_build
@pytest.mark.gpu
def test_c_example_matches_the_oracle(tmp_path):
    import numpy as np
    import oracle
    exe = _build(tmp_path)
    out = tmp_path / "arrays.f32"
    r = subprocess.run([str(exe), str(out)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "ok" in r.stdout, (r.returncode, r.stderr)
    b, L, H, P, N, G = 2, 100, 4, 16, 16, 2
    sizes = [("x", (b, L, H, P)), ("dt", (b, L, H)), ("B", (b, L, G, N)), ("C", (b, L, G, N)), ("A", (H,)),
             ("D", (H,)), ("bias", (H,)), ("y", (b, L, H, P)), ("x1", (b, H, P)), ("dt1", (b, H)),
             ("B1", (b, G, N)), ("C1", (b, G, N)), ("y1", (b, H, P)), ("state", (b, H, N, P))]
    flat = np.fromfile(out, dtype=np.float32)
    a, i = {}, 0
    for k, shp in sizes:
        n = int(np.prod(shp))
        a[k] = flat[i:i + n].reshape(shp).astype(np.float64)
        i += n
    assert i == flat.size
    yr, fr = oracle.ssd_scan(a["x"], a["dt"], a["A"], a["B"], a["C"], dt_bias=a["bias"], D=a["D"])
    sr, y1r = oracle.state_update(fr, a["x1"], a["dt1"], a["A"], a["B1"], a["C1"], dt_bias=a["bias"], D=a["D"])
    for got, ref, what in ((a["y"], yr, "scan y"), (a["y1"], y1r, "decode y"), (a["state"], sr, "state")):
        err = np.max(np.abs(got - ref) / (1 + np.abs(ref)))
        assert err <= 1e-4, (what, err)
