"""The C ABI is usable from plain C: tests/c_api_example.c compiles against
include/ssd.h and links against the in-tree libssd.so (no GPU needed to build)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "state_space_model_07_b200")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.exists(os.path.join(LIB_DIR, "libssd.so")),
                    reason="needs gcc and the built library")
def test_c_example_compiles_and_links(tmp_path):
    exe = tmp_path / "c_api_example"
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_api_example.c"),
           "-L", LIB_DIR, "-lssd", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + LIB_DIR, "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert exe.exists()
