"""Host-only checks of the C ABI: the library loads, exports every function
include/ssd.h declares, and rejects bad arguments before touching a device.

The pointers passed here are never dereferenced: validation happens on the
host before any CUDA call, so these tests run without a GPU.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from state_space_model_07_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")
FAKE = 0x10000  # 16-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", src)))


def test_header_declares_the_bound_functions():
    assert declared_functions() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)$", out, re.M))
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(L, name)
    # nothing else leaks out of the library
    assert {n for n in exported if n.startswith("ssd")} == set(declared_functions())


def test_status_strings(L):
    for code in range(10):
        s = L.ssd_status_string(code).decode()
        assert s and s != "unknown status"
    assert L.ssd_status_string(99).decode() == "unknown status"


def dims(**kw):
    base = dict(batch=2, seqlen=64, nheads=4, headdim=64, dstate=128, ngroups=2, nseqs=0, dtype=1)
    base.update(kw)
    return _lib.SsdDims(**base)


def scan(L, d, chunk=128, entry="ssd_chunk_scan_fwd", **ptrs):
    p = dict(x=FAKE, dt=FAKE * 2, dt_bias=None, A=FAKE * 3, B=FAKE * 40, C=FAKE * 80, D=None,
             init_state=None, seq_idx=None, y=FAKE * 120, final_state=None)
    p.update(ptrs)
    v = lambda k: None if p[k] is None else ctypes.c_void_p(p[k])
    return getattr(L, entry)(ctypes.byref(d) if d is not None else None, v("x"), v("dt"), v("dt_bias"),
                             v("A"), v("B"), v("C"), v("D"), v("init_state"), v("seq_idx"), chunk,
                             v("y"), v("final_state"), None)


ENTRIES = ["ssd_chunk_scan_fwd", "ssd_chunk_scan_fwd_noalloc"]


@pytest.mark.parametrize("kw,chunk,ptrs,code", [
    ({}, 128, {"x": None}, 1),
    ({}, 128, {"A": None}, 1),
    ({"dtype": 7}, 128, {}, 3),
    ({"headdim": 24}, 128, {}, 2),
    ({"dstate": 512}, 128, {}, 2),
    ({"nheads": 6, "ngroups": 4}, 128, {}, 2),
    ({"seqlen": -1}, 128, {}, 2),
    ({}, 96, {}, 4),
    ({}, 512, {}, 4),
    ({}, 8, {}, 4),
    ({}, 128, {"x": FAKE + 4}, 2),                         # misaligned
    ({}, 128, {"y": FAKE}, 2),                             # y aliases x
    ({}, 128, {"seq_idx": FAKE * 200}, 2),                 # packing needs batch 1
    ({"batch": 1, "nseqs": 0}, 128, {"seq_idx": FAKE * 200}, 2),
    ({"batch": 1, "nseqs": 65}, 128, {"seq_idx": FAKE * 200}, 2),
    ({}, 128, {"init_state": FAKE * 300, "final_state": FAKE * 300 + 64}, 2),  # partial overlap
])
@pytest.mark.parametrize("entry", ENTRIES)
def test_scan_rejects_bad_arguments(L, kw, chunk, ptrs, code, entry):
    assert scan(L, dims(**kw), chunk, entry=entry, **ptrs) == code
    assert L.ssd_last_error().decode()


@pytest.mark.parametrize("entry", ENTRIES)
def test_scan_null_dims(L, entry):
    assert scan(L, None, entry=entry) == 1


@pytest.mark.parametrize("entry", ENTRIES)
def test_empty_scan_without_states_is_a_host_side_no_op(L, entry):
    # no tokens and no final_state to fill: nothing reaches a device
    assert scan(L, dims(seqlen=0), entry=entry, x=None, dt=None, B=None, C=None, y=None) == 0
    assert scan(L, dims(batch=0), entry=entry) == 0


def update(L, d, **ptrs):
    p = dict(state=FAKE, x=FAKE * 2, dt=FAKE * 3, A=FAKE * 4, B=FAKE * 5, C=FAKE * 6, D=None, y=FAKE * 500,
             dt_bias=None)
    p.update(ptrs)
    v = lambda k: None if p[k] is None else ctypes.c_void_p(p[k])
    return L.ssd_state_update(ctypes.byref(d), v("state"), v("x"), v("dt"), v("A"), v("B"), v("C"), v("D"),
                              v("y"), None, v("dt_bias"))


def test_state_update_rejects_bad_arguments(L):
    assert update(L, dims(), state=None) == 1
    assert update(L, dims(dtype=3)) == 3
    assert update(L, dims(headdim=8)) == 2
    assert update(L, dims(), state=FAKE + 8) == 2
    assert update(L, dims(), y=FAKE * 2) == 2          # y aliases x
    assert update(L, dims(batch=0)) == 0               # empty batch is a no-op


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a CUDA device")
@pytest.mark.parametrize("entry", ENTRIES)
def test_valid_call_without_device_reports_cuda_error(L, entry):
    # All arguments valid: the first CUDA call (workspace allocation, or the
    # scratch array's address) fails cleanly because this host has no GPU.
    assert scan(L, dims(), entry=entry) == 6
    assert L.ssd_last_error().decode()


def test_python_wrapper_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="CUDA library missing"):
        _lib.lib()


def test_noalloc_scan_refuses_oversized_calls_on_the_host(L):
    # Refused before any device work: the fake pointers are never touched.
    d = dims(batch=8, seqlen=4096, nheads=80, headdim=64, dstate=128, ngroups=1)
    v = ctypes.c_void_p
    rc = L.ssd_chunk_scan_fwd_noalloc(ctypes.byref(d), v(FAKE), v(FAKE * 2), None, v(FAKE * 3),
                                      v(FAKE * 40000), v(FAKE * 80000), None, None, None, 256,
                                      v(FAKE * 120000), None, None)
    assert rc == 5
    assert "32 MiB" in L.ssd_last_error().decode()


def test_python_wrapper_rejects_host_and_mistyped_tensors_before_any_call():
    """The binding validates on the host and raises before reaching the library:
    no CPU path exists, so CPU tensors are an error, as are wrong dtypes and layouts."""
    import torch
    import state_space_model_07_b200 as ssd
    x = torch.zeros(1, 8, 2, 16, dtype=torch.bfloat16)
    dt = torch.zeros(1, 8, 2, dtype=torch.bfloat16)
    A = torch.zeros(2)
    B = torch.zeros(1, 8, 1, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ssd.chunk_scan_fwd(x, dt, A, B, B, chunk=16)
    with pytest.raises(TypeError):
        ssd.chunk_scan_fwd([0], dt, A, B, B, chunk=16)
    st = torch.zeros(1, 2, 16, 16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ssd.state_update(st, x[:, 0], dt[:, 0], A, B[:, 0], B[:, 0])


def test_selftest_wait_checks_its_limit_on_the_host(L):
    assert L.ssd_selftest_bounded_wait(10, None) == 2
    assert L.ssd_selftest_bounded_wait(5_000_000_000, None) == 2
    assert "limit_cycles" in L.ssd_last_error().decode()


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a CUDA device")
def test_selftest_wait_without_device_reports_cuda_error(L):
    assert L.ssd_selftest_bounded_wait(2_000_000, None) == 6
