"""Host-side pieces of bench.py that need no GPU."""
import json

import pytest

import bench


def test_roofline_traffic_is_attached_to_the_measured_code_only(tmp_path, monkeypatch):
    src = open(bench.os.path.join(bench.ROOT, "state_space_model_07_b200", "csrc", "ssd_tc.cu")).read()
    csrc = tmp_path / "state_space_model_07_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "ssd_tc.cu").write_text(src)
    p = tmp_path / "profiles"
    p.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"source_sha": bench.kernel_source_sha("tc_scan"), "dram_bytes": 1000, "units": 10}
    (p / "traffic.json").write_text(json.dumps({"tc_scan": rec}))
    # a DRAM capture is reported for the kernel as it stands ...
    assert bench.traffic_for("tc_scan", 10) == 1000
    # ... scales with the units a launch processes ...
    assert bench.traffic_for("tc_scan", 20) == 2000
    # ... and is dropped once the recorded hash no longer matches the code
    (p / "traffic.json").write_text(json.dumps({"tc_scan": dict(rec, source_sha="0" * 16)}))
    assert bench.traffic_for("tc_scan", 10) is None


def test_committed_traffic_record_names_its_kernel_and_summary():
    rec = json.load(open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for name, r in rec.items():
        assert {"kernel", "workload", "source_sha", "dram_bytes", "units", "summary"} <= set(r), name
        assert bench.os.path.exists(bench.os.path.join(bench.ROOT, "profiles", r["summary"])), name


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "state_space_model_07_b200" / "csrc"
    csrc.mkdir(parents=True)
    f = csrc / "ssd_tc.cu"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f.write_text("int a = 1;  // one\n/* block */\nint b = 2;\n")
    h0 = bench.kernel_source_sha("tc_scan")
    f.write_text("// header\nint a = 1;\n\nint b = 2;  /* two */\n")
    assert bench.kernel_source_sha("tc_scan") == h0
    f.write_text("int a = 1;\nint b = 3;\n")
    assert bench.kernel_source_sha("tc_scan") != h0


def test_algorithmic_bytes_of_the_bench_workload():
    from state_space_model_07_b200 import inputs
    w = inputs.WORKLOADS["mamba2_2.7b_layer"]
    tokens = w.batch * w.seqlen
    # x + y (80 heads x 64 x 2 B each), dt (80 x 2 B), B + C (128 x 2 B each) per token, plus the final state
    per_tok = 2 * 80 * 64 * 2 + 80 * 2 + 2 * 128 * 2
    assert bench.workload_bytes(w, w.batch, tokens, 2) == tokens * per_tok + 8 * 80 * 128 * 64 * 4 == 714080256


def test_algorithmic_flops_count_the_causal_pairs_once():
    """The chunked form's multiply-adds counted by enumeration on a small case: per chunk and head
    every causal pair (i <= j) once for S x (P each) and per group once for C B^T (N each), every
    token's B x^T and C h_prev (N P each), and one N x P state update per chunk."""
    from state_space_model_07_b200 import inputs
    w = inputs.Workload("f", 2, 24, 3, 8, 16, 1, 8, "bf16", 0, False)
    L_tot, Q, H, P, N, G = w.batch * w.seqlen, w.chunk, w.nheads, w.headdim, w.dstate, w.ngroups
    pairs = sum(1 for _ in range(L_tot // Q) for j in range(Q) for i in range(j + 1))
    macs = H * (pairs * P + L_tot * N * P * 2 + (L_tot // Q) * N * P) + G * pairs * N
    assert bench.workload_flops(w, L_tot, Q) == pytest.approx(2 * macs, rel=1e-12)


def test_scan_hash_covers_the_measured_kernel_not_the_d_state_256_one(tmp_path, monkeypatch):
    src = open(bench.os.path.join(bench.ROOT, "state_space_model_07_b200", "csrc", "ssd_tc.cu")).read()
    csrc = tmp_path / "state_space_model_07_b200" / "csrc"
    csrc.mkdir(parents=True)
    f = csrc / "ssd_tc.cu"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f.write_text(src)
    h0 = bench.kernel_source_sha("tc_scan")
    # an edit inside the first-generation k_tc_scan<N> (another kernel) keeps the hash ...
    sig = "k_tc_scan(const __grid_constant__"
    i = src.index("{", src.index(sig))
    f.write_text(src[:i + 1] + "\n    int unused_probe = 0;\n" + src[i + 1:])
    assert bench.kernel_source_sha("tc_scan") == h0
    # ... one inside k_tc_scan3 does not
    j = src.index("{", src.index("k_tc_scan3(const __grid_constant__"))
    f.write_text(src[:j + 1] + "\n    int unused_probe = 0;\n" + src[j + 1:])
    assert bench.kernel_source_sha("tc_scan") != h0


def test_profiling_overrides_shrink_the_workload_and_reject_bad_heads():
    import argparse
    import bench
    ns = lambda **kw: argparse.Namespace(**dict({"workload": "packed_varlen", "batch": None, "heads": None}, **kw))
    w = bench.workload_of(ns(heads=16))
    assert (w.nheads, w.ngroups, w.dstate, w.packed_nseqs) == (16, 4, 256, 16)
    w = bench.workload_of(ns(workload="mamba2_2.7b_layer", batch=2))
    assert (w.batch, w.seqlen, w.nheads) == (2, 4096, 80)
    assert bench.workload_of(ns(batch=2)).batch == 1          # packed input has one row
    for bad in (0, 6, -4):
        with pytest.raises(SystemExit):
            bench.workload_of(ns(heads=bad))
