#!/usr/bin/env python
"""SSD chunked-scan forward throughput on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--batch B] [--no-e2e] [--no-cpu-baseline]

A step is one pass of the whole hot path over one batch of synthetic input:
ssd_chunk_scan_fwd over the workload (decay cumsum, intra-chunk quadratic
block, chunk states, state passing, state-to-output + D skip), then one
ssd_state_update continuing from the scan's final state with fresh
single-token inputs.  `value` counts the scan's tokens (batch x seqlen) per
second over all ranks.  Inputs already sit in HBM when the timed region
starts; x and y alone (671 MB for the default workload) exceed the 126 MB L2,
so no flush is needed between steps.

Multi-GPU: the path has no exchange step on one node's data-parallel axis, so
N ranks run N independent replicas (weak scaling), timed on the device and
reduced with max over ranks.

`--impl reference` times the fp64 CPU oracle on this host's cores on a
bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSD scan fwd tokens/s on 1 B200 + % of roofline (HBM GB/s, tensor-pipe util)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="mamba2_2.7b_layer")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seqpar", action="store_true",
                    help="split each sequence of the workload over the ranks (state passed along a ring); "
                         "default: every rank runs its own replica")
    ap.add_argument("--mixer", default=None, metavar="CONFIG",
                    help="time the head-sharded mixer layer (tensor parallel over the ranks, quantised "
                         "all-reduce) on this configuration, e.g. mixer_2.7b, instead of the scan")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward of the scan (ssd_chunk_scan_bwd) on the workload instead")
    ap.add_argument("--exact-allreduce", action="store_true",
                    help="with --mixer: an fp32 all-reduce instead of the quantised one")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (small cases for profiling; not a bench line)")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the workload's head count, a multiple of its groups (small cases for "
                         "profiling; not a bench line)")
    return ap.parse_args()


def workload_of(args):
    from state_space_model_07_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    if args.batch is not None and not w.packed_nseqs:
        w = inputs.scaled(w, batch=args.batch)
    if args.heads is not None:
        if args.heads <= 0 or args.heads % w.ngroups:
            raise SystemExit(f"--heads must be a positive multiple of the {w.ngroups} groups")
        w = inputs.scaled(w, nheads=args.heads)
    return w


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# --- algorithmic work per kernel launch -------------------------------------------------

def workload_bytes(w, S, L_tot, es):
    """Minimum HBM bytes of one scan: inputs read once, y written once, states."""
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups
    ntok = L_tot
    b = ntok * (2 * H * P * es + H * es + 2 * G * N * es)       # x + y, dt, B + C
    b += S * H * N * P * 4 * (2 if w.init_state else 1)          # final (+ init) state
    if w.packed_nseqs:
        b += ntok * 4                                            # seq_idx
    return b


def workload_flops(w, L_tot, Q):
    """Causal algorithmic flops of the chunked form (CB once per group)."""
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups
    per_tok_head = 2 * ((Q + 1) / 2) * P + 2 * N * P + 2 * N * P + 2 * N * P / Q
    per_tok_group = 2 * ((Q + 1) / 2) * N
    return L_tot * (H * per_tok_head + G * per_tok_group)


def decode_bytes(b, H, P, N, G, es):
    return b * H * N * P * 4 * 2 + b * H * (2 * P * es + es) + b * G * N * 2 * es


# --- clocks -----------------------------------------------------------------------------

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    def __init__(self, torch_device, period_s=0.0005):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            props = torch.cuda.get_device_properties(torch_device)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self._reasons()))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "err", "")}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        mask = 0
        for _, r in busy:
            mask |= r
        return {"sm_mhz": statistics.median([s[0] for s in busy]) if busy else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [n for bit, n in REASONS.items() if mask & bit and bit != 0x1]}


# --- the oracle on a bounded sample (reference arm / cpu baseline) ----------------------

_CPU_INPUTS = {}


def oracle_sample(w, heads, rows=None):
    """Runs the fp64 oracle on `heads` heads (all tokens) of the workload's
    first `rows` batch rows; returns (seconds, token-equivalents, threads)."""
    import oracle
    from state_space_model_07_b200 import inputs
    if (w.name, w.batch) not in _CPU_INPUTS:
        _CPU_INPUTS[(w.name, w.batch)] = inputs.make_inputs(w, "cpu")
    d = _CPU_INPUTS[(w.name, w.batch)]
    H, G = w.nheads, w.ngroups
    hs = list(range(heads))
    gs = [h // (H // G) for h in hs]
    rows = rows or d["x"].shape[0]
    sl = slice(0, rows)
    sub = dict(x=d["x"][sl][:, :, hs], dt=d["dt"][sl][:, :, hs], A=d["A"][hs], B=d["B"][sl][:, :, gs],
               C=d["C"][sl][:, :, gs], dt_bias=d["dt_bias"][hs], D=d["D"][hs],
               init_state=None if d["init_state"] is None else d["init_state"][:, hs])
    if d["seq_idx"] is None and sub["init_state"] is not None:
        sub["init_state"] = sub["init_state"][sl]
    threads = oracle.default_threads()
    args = dict(sub)
    t0 = time.perf_counter()
    oracle.ssd_scan(args["x"], args["dt"], args["A"], args["B"], args["C"], dt_bias=args["dt_bias"],
                    D=args["D"], init_state=args["init_state"], seq_idx=d["seq_idx"], nseqs=d["nseqs"],
                    nthreads=threads)
    dt = time.perf_counter() - t0
    ntok = rows * d["x"].shape[1]
    return dt, ntok * heads / H, threads


def cpu_baseline(w, target_s=8.0):
    heads = 1
    while True:
        secs, toks, threads = oracle_sample(w, heads)
        if secs >= target_s or heads >= w.nheads:
            break
        heads = min(w.nheads, max(heads * 2, int(heads * target_s / max(secs, 1e-3))))
    return {"value": toks / secs, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{heads} of {w.nheads} heads, all tokens of every sequence, fp64 token loop; "
                      f"{secs:.1f} s wall; value = tokens x (sampled heads / all heads) / s"}


# --- distributed plumbing ----------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(v, world, device):
    """Max of a per-rank float over all ranks (device-timed numbers are
    reported as the slowest rank's)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(tokens_per_rank, world, steps, ms):
    """Whole-job tokens/s: every rank processes its own replica of the workload."""
    return tokens_per_rank * world * steps / (ms * 1e-3)


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    w = workload_of(args)
    # Each step: the oracle on 2 heads of every sequence (a bounded sample).
    heads = max(1, min(w.nheads, 2))
    for _ in range(args.warmup):
        oracle_sample(w, heads)
    secs, toks, threads = [], 0.0, 1
    for _ in range(args.steps):
        s, t, threads = oracle_sample(w, heads)
        secs.append(s)
        toks = t
    total = sum(secs)
    value = toks * args.steps / total
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{heads} of {w.nheads} heads per step, all tokens; fp64 token loop"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w):
    c = {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "nheads": w.nheads, "headdim": w.headdim,
         "dstate": w.dstate, "ngroups": w.ngroups, "chunk": w.chunk, "input_dtype": w.dtype,
         "state_dtype": "f32", "parallelism": "replicas",
         "step": "ssd_chunk_scan_fwd over the workload + 1 ssd_state_update from its final state",
         "l2": "no flush: x and y alone exceed the 126 MB L2"}
    if w.packed_nseqs:
        c["packed_nseqs"] = w.packed_nseqs
    return c


# Definitions in a source file that belong only to kernels other than the one a
# capture measured: removed before hashing.  ssd_tc.cu also holds the
# first-generation k_tc_scan<N> (the d_state 256 kernel), its shared-memory
# layout TcSmem<N> and its constants Cfg<N>, none of which the measured
# k_tc_scan3 uses.
_NOT_MEASURED = {"tc_scan": (("template <int N>", "k_tc_scan(const __grid_constant__"),
                             ("template <int N>", "struct __align__(1024) TcSmem {"),
                             ("template <int N>", "struct Cfg {"))}


def _drop_definition(code, head, signature):
    """`code` without the definition whose signature contains `signature`, from
    the nearest `head` before it to its closing brace."""
    i = code.find(signature)
    if i < 0:
        return code
    start = code.rfind(head, 0, i)
    depth = 0
    for k in range(code.index("{", i), len(code)):
        depth += {"{": 1, "}": -1}.get(code[k], 0)
        if depth == 0:
            return code[:start] + code[k + 1:]
    return code


def kernel_source_sha(name):
    """Hash of the kernel's source with comments and blank lines removed, so
    that a recorded DRAM capture stays attached to the code it measured and
    drops off as soon as the code (not its comments) changes."""
    import re
    src = {"tc_scan": "ssd_tc.cu", "tc_prep": "ssd_tc.cu", "simt_chunk_out": "ssd_simt.cu",
           "state_update": "ssd_decode.cu"}.get(name)
    if not src:
        return None
    p = os.path.join(ROOT, "state_space_model_07_b200", "csrc", src)
    with open(p, encoding="utf-8") as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    code = "\n".join(line.rstrip() for line in text.splitlines() if line.strip())
    for head, signature in _NOT_MEASURED.get(name, ()):
        code = _drop_definition(code, head, signature)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def traffic_for(name, units_per_launch):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the kernel as it stands (same source hash); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f).get(name)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha") != kernel_source_sha(name):
        return None
    return rec["dram_bytes"] * units_per_launch / rec["units"]


def run_ours(args):
    import torch
    import torch.distributed as dist
    import state_space_model_07_b200 as ssd
    from state_space_model_07_b200 import _lib, inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    w = workload_of(args)
    d = inputs.make_inputs(w, dev)
    b, L, H, P = d["x"].shape
    N, G, S = w.dstate, w.ngroups, d["nseqs"]
    es = d["x"].element_size()
    y = torch.empty_like(d["x"])
    fs = torch.empty((S, H, N, P), dtype=torch.float32, device=dev)
    dec = [inputs.make_decode_inputs(w, k, S if w.packed_nseqs else b, dev) for k in range(4)]
    dec_y = torch.empty_like(dec[0]["x"])
    stream = torch.cuda.current_stream(dev)

    def step(k, xs=None, yout=None):
        src = xs or d
        ssd.chunk_scan_fwd(src["x"], src["dt"], d["A"], src["B"], src["C"], dt_bias=d["dt_bias"], D=d["D"],
                           init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=S, chunk=w.chunk,
                           y=y if yout is None else yout, final_state=fs)
        dd = dec[k % len(dec)]
        ssd.state_update(fs, dd["x"], dd["dt"], d["A"], dd["B"], dd["C"], D=d["D"], dt_bias=d["dt_bias"],
                         y=dec_y)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    # clocks are sampled through the warm-up steps and the timed region (both keep the GPU busy),
    # so that a short timed region still has several samples under load.  The timed region runs
    # the steps as a user would, without the library's per-kernel event records (they add about
    # 17 us to a 0.43 ms step); the per-kernel figures come from a second, profiled run of the
    # same steps right after it.
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        for k in range(args.warmup):
            step(k)
        barrier()
        e0.record(stream)
        for k in range(args.steps):
            step(k)
        e1.record(stream)
        barrier()
        _lib.profile_read(reset=True)
        _lib.profile_enable(True)
        for k in range(args.steps):
            step(k)
        barrier()
    _lib.profile_enable(False)
    stats = _lib.profile_read(reset=True)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_step = ms / args.steps
    tokens = b * L if not w.packed_nseqs else L
    value = throughput(tokens, world, args.steps, ms)
    launches = sum(v[0] for v in stats.values())

    pk, pk_src = peaks()
    # dominant kernel; a long sequence with few heads runs the scan kernel twice per step (the
    # two-pass segment split), so the algorithmic bytes of a step are set against the kernel's
    # whole time per step
    dom = max(stats.items(), key=lambda kv: kv[1][2])
    name, (nl, nt, tot_ms) = dom
    per_step = max(1, round(nl / args.steps))
    avg_ms = tot_ms / max(nt, 1) * per_step
    scan_bytes = workload_bytes(w, S, tokens, es)
    if name in ("tc_scan", "simt_chunk_out"):
        alg_bytes = scan_bytes
        units = tokens
    elif name == "state_update":
        alg_bytes = decode_bytes(S, H, P, N, G, es)
        units = S * H
    else:
        alg_bytes, units = scan_bytes, tokens
    roof = {"kernel": name, "bound": "hbm", "achieved": alg_bytes / (avg_ms * 1e-3) / 1e9,
            "peak": pk["hbm_gbs"], "unit": "GB/s", "peak_source": pk_src,
            "avg_launch_ms": avg_ms / per_step, "launches": nl, "launches_per_step": per_step,
            "algorithmic_bytes_per_launch": alg_bytes / per_step,
            "traffic": traffic_for(name, units) if per_step == 1 else None}
    roof["frac"] = roof["achieved"] / roof["peak"]
    # the same against the nominal 8 TB/s HBM3e figure (context; the measured copy peak is the target)
    roof["frac_of_nominal_8000_gbs"] = roof["achieved"] / 8000.0
    flops = workload_flops(w, tokens, w.chunk)
    roof["tensor_equiv"] = {"algorithmic_flops": flops, "achieved_tflops": flops / (avg_ms * 1e-3) / 1e12,
                            "peak_tflops": pk["bf16_tflops"]}
    per_kernel = {k: {"launches": v[0], "avg_ms": v[2] / max(v[1], 1)} for k, v in stats.items()}
    # decode kernel on its own (part of the step)
    if "state_update" in stats:
        su = stats["state_update"]
        su_ms = su[2] / max(su[1], 1)
        per_kernel["state_update"]["achieved_gbs"] = decode_bytes(S, H, P, N, G, es) / (su_ms * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        # End to end through the public API with host buffers: every step copies its inputs
        # from pinned host memory, runs the scan + decode step, and copies y back.  Steps are
        # pipelined the way a serving loop would run them: copies in on one stream, compute on
        # another, copies out on a third, with two device buffer sets so that step k + 1's
        # inputs and step k - 1's output cross PCIe while step k computes.
        host = {k: d[k].cpu().pin_memory() for k in ("x", "dt", "B", "C")}
        bufs = [{k: torch.empty_like(d[k]) for k in host} for _ in range(2)]
        ys = [torch.empty_like(y) for _ in range(2)]
        y_hosts = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        n_e2e = max(2, min(args.steps, 20))
        for b in range(2):
            for kk in host:
                bufs[b][kk].copy_(host[kk])
        step(0, bufs[0], ys[0])
        barrier()
        ev = lambda: torch.cuda.Event(enable_timing=True)
        in_done = [ev() for _ in range(n_e2e)]
        comp_done = [ev() for _ in range(n_e2e)]
        out_done = [ev() for _ in range(n_e2e)]
        f0 = ev()
        f0.record(s_in)
        s_comp.wait_event(f0)
        s_out.wait_event(f0)
        for k in range(n_e2e):
            b = k % 2
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(comp_done[k - 2])     # buffer set b read by step k - 2
                for kk in host:
                    bufs[b][kk].copy_(host[kk], non_blocking=True)
                in_done[k].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_done[k])
                if k >= 2:
                    s_comp.wait_event(out_done[k - 2])    # ys[b] copied out by step k - 2
                step(k, bufs[b], ys[b])
                comp_done[k].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[k])
                y_hosts[b].copy_(ys[b], non_blocking=True)
                out_done[k].record(s_out)
        barrier()
        e_ms = max_over_ranks(f0.elapsed_time(out_done[-1]), world, dev)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        e2e = {"value": throughput(tokens, world, n_e2e, e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": y.numel() * y.element_size(),
               "steps": n_e2e, "path": "pinned host -> device copies, ssd_chunk_scan_fwd + ssd_state_update "
                                       "through the C ABI, y copied back; copies in, compute and copies out "
                                       "on three streams with two device buffer sets (step k + 1 in and "
                                       "step k - 1 out overlap step k)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if es == 2 else "f32", "data": "synthetic",
            "config": config_of(w), "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "kernels": per_kernel, "clocks": clk.summary()}
    line["config"]["timing"] = ("timed steps run without per-kernel events; kernels, roofline and "
                                "gpu_launches from an identical profiled run of the same steps")
    print(json.dumps(line), flush=True)
    return 0


def run_seqpar(args):
    """One scan of the workload split along the sequence over the ranks: rank r holds tokens
    [r L/N, (r + 1) L/N) of every batch row, scans them, receives the state entering its slice
    from rank r - 1 (NCCL point-to-point), passes the state leaving it on and adds the output of
    the state it received (state_space_model_07_b200.seqpar).  Total work is fixed as N grows."""
    import torch
    import torch.distributed as dist
    from state_space_model_07_b200 import _lib, inputs, seqpar

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    w = workload_of(args)
    if w.packed_nseqs:
        raise SystemExit("--seqpar splits batch rows; packed workloads are not supported")
    d = inputs.make_inputs(w, dev)
    b, L, H, P = d["x"].shape
    lo, hi = rank * L // world, (rank + 1) * L // world
    part = {k: d[k][:, lo:hi].contiguous() for k in ("x", "dt", "B", "C")}
    del d["x"], d["B"], d["C"]
    comm = seqpar.TorchDistComm() if world > 1 else seqpar.LocalRing(1)
    stream = torch.cuda.current_stream(dev)

    def step():
        return seqpar.chunk_scan_fwd_seqpar(part["x"], part["dt"], d["A"], part["B"], part["C"], comm=comm,
                                            dt_bias=d["dt_bias"], D=d["D"], init_state=d["init_state"],
                                            chunk=w.chunk)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        for _ in range(args.warmup):
            step()
        barrier()
        _lib.profile_read(reset=True)
        _lib.profile_enable(True)
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
    _lib.profile_enable(False)
    stats = _lib.profile_read(reset=True)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    tokens = b * L
    value = tokens * args.steps / (ms * 1e-3)
    pk, pk_src = peaks()
    nl, nt, tot = stats.get("tc_scan", stats.get("simt_chunk_out", (0, 0, 0.0)))
    per_step = max(1, round(nl / args.steps))
    step_ms = tot / max(nt, 1) * per_step
    alg = workload_bytes(inputs.scaled(w, seqlen=hi - lo), b, b * (hi - lo), part["x"].element_size())
    roof = {"kernel": "tc_scan", "bound": "hbm", "achieved": alg / (step_ms * 1e-3) / 1e9 if step_ms else None,
            "peak": pk["hbm_gbs"], "unit": "GB/s", "peak_source": pk_src, "avg_launch_ms": step_ms / per_step,
            "launches": nl, "launches_per_step": per_step, "algorithmic_bytes_per_step_of_the_slice": alg,
            "traffic": None}
    roof["frac"] = roof["achieved"] / roof["peak"] if roof["achieved"] else None
    launches = sum(v[0] for v in stats.values())
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    cfg = config_of(w)
    cfg.update(parallelism=f"seqpar{world}", step="one ssd_chunk_scan_fwd of the workload split along the "
               "sequence over the ranks: local scan, state ring (NCCL send / recv), the entering state's "
               "output added on ranks >= 1",
               tokens_per_rank=hi - lo)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16" if part["x"].element_size() == 2 else "f32", "data": "synthetic",
            "config": cfg, "roofline": roof, "cpu_baseline": None,
            "e2e": None, "e2e_note": "sequence-parallel mode times device-resident slices only",
            "gpu_launches": launches, "kernels": {k: {"launches": v[0], "avg_ms": v[2] / max(v[1], 1)}
                                                  for k, v in stats.items()},
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def bwd_flops(w, tokens):
    """Multiply-adds of the chunked backward (64-token chunks, as evaluated) x 2: per token and
    head the chunk's state and adjoint terms (2 N P), dy x^T and W^T dy (2 Q P), B dh_end and
    C h_prev (2 N P), K^T C, K B (2 Q N) and x dh_end^T, dy h_prev^T (2 P N); per token and group
    C B^T (Q N)."""
    Q, P, N, H, G = 64, w.headdim, w.dstate, w.nheads, w.ngroups
    per_head = 2 * N * P + 2 * Q * P + 2 * N * P + 2 * Q * N + 2 * P * N
    return 2.0 * tokens * (H * per_head + G * Q * N)


def run_bwd(args):
    """The backward of the scan on the workload (one GPU; replicas under torchrun): dx, ddt, dB,
    dC, ddt_bias, dA, dD and the initial state's gradient from a seeded upstream gradient dy (and
    dfinal where the workload has an initial state)."""
    import torch
    import torch.distributed as dist
    import state_space_model_07_b200 as ssd
    from state_space_model_07_b200 import _lib, inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    w = workload_of(args)
    d = inputs.make_inputs(w, dev)
    gen = torch.Generator(device="cpu").manual_seed(7)
    dy = torch.randn(d["x"].shape, generator=gen).to(d["x"].dtype).to(dev)
    dfinal = None
    if d["init_state"] is not None:
        dfinal = torch.randn(d["init_state"].shape, generator=gen).to(dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        return ssd.chunk_scan_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, dt_bias=d["dt_bias"], D=d["D"],
                                  init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=d["nseqs"], chunk=w.chunk,
                                  dfinal=dfinal)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        for _ in range(args.warmup):
            step()
        barrier()
        _lib.profile_read(reset=True)
        _lib.profile_enable(True)
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
    _lib.profile_enable(False)
    stats = _lib.profile_read(reset=True)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    tokens = int(d["x"].shape[0] * d["x"].shape[1])
    value = tokens * world * args.steps / (ms * 1e-3)
    pk, pk_src = peaks()
    step_ms = ms / args.steps
    flops = bwd_flops(w, tokens)
    es = d["x"].element_size()
    bytes_ = es * tokens * (w.nheads * (3 * w.headdim + 2) + 4 * w.ngroups * w.dstate)   # x, dy, dx; dt, ddt; B, C, dB, dC
    line = {"metric": "SSD scan backward tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if es == 2 else "f32", "data": "synthetic",
            "config": dict(config_of(w), step="ssd_chunk_scan_bwd over the workload (dy seeded)",
                           parallelism=f"replicas{world}"),
            "roofline": {"bound": "tensor", "algorithmic_flops": flops, "achieved": flops / (step_ms * 1e-3) / 1e12,
                         "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "peak_source": pk_src,
                         "frac": flops / (step_ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                         "hbm_min_bytes": bytes_, "hbm_frac": bytes_ / (step_ms * 1e-3) / 1e9 / pk["hbm_gbs"]},
            "cpu_baseline": None, "e2e": None,
            "gpu_launches": sum(v[0] for v in stats.values()),
            "kernels": {k: {"launches": v[0], "avg_ms": v[2] / max(v[1], 1)} for k, v in stats.items()},
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_mixer(args):
    """The head-sharded mixer layer ("5.3 Tensor Parallelism support and large-cluster training",
    section 4.1) on the ranks: each holds H / N heads, computes its projections (cuBLAS), scan and
    group norm (library kernels) and its partial output projection, and the partials are summed by
    the quantised all-reduce (library quantisation kernels; all-to-all and all-gather over NCCL).
    Every rank holds the whole input; total work is fixed as N grows."""
    import torch
    import torch.distributed as dist
    from state_space_model_07_b200 import _lib, inputs, tp

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    cfg = inputs.MIXERS[args.mixer]
    if args.batch:
        cfg = inputs.dataclasses.replace(cfg, batch=args.batch)
    u, w = inputs.make_mixer(cfg, dev)
    sh = tp.shard(w, rank, world)
    del w
    comm = tp.TorchDistTPComm() if world > 1 else tp.SingleRankComm()
    quantized = not args.exact_allreduce
    stream = torch.cuda.current_stream(dev)

    def step():
        return tp.mixer_fwd(u, sh, comm, ngroups=cfg.ngroups, dstate=cfg.dstate, headdim=cfg.headdim,
                            chunk=cfg.chunk, quantized=quantized)

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        for _ in range(args.warmup):
            step()
        barrier()
        _lib.profile_read(reset=True)
        _lib.profile_enable(True)
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
    _lib.profile_enable(False)
    stats = _lib.profile_read(reset=True)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    T = cfg.batch * cfg.seqlen
    value = T * args.steps / (ms * 1e-3)
    launches = sum(v[0] for v in stats.values())
    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    Hr = cfg.nheads // world
    gemm_flops = 2 * T * cfg.d_model * (Hr * cfg.headdim * 2 + 2 * cfg.ngroups // world * cfg.dstate + Hr)
    code_bytes = 2 * (world - 1) / world * T * cfg.d_model * (1 + 4 / 64)
    pk, pk_src = peaks()
    line = {"metric": "head-sharded SSD mixer layer tokens/s (tensor parallel over the GPUs)", "value": value,
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "batch": cfg.batch, "seqlen": cfg.seqlen, "d_model": cfg.d_model,
                       "nheads": cfg.nheads, "headdim": cfg.headdim, "dstate": cfg.dstate,
                       "ngroups": cfg.ngroups, "chunk": cfg.chunk, "parallelism": f"tp{world}",
                       "allreduce": "int8 codes, one fp32 scale per 64 columns" if quantized else "fp32",
                       "step": "input projections (cuBLAS), scan and group norm of the rank's heads, partial "
                               "output projection, all-reduce of the partials"},
            "per_rank": {"heads": Hr, "gemm_flops": gemm_flops,
                         "allreduce_bytes_sent": code_bytes if quantized else 2 * (world - 1) / world * T *
                         cfg.d_model * 4},
            "roofline": None, "cpu_baseline": None, "e2e": None,
            "note": "the layer around the scan: GEMMs by cuBLAS; the scan's own roofline is the scan line's",
            "gpu_launches": launches, "kernels": {k: {"launches": v[0], "avg_ms": v[2] / max(v[1], 1)}
                                                  for k, v in stats.items()},
            "peaks": {"source": pk_src}, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.seqpar:
        return run_seqpar(args)
    if args.mixer:
        return run_mixer(args)
    if args.bwd:
        return run_bwd(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
