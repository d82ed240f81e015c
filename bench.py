#!/usr/bin/env python
"""Benchmark of the DISCO convolution hot path on B200.

One step is one pass of the whole hot path over one batch of the workload:
the sparse Psi contraction (x -> y), the weight einsum (y -> out), the fused
forward (x -> out, y never stored), the input gradient (dout -> dx) and the
weight gradient (dout, y -> dw, dbias).  The metric is grid-points x channels
per second: each op counts the points x channels of the tensor it produces
(out for the forward ops and for dw, dx for the input gradient).

Default workload: the 721x1440 weather-scale layer (B1, C 64->64, isotropic
K=3, theta_c = 2*pi/720, bf16 storage).  Its x (133 MB) and y (399 MB) are
larger than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl disco|reference]

With N > 1 (torchrun, one process per GPU) every rank runs an independent
batch (weak scaling, no collective on the data path); the timed region is
bracketed by a barrier and synchronisation and the max over ranks is used.
`--impl reference` times the CPU oracle (fp64, OpenMP) on a bounded channel
sample of the same workload, on rank 0 only.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DISCO conv fwd/bwd grid-points·channels/s and % HBM roofline on 1 B200"
UNIT = "grid-points*channels/s"
PSI_ENTRY_BYTES = 13  # algorithmic Psi bytes per entry: fp32 value + int32 i + int32 p + int8 k
OPS = ("contract", "einsum", "fused", "dx", "dw")
# single-launch kernels of the step, timed one by one for the roofline: the contraction, the weight
# einsum, the fused forward and the input gradient (one launch on this layer: the transposed
# contraction of dout with the mix by W^T in its epilogue)
KERNELS = ("contract", "einsum", "fused", "dx")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="disco", choices=["disco", "reference"])
    ap.add_argument("--workload", default="weather")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the activation-memory and other-workload records")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers

def units_per_step(wl) -> dict:
    n_out = wl.B * wl.C_out * wl.nlat_out * wl.nlon_out
    return {"contract": 0, "einsum": n_out, "fused": n_out, "dx": wl.B * wl.C_in * wl.nlat_in * wl.nlon_in,
            "dw": n_out}


def algorithmic_bytes(wl, nnz: int) -> dict:
    """Bytes each op must move at least once (storage width), per launch."""
    es = 2 if wl.dtype == "bf16" else 4
    x = wl.B * wl.C_in * wl.nlat_in * wl.nlon_in * es
    y = wl.B * wl.C_in * wl.K * wl.nlat_out * wl.nlon_out * es
    out = wl.B * wl.C_out * wl.nlat_out * wl.nlon_out * es
    w = wl.C_out * (wl.C_in // wl.groups) * wl.K * es
    b = wl.C_out * es
    psi = nnz * PSI_ENTRY_BYTES
    return {"contract": x + psi + y, "einsum": y + w + b + out, "fused": x + psi + w + b + out,
            "dx": out + w + psi + x, "dw": out + y + w + b}


def measured_peaks() -> tuple:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def source_digest(files) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[kernel]
    except Exception:
        return None
    if rec.get("workload") != workload or rec.get("source_digest") != source_digest(rec.get("sources", [])):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 6:
                self.samples.append(parts)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[2 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


def dist_setup():
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    return world, rank, local


def aggregate(elapsed_ms: float, units: float, world: int, device=None):
    """(max elapsed over ranks, total units over ranks); identity with one rank."""
    if world == 1:
        return elapsed_ms, units
    import torch
    import torch.distributed as dist

    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# ----------------------------------------------------------- CPU oracle leg

def cpu_sample_workload(wl):
    """A bounded channel sample of the workload (same grid and basis)."""
    c = 4 if wl.C_in >= 4 else wl.C_in
    g = 1
    return wl.scaled(B=1, C_in=c, C_out=c, groups=g)


def oracle_steps(wl, steps, warmup: int, min_seconds: float = 0.0, threads: int = 0):
    """Times the CPU oracle on the channel sample: per step forward, forward again (the fused mode
    computes the same out), dx, dw.  With min_seconds, repeats steps until that much time has passed;
    threads > 0 sets the oracle's OpenMP thread count first.
    Returns (units per second, cores, sample description, seconds, steps)."""
    import oracle
    from spherical_disco_convolution_b200.workloads import make_inputs

    sw = cpu_sample_workload(wl)
    inp = make_inputs(sw, 0)
    P = oracle.Psi(oracle.Spec(sw.nlat_in, sw.nlon_in, sw.nlat_out, sw.nlon_out, sw.kernel_shape[0],
                               sw.kernel_shape[1], sw.theta_cutoff))
    if threads > 0:
        oracle.set_num_threads(threads)

    def step():
        P.forward(inp["x"], inp["w"], inp["bias"], groups=sw.groups)
        P.forward(inp["x"], inp["w"], inp["bias"], groups=sw.groups)
        P.backward_input(inp["dout"], inp["w"], sw.C_in, groups=sw.groups)
        P.backward_weight(inp["dout"], inp["x"], groups=sw.groups)

    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    done = 0
    while done < steps or time.perf_counter() - t0 < min_seconds:
        step()
        done += 1
    dt = time.perf_counter() - t0
    u = sum(units_per_step(sw).values()) * done
    desc = (f"oracle fp64 on B={sw.B}, C {sw.C_in}->{sw.C_out} of the {sw.nlat_in}x{sw.nlon_in} grid "
            f"(Psi build untimed), {done} step(s) of fwd+fwd+dx+dw in {dt:.1f} s")
    return u / dt, oracle.num_threads(), desc, dt, done


def cpu_baseline(wl) -> dict:
    """The oracle timed on all host cores and on one thread, median of three runs each, on a
    channel sample of the workload (about 20-40 s of CPU work in all)."""
    import oracle

    cores = os.cpu_count() or 1
    runs_all = [oracle_steps(wl, 1, 1 if i == 0 else 0, min_seconds=2.0, threads=cores) for i in range(3)]
    runs_one = [oracle_steps(wl, 1, 0, threads=1) for _ in range(3)]
    oracle.set_num_threads(cores)
    v_all = statistics.median(r[0] for r in runs_all)
    v_one = statistics.median(r[0] for r in runs_one)
    sw = cpu_sample_workload(wl)
    note = (f"{runs_all[0][2]}; median of 3 runs on {cores} threads, and of 3 one-step runs on 1 thread "
            f"({v_one:.4g} {UNIT}).  The sample has {sw.C_in} of {wl.C_in} channels: the oracle's weight "
            f"einsum costs C_in/G*K = {sw.C_in // sw.groups * sw.K} multiply-adds per output point here "
            f"against {wl.C_in // wl.groups * wl.K} on the full layer, so the sample overstates its "
            f"throughput there")
    return {"value": v_all, "unit": UNIT, "cores": runs_all[0][1], "kind": "oracle", "sample": note,
            "one_thread": {"value": v_one, "unit": UNIT, "cores": 1}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from spherical_disco_convolution_b200.workloads import WORKLOADS

    wl = WORKLOADS[args.workload]
    value, cores, desc, dt, _ = oracle_steps(wl, max(1, args.steps), max(0, args.warmup))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * dt / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl) -> dict:
    return {"workload": f"{wl.name} {wl.nlat_in}x{wl.nlon_in}->{wl.nlat_out}x{wl.nlon_out} B{wl.B} "
                        f"C{wl.C_in}->{wl.C_out} G{wl.groups} K{wl.K} {wl.dtype}",
            "B": wl.B, "C_in": wl.C_in, "C_out": wl.C_out, "groups": wl.groups,
            "in_shape": [wl.nlat_in, wl.nlon_in], "out_shape": [wl.nlat_out, wl.nlon_out],
            "kernel_shape": list(wl.kernel_shape), "theta_cutoff": wl.theta_cutoff,
            "step": "contract + einsum + fused forward + dx + dw/dbias",
            "l2": "inputs larger than L2 (x and y exceed 126 MB); no flush"}


# ------------------------------------------------------ extra GPU records

def activation_memory(wl, dev, dt, x) -> dict:
    """What the autograd layer keeps for backward after one forward, unfused (y) and fused (x, which
    the caller holds anyway): torch allocator bytes after the forward minus before it, less out."""
    import torch

    from spherical_disco_convolution_b200 import conv

    res = {}
    for fused in (False, True):
        layer = conv.DiscreteContinuousConvS2(wl.C_in, wl.C_out, (wl.nlat_in, wl.nlon_in), (wl.nlat_out, wl.nlon_out),
                                              wl.kernel_shape, groups=wl.groups, theta_cutoff=wl.theta_cutoff,
                                              fused=fused, device=dev, dtype=dt)
        torch.cuda.synchronize(dev)
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        out = layer(x)
        torch.cuda.synchronize(dev)
        kept = torch.cuda.memory_allocated(dev) - base - out.numel() * out.element_size()
        peak = torch.cuda.max_memory_allocated(dev) - base
        res["fused" if fused else "unfused"] = (kept / 1e6, peak / 1e6)
        del out, layer
        torch.cuda.synchronize(dev)
    es = 2 if wl.dtype == "bf16" else 4
    y_mb = wl.B * wl.C_in * wl.K * wl.nlat_out * wl.nlon_out * es / 1e6
    return {"unfused_mb": res["unfused"][0], "fused_mb": res["fused"][0],
            "saving_mb": res["unfused"][0] - res["fused"][0], "y_mb": y_mb,
            "forward_peak_mb": {"unfused": res["unfused"][1], "fused": res["fused"][1]},
            "how": "torch.cuda.memory_allocated after minus before one autograd forward, less out"}


def workload_record(name: str, dev, steps: int = 5, warmup: int = 3) -> dict:
    """Per-op times of another workload (same ops as the headline step, CUDA events on the
    launching stream, median over the timed steps) with GB/s and the HBM roofline fraction."""
    import numpy as np
    import torch

    from spherical_disco_convolution_b200 import conv
    from spherical_disco_convolution_b200 import disco as D
    from spherical_disco_convolution_b200.workloads import WORKLOADS, make_inputs

    wl = WORKLOADS[name]
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dcode = D.DISCO_BF16 if wl.dtype == "bf16" else D.DISCO_F32
    psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, dev)
    inp = make_inputs(wl, 0)
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dt).to(dev) for k, v in inp.items() if v is not None}
    sh = wl.shapes()
    y = torch.empty(sh["y"], dtype=dt, device=dev)
    out, out_f = (torch.empty(sh["out"], dtype=dt, device=dev) for _ in range(2))
    dx = torch.empty(sh["x"], dtype=dt, device=dev)
    dw = torch.empty(sh["w"], dtype=dt, device=dev)
    db = torch.empty(sh["bias"], dtype=dt, device=dev) if "bias" in t else None
    ws_dx, n_dx = psi.workspace(D.DISCO_OP_BWD_INPUT, wl.B, wl.C_in, wl.C_out, wl.groups, dcode)
    ws_dw, n_dw = psi.workspace(D.DISCO_OP_BWD_WEIGHT, wl.B, wl.C_in, wl.C_out, wl.groups, dcode)
    stream = torch.cuda.current_stream(dev)
    st = stream.cuda_stream
    p = lambda v: None if v is None else v.data_ptr()  # noqa: E731
    h, B, Ci, Co, G = psi.handle, wl.B, wl.C_in, wl.C_out, wl.groups
    calls = [
        ("contract", lambda: D.disco_contract(h, B, Ci, dcode, p(t["x"]), p(y), st)),
        ("einsum", lambda: D.disco_einsum(h, B, Ci, Co, G, dcode, p(y), p(t["w"]), p(t.get("bias")), p(out), st)),
        ("fused", lambda: D.disco_fwd_fused(h, B, Ci, Co, G, dcode, p(t["x"]), p(t["w"]), p(t.get("bias")),
                                            p(out_f), None, 0, st)),
        ("dx", lambda: D.disco_bwd_input(h, B, Ci, Co, G, dcode, p(t["dout"]), p(t["w"]), p(dx), p(ws_dx), n_dx, st)),
        ("dw", lambda: D.disco_bwd_weight(h, B, Ci, Co, G, dcode, p(t["dout"]), p(y), None, p(dw), p(db), p(ws_dw),
                                          n_dw, st)),
    ]
    for _ in range(warmup):
        for _, c in calls:
            c()
    torch.cuda.synchronize(dev)
    ms = {k: [] for k, _ in calls}
    for _ in range(steps):
        for k, c in calls:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            c()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ms[k].append(e0.elapsed_time(e1))
    peak, _ = measured_peaks()
    alg = algorithmic_bytes(wl, psi.nnz)
    ups = units_per_step(wl)
    ops = {}
    for k, _ in calls:
        m = statistics.median(ms[k])
        ops[k] = {"ms": m, "GBps": alg[k] / (m * 1e-3) / 1e9, "frac_hbm": alg[k] / (m * 1e-3) / 1e9 / peak,
                  "alg_bytes": alg[k]}
        if ups[k]:
            ops[k]["units_per_s"] = ups[k] / (m * 1e-3)
    train = ops["contract"]["ms"] + ops["einsum"]["ms"] + ops["dx"]["ms"] + ops["dw"]["ms"]
    return {"config": workload_config(wl), "ops": ops, "training_step_ms": train,
            "training_step": "contract + einsum + dx + dw (the unfused forward and the backward)",
            "l2": "no flush: the step's tensors exceed 126 MB" if wl.name == "grouped" else
                  "no flush between ops; inputs of this layer fit L2, so these times can include L2 hits"}


# ------------------------------------------------------------------ GPU arm

def run_gpu(args):
    import numpy as np
    import torch

    from spherical_disco_convolution_b200 import conv
    from spherical_disco_convolution_b200 import disco as D
    from spherical_disco_convolution_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = WORKLOADS[args.workload]
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dcode = D.DISCO_BF16 if wl.dtype == "bf16" else D.DISCO_F32

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)  # before any GPU work starts

    psi = conv.Psi(wl.nlat_in, wl.nlon_in, wl.nlat_out, wl.nlon_out, wl.kernel_shape, wl.theta_cutoff, dev)
    inp = make_inputs(wl, seed=rank)
    host = {k: torch.from_numpy(np.ascontiguousarray(v)).to(dt).pin_memory() for k, v in inp.items()
            if v is not None}
    x, w, dout = (host[k].to(dev) for k in ("x", "w", "dout"))
    bias = host["bias"].to(dev) if "bias" in host else None
    sh = wl.shapes()
    y = torch.empty(sh["y"], dtype=dt, device=dev)
    out = torch.empty(sh["out"], dtype=dt, device=dev)
    out_f = torch.empty_like(out)
    dx = torch.empty(sh["x"], dtype=dt, device=dev)
    dw = torch.empty(sh["w"], dtype=dt, device=dev)
    db = torch.empty(sh["bias"], dtype=dt, device=dev) if bias is not None else None
    ws_dx, n_dx = psi.workspace(D.DISCO_OP_BWD_INPUT, wl.B, wl.C_in, wl.C_out, wl.groups, dcode)
    ws_dw, n_dw = psi.workspace(D.DISCO_OP_BWD_WEIGHT, wl.B, wl.C_in, wl.C_out, wl.groups, dcode)
    stream = torch.cuda.current_stream(dev)
    st = stream.cuda_stream
    p = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    h = psi.handle
    B, Ci, Co, G = wl.B, wl.C_in, wl.C_out, wl.groups

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        D.disco_contract(h, B, Ci, dcode, p(x), p(y), st)
        if ev:
            ev[1].record(stream)
        D.disco_einsum(h, B, Ci, Co, G, dcode, p(y), p(w), p(bias), p(out), st)
        if ev:
            ev[2].record(stream)
        D.disco_fwd_fused(h, B, Ci, Co, G, dcode, p(x), p(w), p(bias), p(out_f), None, 0, st)
        if ev:
            ev[3].record(stream)
        D.disco_bwd_input(h, B, Ci, Co, G, dcode, p(dout), p(w), p(dx), p(ws_dx), n_dx, st)
        if ev:
            ev[4].record(stream)
        D.disco_bwd_weight(h, B, Ci, Co, G, dcode, p(dout), p(y), None, p(dw), p(db), p(ws_dw), n_dw, st)
        if ev:
            ev[5].record(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    n0 = D.disco_launch_count()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    launches = D.disco_launch_count() - n0
    clk = clocks.stop()
    barrier()
    elapsed = t0.elapsed_time(t1)
    ups = units_per_step(wl)
    units = sum(ups.values()) * args.steps
    el_max, units_all = aggregate(elapsed, units, world, dev)
    span = lambda i, j: statistics.mean(e[i].elapsed_time(e[j]) for e in evs)  # noqa: E731
    op_ms = {"contract": span(0, 1), "einsum": span(1, 2), "fused": span(2, 3), "dx": span(3, 4), "dw": span(4, 5)}
    kern_ms = {"contract": op_ms["contract"], "einsum": op_ms["einsum"], "fused": op_ms["fused"], "dx": op_ms["dx"]}

    # end to end through the C ABI from pinned host buffers: inputs in, results out, every step
    e2e = None
    if not args.no_e2e:
        res_host = {"out": torch.empty(sh["out"], dtype=dt).pin_memory(),
                    "out_f": torch.empty(sh["out"], dtype=dt).pin_memory(),
                    "dx": torch.empty(sh["x"], dtype=dt).pin_memory(),
                    "dw": torch.empty(sh["w"], dtype=dt).pin_memory()}
        if db is not None:
            res_host["db"] = torch.empty(sh["bias"], dtype=dt).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in res_host.values())

        def e2e_step():
            x.copy_(host["x"], non_blocking=True)
            w.copy_(host["w"], non_blocking=True)
            dout.copy_(host["dout"], non_blocking=True)
            if bias is not None:
                bias.copy_(host["bias"], non_blocking=True)
            step()
            res_host["out"].copy_(out, non_blocking=True)
            res_host["out_f"].copy_(out_f, non_blocking=True)
            res_host["dx"].copy_(dx, non_blocking=True)
            res_host["dw"].copy_(dw, non_blocking=True)
            if db is not None:
                res_host["db"].copy_(db, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_max, e_units = aggregate(a0.elapsed_time(a1), units, world, dev)
        e2e = {"value": e_units / (e_max / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}

    if rank != 0:
        return 0
    extra = {}
    if world == 1 and not args.no_extra:
        extra["activation_memory"] = activation_memory(wl, dev, dt, x)
        for name in ("grouped", "downsample"):
            if name != wl.name:
                extra[name] = workload_record(name, dev)
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(wl, psi.nnz)
    ops = {op: {"ms": op_ms[op], "GBps": alg[op] / (op_ms[op] * 1e-3) / 1e9,
                "frac_hbm": alg[op] / (op_ms[op] * 1e-3) / 1e9 / peak, "alg_bytes": alg[op]} for op in OPS}
    kernels = {k: {"ms": kern_ms[k], "GBps": alg[k] / (kern_ms[k] * 1e-3) / 1e9,
                   "frac_hbm": alg[k] / (kern_ms[k] * 1e-3) / 1e9 / peak, "alg_bytes": alg[k]} for k in KERNELS}
    dom = max(KERNELS, key=lambda k: kern_ms[k])  # the longest single launch of the step
    traffic = recorded_traffic(dom, wl.name)
    roof = {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["GBps"], "peak": peak, "unit": "GB/s",
            "frac": kernels[dom]["frac_hbm"], "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs",
            "headline_contract": {"achieved": kernels["contract"]["GBps"], "frac": kernels["contract"]["frac_hbm"],
                                  "traffic": recorded_traffic("contract", wl.name)}}
    line = {
        "metric": METRIC, "value": units_all / (el_max / 1000.0), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": el_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": workload_config(wl), "roofline": roof, "ops": ops, "kernels": kernels, "clocks": clk,
        "gpu_launches": launches,
        "e2e": e2e,
    }
    if extra:
        line["activation_memory"] = extra.pop("activation_memory")
        line["workloads"] = extra
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    rc = run_gpu(args)
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        import torch.distributed as dist

        if dist.is_initialized():
            dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
