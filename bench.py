"""Benchmark of the 2D selective-scan forward on B200: Gelem/s (batch*D*H*W per second) and
the fraction of the kernel's roofline.  One JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload giga|vision|small|wsi|tiny]
                    [--impl ours|reference] [--no-cpu-baseline] [--others] [--pass fwd|bwd]

--pass bwd times the gradients (scan2d_bwd, one call per step) on the same workloads instead;
--pass wsi --workload wsi times the whole-slide path built from a bag of patch features;
--pass proj times the input projections (x -> delta, B, C) and then the scan on their output.

A step is one scan2d_fwd call over one batch of the workload (every step of the path runs
in it).  N > 1 runs under torchrun, one rank per GPU; the (b, d) maps are independent, so
each rank runs its own instance of the workload (weak scaling, no collective on the data
path) and the value is all ranks' elements over the slowest rank's time.

--impl reference times the fp64 oracle (the CPU reference of this path) on the host cores,
each step a bounded sample of the workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from selective_state_space_scan2d_b200 import inputs  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
SMS = 148
MUFU_PER_CLK_SM = 16          # ex2 per clock per SM (sm_100 throughput table, confirmed by probe)
FP32_PER_CLK_SM = 128         # FP32 lanes per clock per SM
SM_MAX_MHZ = 1965.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured", float(p.get("sm_max_mhz", SM_MAX_MHZ))
    except Exception:
        return 6650.0, "fallback", SM_MAX_MHZ


def roofline_model(w: inputs.Workload):
    """Algorithmic work per element (batch*D*H*W unit) and the bound at peak rates."""
    s = 2 if w.dtype == "bf16" else 4
    sy = s
    bytes_el = 2 * s + sy + w.K * 2 * w.N * s / w.channels
    exps_el = w.N                                   # Abar once per (position, state)
    fp32_el = w.N * (1 + 4 * w.K) + 2               # dA mul; per orientation Bbar x, hor, vert, C
    hbm_gbs, hbm_kind, sm_mhz = _peaks()
    clk = sm_mhz * 1e6
    t_hbm = bytes_el / (hbm_gbs * 1e9)
    t_sfu = exps_el / (SMS * MUFU_PER_CLK_SM * clk)
    t_fp32 = fp32_el / (SMS * FP32_PER_CLK_SM * clk)
    bound = max((t_hbm, "hbm"), (t_sfu, "sfu"), (t_fp32, "fp32"))[1]
    return dict(bytes_el=bytes_el, exps_el=exps_el, fp32_el=fp32_el, t_hbm=t_hbm, t_sfu=t_sfu,
                t_fp32=t_fp32, bound=bound, hbm_gbs=hbm_gbs, hbm_kind=hbm_kind, sm_mhz=sm_mhz,
                roof_gelem=1e-9 / max(t_hbm, t_sfu, t_fp32))


METRIC = "2D selective-scan fwd Gelem/s (B*D*H*W) and % of HBM/SFU roofline"
METRIC_BWD = "2D selective-scan bwd Gelem/s (B*D*H*W) and % of roofline"


def roofline_model_bwd(w: inputs.Workload):
    """Algorithmic work per element of the gradients: every input and the cotangent read
    once, every gradient written once, Abar once per (position, state), and per (element,
    state, orientation) the adjoint's fp32 work: Abar's argument, the forward horizontal
    and vertical updates with Bbar x, the two adjoint updates (FMA and multiply each), and
    the five products and three sums that feed dx, ddelta, dA, dB, dC (16 operations)."""
    s = 2 if w.dtype == "bf16" else 4
    bytes_el = 3 * s + 2 * s + w.K * 2 * w.N * (s + 4) / w.channels
    exps_el = w.N
    fp32_el = 16 * w.N * w.K + 4
    hbm_gbs, hbm_kind, sm_mhz = _peaks()
    clk = sm_mhz * 1e6
    t_hbm = bytes_el / (hbm_gbs * 1e9)
    t_sfu = exps_el / (SMS * MUFU_PER_CLK_SM * clk)
    t_fp32 = fp32_el / (SMS * FP32_PER_CLK_SM * clk)
    bound = max((t_hbm, "hbm"), (t_sfu, "sfu"), (t_fp32, "fp32"))[1]
    return dict(bytes_el=bytes_el, exps_el=exps_el, fp32_el=fp32_el, t_hbm=t_hbm, t_sfu=t_sfu,
                t_fp32=t_fp32, bound=bound, hbm_gbs=hbm_gbs, hbm_kind=hbm_kind, sm_mhz=sm_mhz,
                roof_gelem=1e-9 / max(t_hbm, t_sfu, t_fp32))


def base_config(w: inputs.Workload, world: int) -> dict:
    return {"workload": w.name, "batch": w.batch, "channels": w.channels, "N": w.N,
            "H": w.H, "W": w.W, "dtype_in": w.dtype, "orientations": w.K,
            "global_batch": w.batch * world, "parallelism": f"replicas x{world}"}


def max_over_ranks(values, device=None):
    """Element-wise max of per-rank values over all ranks (the values themselves without a
    process group); every rank calls it with the same number of values."""
    import torch
    if not torch.distributed.is_initialized() or torch.distributed.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_gelem(elements_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank processes its own instance of the workload (weak
    scaling), timed by the slowest rank."""
    return world * elements_per_rank / (ms * 1e-3) / 1e9


KERNEL_SOURCES = ("selective_state_space_scan2d_b200/csrc/scan2d.cu",
                  "selective_state_space_scan2d_b200/csrc/scan2d_kernels.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "scan2d_dram_traffic.txt")


def kernel_source_hash() -> str:
    """Hash of the forward's sources with comments and blank lines removed, so that the
    recorded DRAM traffic stays attached to the code it was measured on."""
    import hashlib
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        text = "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())
        h.update(text.encode())
    return h.hexdigest()[:16]


def dram_traffic(w: inputs.Workload):
    """DRAM bytes (read + write) per launch of the scan kernel for this workload, from the
    committed ncu summary; None when there is none or the kernel sources changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            lines = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    except OSError:
        return None
    key = f"{w.name}:{w.batch}x{w.channels}x{w.H}x{w.W}"
    src = kernel_source_hash()
    for parts in lines:
        # <workload:BxDxHxW> <kernel source hash> <bytes per launch> ...
        if len(parts) >= 3 and parts[0] == key and parts[1] == src:
            return float(parts[2])
    return None


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_dev: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self.nv = None
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        getr = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = getr(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def _to_dev(a, torch, device):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def _to_pinned(a, torch):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
    return torch.from_numpy(a).pin_memory()


def _oracle_sample_rate(w: inputs.Workload, d: dict, budget_s: float):
    """Time the fp64 oracle on whole (b, d) maps of the workload, as many as fit the budget."""
    import oracle
    oracle.build()
    maps = [(b, c) for b in range(w.batch) for c in range(w.channels)]
    done, t_used, elems = 0, 0.0, 0
    t0 = time.perf_counter()
    while done < len(maps):
        # one map at a time until the budget is used
        oracle.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], [maps[done]],
                           d["orient_mask"])
        done += 1
        elems += w.H * w.W
        t_used = time.perf_counter() - t0
        if t_used >= budget_s:
            break
    return elems / t_used / 1e9, done, t_used


def run_reference(args, w: inputs.Workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    d = inputs.make_inputs(w, seed=0)
    # one step = whole maps of the workload, about 0.5 s of oracle work
    maps_all = [(b, c) for b in range(w.batch) for c in range(w.channels)]
    t0 = time.perf_counter()
    oracle.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], [maps_all[0]], d["orient_mask"])
    t_map = max(time.perf_counter() - t0, 1e-6)
    per_step = max(1, min(len(maps_all), int(0.5 / t_map)))
    step_maps = [maps_all[i % len(maps_all)] for i in range(per_step)]
    for _ in range(args.warmup):
        oracle.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], step_maps, d["orient_mask"])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.scan2d_maps(d["x"], d["delta"], d["A"], d["B"], d["C"], d["Dskip"], step_maps, d["orient_mask"])
    dt = (time.perf_counter() - t0) / args.steps
    elems = per_step * w.H * w.W
    value = elems / dt / 1e9
    sample = f"{per_step} whole (b,d) maps of {w.name} per step ({elems} elements), fp64 C oracle"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "Gelem/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": base_config(w, 1),
        "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def measure_workload(w, args, torch, scan2d, device, rank, seed, steps, warmup, with_e2e):
    d = inputs.make_inputs(w, seed=seed)
    flags = scan2d.flags_for(w.dtype == "bf16", w.orient_mask)
    plan = scan2d.scan2d_query_plan(w.batch, w.channels, w.H, w.W, w.N, flags)
    t = {k: _to_dev(d[k], torch, device) for k in ("x", "delta", "A", "B", "C", "Dskip")}
    set_bytes = sum(v.numel() * v.element_size() for v in t.values() if v is not None)
    out_dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    y_bytes = w.elements * (2 if w.dtype == "bf16" else 4)
    set_bytes += y_bytes
    # rotate through copies of the inputs so that no step finds its data in L2
    n_sets = max(1, math.ceil(3 * L2_BYTES / set_bytes))
    sets = [t] + [{k: (v.clone() if v is not None else None) for k, v in t.items()} for _ in range(n_sets - 1)]
    ys = [torch.empty((w.batch, w.channels, w.H, w.W), dtype=out_dtype, device=device) for _ in range(n_sets)]
    stream = torch.cuda.current_stream()

    def step(i):
        s = sets[i % n_sets]
        scan2d.scan2d_fwd(s["x"], s["delta"], s["A"], s["B"], s["C"], s["Dskip"], y=ys[i % n_sets],
                          flags=flags, stream=stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    if torch.distributed.is_initialized():
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        e0.record(stream)
        for i in range(steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
    if torch.distributed.is_initialized():
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1) / steps
    err = scan2d.scan2d_get_device_error()
    if err:
        raise RuntimeError(f"device error {err}: {scan2d.scan2d_strerror(err)}")
    res = dict(ms=ms, plan=plan, n_sets=n_sets, clocks=clk.summary(), flags=flags, d=d)
    if with_e2e:
        res["e2e"] = measure_e2e(w, d, torch, scan2d, device, flags, steps)
    del sets, ys, t
    return res


def measure_e2e(w, d, torch, scan2d, device, flags, steps):
    """scan2d_fwd_host on pinned host buffers: H2D of the inputs, the scan, D2H of y."""
    h = {k: _to_pinned(d[k], torch) for k in ("x", "delta", "A", "B", "C", "Dskip")}
    out_dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    yh = torch.empty((w.batch, w.channels, w.H, w.W), dtype=out_dtype).pin_memory()
    nbytes = scan2d.scan2d_host_staging_bytes(w.batch, w.channels, w.H, w.W, w.N, flags)
    staging = torch.empty(nbytes, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    n = max(2, min(steps, 10))
    scan2d.scan2d_fwd_host(h["x"], h["delta"], h["A"], h["B"], h["C"], h["Dskip"], yh, staging, flags, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        scan2d.scan2d_fwd_host(h["x"], h["delta"], h["A"], h["B"], h["C"], h["Dskip"], yh, staging, flags, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / n
    h2d = sum(v.numel() * v.element_size() for v in h.values() if v is not None)
    d2h = yh.numel() * yh.element_size()
    return dict(ms=ms, steps=n, h2d=h2d, d2h=d2h)


def measure_backward(w, torch, scan2d, device, seed, steps, warmup):
    """scan2d_bwd on device-resident inputs and cotangent, one caller-owned workspace."""
    d = inputs.make_inputs(w, seed=seed)
    dy = inputs.make_cotangent(w, seed=seed)
    flags = scan2d.flags_for(w.dtype == "bf16", w.orient_mask)
    t = {k: _to_dev(d[k], torch, device) for k in ("x", "delta", "A", "B", "C", "Dskip")}
    t["dy"] = _to_dev(dy, torch, device)
    set_bytes = sum(v.numel() * v.element_size() for v in t.values() if v is not None)
    n_sets = max(1, math.ceil(3 * L2_BYTES / set_bytes))
    sets = [t] + [{k: (v.clone() if v is not None else None) for k, v in t.items()} for _ in range(n_sets - 1)]
    ws = torch.empty(scan2d.scan2d_bwd_workspace_bytes(w.batch, w.channels, w.H, w.W, w.N, flags),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step(i):
        s = sets[i % n_sets]
        return scan2d.scan2d_bwd(s["x"], s["delta"], s["A"], s["B"], s["C"], s["Dskip"], s["dy"],
                                 flags=flags, workspace=ws, stream=stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        e0.record(stream)
        for i in range(steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    err = scan2d.scan2d_get_device_error()
    if err:
        raise RuntimeError(f"device error {err}: {scan2d.scan2d_strerror(err)}")
    return dict(ms=ms, n_sets=n_sets, clocks=clk.summary(), d=d, dy=dy, ws_bytes=ws.numel())


def _oracle_bwd_sample_rate(w: inputs.Workload, d: dict, dy, budget_s: float):
    """Time the fp64 oracle's gradients on whole maps (one batch element, growing channel
    counts) until the budget is used."""
    import oracle
    oracle.build()
    dyf = inputs.bf16_bits_to_f32(dy).astype(np.float64) if dy.dtype == np.uint16 else dy.astype(np.float64)
    elems, t_used, ch = 0, 0.0, 1
    while True:
        sub = slice(0, min(ch, w.channels))
        t0 = time.perf_counter()
        oracle.scan2d_bwd(d["x"][:1, sub], d["delta"][:1, sub], d["A"][sub], d["B"][:1], d["C"][:1],
                          None if d["Dskip"] is None else d["Dskip"][sub], dyf[:1, sub], d["orient_mask"])
        t_used += time.perf_counter() - t0
        elems += (sub.stop - sub.start) * w.H * w.W
        if t_used >= budget_s or ch >= w.channels:
            break
        ch *= 2
    return elems / t_used / 1e9, elems, t_used


def run_backward(args, w):
    import torch
    from selective_state_space_scan2d_b200 import scan2d
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        torch.distributed.barrier()
    res = measure_backward(w, torch, scan2d, device, seed=rank, steps=args.steps, warmup=args.warmup)
    (ms,) = max_over_ranks([res["ms"]], device=device)
    value = whole_job_gelem(w.elements, world, ms)
    rm = roofline_model_bwd(w)
    if rm["bound"] == "sfu":
        achieved, peak, unit = w.elements * rm["exps_el"] / (ms * 1e-3) / 1e9, SMS * MUFU_PER_CLK_SM * rm["sm_mhz"] * 1e-3, "Gex2/s"
    elif rm["bound"] == "fp32":
        achieved, peak, unit = w.elements * rm["fp32_el"] / (ms * 1e-3) / 1e9, SMS * FP32_PER_CLK_SM * rm["sm_mhz"] * 1e-3, "Gfp32op/s"
    else:
        achieved, peak, unit = w.elements * rm["bytes_el"] / (ms * 1e-3) / 1e9, rm["hbm_gbs"], "GB/s"
    launches = 4 * w.K
    line = {
        "metric": METRIC_BWD, "value": value, "unit": "Gelem/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if w.dtype == "f32" else "bf16-in/f32-acc", "data": "synthetic",
        "config": {**base_config(w, world), "pass": "bwd",
                   "l2": f"inputs rotated over {res['n_sets']} device copies (> 3x L2 per rotation)",
                   "workspace_bytes": res["ws_bytes"]},
        "roofline": {"bound": "alu" if rm["bound"] != "hbm" else "hbm", "unit_of_bound": rm["bound"],
                     "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                     "traffic": None, "scope": f"whole scan2d_bwd call ({launches} kernel launches)",
                     "roofline_gelem_s": rm["roof_gelem"]},
        "clocks": res["clocks"], "gpu_launches": args.steps * launches,
        "e2e": None,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, elems, secs = _oracle_bwd_sample_rate(w, res["d"], res["dy"], args.cpu_budget)
        line["cpu_baseline"] = {"value": rate, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
                                "sample": f"gradients of whole maps of batch element 0 of {w.name} ({elems} elements) in {secs:.1f} s, fp64 C oracle, 1 thread"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_wsi(args, w):
    """The whole-slide path: cell map and map built from a bag of patches, then the scan, as
    two steps (grid gather + scan2d_fwd) and fused (scan2d_fwd_wsi reads x through the cell
    map).  value = the fused path's Gelem/s; the grid gather's HBM roofline is reported."""
    import torch
    from selective_state_space_scan2d_b200 import scan2d
    if w.name != "wsi" and not w.wsi_mask:
        raise SystemExit("--pass wsi needs a whole-slide workload (--workload wsi)")
    if int(os.environ.get("RANK", "0")) != 0:
        return                       # a one-GPU measurement: under torchrun only rank 0 runs it
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    b = inputs.make_wsi_bag(w, seed=0)
    t = {k: _to_dev(b[k], torch, device) for k in ("delta", "A", "B", "C", "Dskip", "feat", "pad")}
    coords = torch.from_numpy(b["coords"]).to(device)
    flags = scan2d.flags_for(w.dtype == "bf16", w.orient_mask)
    npatch = b["feat"].shape[0]
    out_dtype = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    cell = torch.empty(w.H * w.W, dtype=torch.int32, device=device)
    x = torch.empty((1, w.channels, w.H, w.W), dtype=t["feat"].dtype, device=device)
    y = torch.empty((1, w.channels, w.H, w.W), dtype=out_dtype, device=device)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)   # written between steps
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        total = 0.0
        with ClockSampler(device.index) as clk:
            for _ in range(args.steps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                e1.synchronize()
                total += e0.elapsed_time(e1)
        return total / args.steps, clk.summary()

    cells_ms, _ = timed(lambda: scan2d.scan2d_grid_cells(coords, w.H, w.W, cell_patch=cell, stream=stream))
    gather_ms, _ = timed(lambda: scan2d.scan2d_grid_gather(t["feat"], cell, t["pad"], w.H, w.W, x=x, stream=stream))

    def unfused():
        scan2d.scan2d_grid_gather(t["feat"], cell, t["pad"], w.H, w.W, x=x, stream=stream)
        scan2d.scan2d_fwd(x, t["delta"], t["A"], t["B"], t["C"], t["Dskip"], y=y, flags=flags, stream=stream)

    def fused():
        scan2d.scan2d_fwd_wsi(t["feat"], cell, t["pad"], t["delta"], t["A"], t["B"], t["C"], t["Dskip"],
                              y=y, flags=flags, stream=stream)

    unfused_ms, _ = timed(unfused)
    fused_ms, clocks = timed(fused)
    err = scan2d.scan2d_get_device_error()
    if err:
        raise RuntimeError(f"device error {err}")
    s = 2 if w.dtype == "bf16" else 4
    gather_bytes = npatch * w.channels * s + w.H * w.W * 4 + w.channels * w.H * w.W * s
    hbm_gbs, hbm_kind, _ = _peaks()
    achieved = gather_bytes / (gather_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC + " (whole-slide map read from its bag of patches)",
        "value": w.elements / (fused_ms * 1e-3) / 1e9, "unit": "Gelem/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": fused_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32" if w.dtype == "f32" else "bf16-in/f32-acc",
        "data": "synthetic",
        "config": {**base_config(w, 1), "pass": "wsi", "npatch": npatch,
                   "l2": "a 252 MB buffer is written before every timed step"},
        "unfused": {"ms_per_step": unfused_ms, "value": w.elements / (unfused_ms * 1e-3) / 1e9,
                    "steps": "scan2d_grid_gather + scan2d_fwd"},
        "grid_cells_ms": cells_ms, "grid_gather_ms": gather_ms,
        "roofline": {"bound": "hbm", "kernel": "grid gather", "achieved": achieved, "peak": hbm_gbs,
                     "unit": "GB/s", "frac": achieved / hbm_gbs, "traffic": None,
                     "algorithmic_bytes": gather_bytes, "peak_kind": f"{hbm_kind} copy bandwidth"},
        "clocks": clocks, "gpu_launches": args.steps, "e2e": None,
    }
    print(json.dumps(line), flush=True)


def run_proj(args, w, R: int = 8):
    """The input projections (scan2d_proj: x -> delta, B, C with the bias and softplus), then
    the scan on what they wrote.  value = the projections' Gelem/s (batch*D*H*W of delta per
    second); roofline = the slower of HBM (x read, delta, B, C written once) and the FP32
    lanes (D*(R + 2N) + D*R FMAs per position)."""
    import torch
    from selective_state_space_scan2d_b200 import scan2d
    if int(os.environ.get("RANK", "0")) != 0:
        return                       # a one-GPU measurement: under torchrun only rank 0 runs it
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    d = inputs.make_inputs(w, seed=0)
    wt = inputs.make_proj_weights(w.channels, w.N, R, seed=0)
    x = _to_dev(d["x"], torch, device)
    Wx, Wdt, bdt = (torch.from_numpy(wt[k]).to(device) for k in ("Wx", "Wdt", "bdt"))
    A = torch.from_numpy(d["A"]).to(device)
    Dskip = None if d["Dskip"] is None else torch.from_numpy(d["Dskip"]).to(device)
    delta = torch.empty_like(x)
    Bm = torch.empty((w.batch, w.N, w.H, w.W), dtype=x.dtype, device=device)
    Cm = torch.empty_like(Bm)
    y = torch.empty_like(x)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        total = 0.0
        with ClockSampler(device.index) as clk:
            for _ in range(args.steps):
                flush.fill_(1)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                e1.synchronize()
                total += e0.elapsed_time(e1)
        return total / args.steps, clk.summary()

    proj = lambda: scan2d.scan2d_proj(x, Wx, Wdt, bdt, w.N, R, delta=delta, B=Bm, C=Cm, stream=stream)
    proj_ms, clocks = timed(proj)
    flags = scan2d.flags_for(w.dtype == "bf16", 1)

    def chain():
        proj()
        scan2d.scan2d_fwd(x, delta, A, Bm, Cm, Dskip, y=y, flags=flags, stream=stream)

    chain_ms, _ = timed(chain)
    s = 2 if w.dtype == "bf16" else 4
    pos = w.batch * w.H * w.W
    bytes_ = pos * (2 * w.channels + 2 * w.N) * s
    fmas = pos * (w.channels * (R + 2 * w.N) + w.channels * R)
    hbm_gbs, hbm_kind, sm_mhz = _peaks()
    t_hbm = bytes_ / (hbm_gbs * 1e9)
    t_fp32 = fmas / (SMS * FP32_PER_CLK_SM * sm_mhz * 1e6)
    if t_hbm >= t_fp32:
        roof = {"bound": "hbm", "achieved": bytes_ / (proj_ms * 1e-3) / 1e9, "peak": hbm_gbs, "unit": "GB/s",
                "peak_kind": f"{hbm_kind} copy bandwidth"}
    else:
        roof = {"bound": "alu", "unit_of_bound": "fp32", "achieved": fmas / (proj_ms * 1e-3) / 1e9,
                "peak": SMS * FP32_PER_CLK_SM * sm_mhz * 1e-3, "unit": "GFMA/s",
                "peak_kind": f"nominal {SMS} SMs x {FP32_PER_CLK_SM}/clk x {sm_mhz:.0f} MHz"}
    roof.update({"frac": roof["achieved"] / roof["peak"], "traffic": None, "kernel": "k_proj",
                 "algorithmic_bytes": bytes_, "algorithmic_fma": fmas,
                 "t_hbm_ms": t_hbm * 1e3, "t_fp32_ms": t_fp32 * 1e3})
    line = {
        "metric": "input projections x -> (delta, B, C) Gelem/s (B*D*H*W)", "value": w.elements / (proj_ms * 1e-3) / 1e9,
        "unit": "Gelem/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": proj_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if w.dtype == "f32" else "bf16-in/f32-acc", "data": "synthetic",
        "config": {**base_config(w, 1), "pass": "proj", "R": R,
                   "l2": "a 252 MB buffer is written before every timed step"},
        "roofline": roof, "clocks": clocks, "gpu_launches": args.steps, "e2e": None,
        "with_scan": {"ms_per_step": chain_ms, "steps": "scan2d_proj + scan2d_fwd",
                      "value": w.elements / (chain_ms * 1e-3) / 1e9},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="giga", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--others", action="store_true", help="also time the other workloads (extra key)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--override", action="append", default=[], metavar="KEY=INT",
                    help="change batch/channels/H/W of the workload (smaller cases for ncu captures)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer (e2e) leg")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd", "wsi", "proj"],
                    help="bwd: time the gradients (scan2d_bwd); wsi: the whole-slide path from a bag of patches")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = inputs.WORKLOADS[args.workload]
    if args.override:
        kw = {}
        for item in args.override:
            key, _, val = item.partition("=")
            if key not in ("batch", "channels", "H", "W"):
                ap.error(f"--override: unknown key {key!r}")
            kw[key] = int(val)
        w = w.scaled(**kw)

    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.which == "bwd":
        run_backward(args, w)
        return
    if args.which == "wsi":
        run_wsi(args, w)
        return
    if args.which == "proj":
        run_proj(args, w)
        return

    import torch
    from selective_state_space_scan2d_b200 import scan2d

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)

    res = measure_workload(w, args, torch, scan2d, device, rank, seed=rank, steps=args.steps,
                           warmup=args.warmup, with_e2e=not args.no_e2e)
    ms = res["ms"]
    e2e_ms = res["e2e"]["ms"] if "e2e" in res else float("nan")
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=device)
    value = whole_job_gelem(w.elements, world, ms)
    e2e_value = whole_job_gelem(w.elements, world, e2e_ms)

    rm = roofline_model(w)
    if rm["bound"] == "sfu":
        achieved = w.elements * rm["exps_el"] / (ms * 1e-3) / 1e9
        peak = SMS * MUFU_PER_CLK_SM * rm["sm_mhz"] * 1e6 / 1e9
        unit = "Gex2/s"
    elif rm["bound"] == "fp32":
        achieved = w.elements * rm["fp32_el"] / (ms * 1e-3) / 1e9
        peak = SMS * FP32_PER_CLK_SM * rm["sm_mhz"] * 1e6 / 1e9
        unit = "Gfp32op/s"
    else:
        achieved = w.elements * rm["bytes_el"] / (ms * 1e-3) / 1e9
        peak = rm["hbm_gbs"]
        unit = "GB/s"
    roof = {"bound": "alu" if rm["bound"] != "hbm" else "hbm", "unit_of_bound": rm["bound"],
            "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": dram_traffic(w), "peak_kind": f"nominal {SMS} SMs x {MUFU_PER_CLK_SM if rm['bound']=='sfu' else FP32_PER_CLK_SM}/clk x {rm['sm_mhz']:.0f} MHz (max clock)" if rm["bound"] != "hbm" else f"{rm['hbm_kind']} copy bandwidth",
            "hbm_achieved_gbs": w.elements * rm["bytes_el"] / (ms * 1e-3) / 1e9,
            "hbm_frac_of_measured": w.elements * rm["bytes_el"] / (ms * 1e-3) / 1e9 / rm["hbm_gbs"],
            "roofline_gelem_s": rm["roof_gelem"], "frac_of_roofline_gelem": (w.elements / (ms * 1e-3) / 1e9) / rm["roof_gelem"]}
    clocks = res["clocks"]
    if clocks.get("sm_mhz"):
        roof["frac_at_sampled_clock"] = roof["frac"] * (rm["sm_mhz"] / clocks["sm_mhz"]) if rm["bound"] != "hbm" else roof["frac"]

    line = {
        "metric": METRIC,
        "value": value, "unit": "Gelem/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if w.dtype == "f32" else "bf16-in/f32-acc",
        "data": "synthetic",
        "config": {**base_config(w, world),
                   "l2": f"inputs rotated over {res['n_sets']} device copies (> 3x L2 per rotation)",
                   **({"overrides": args.override} if args.override else {})},
        "roofline": roof,
        "clocks": clocks,
        "gpu_launches": args.steps * res["plan"]["launches"],
        "plan": res["plan"],
    }
    if "e2e" in res:
        line["e2e"] = {"value": e2e_value, "unit": "Gelem/s", "h2d_bytes_per_step": res["e2e"]["h2d"],
                       "d2h_bytes_per_step": res["e2e"]["d2h"], "steps": res["e2e"]["steps"],
                       "api": "scan2d_fwd_host (pinned host buffers)"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, nmaps, secs = _oracle_sample_rate(w, res["d"], args.cpu_budget)
        line["cpu_baseline"] = {"value": rate, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
                                "sample": f"{nmaps} whole (b,d) maps of {w.name} ({nmaps * w.H * w.W} elements) in {secs:.1f} s, fp64 C oracle, 1 thread"}
    if args.others and world == 1:
        others = {}
        for name in ("wsi", "small", "vision", "giga"):
            if name == w.name:
                continue
            ow = inputs.WORKLOADS[name]
            r = measure_workload(ow, args, torch, scan2d, device, rank, seed=0,
                                 steps=max(20, args.steps // 4), warmup=args.warmup, with_e2e=False)
            orm = roofline_model(ow)
            gel = ow.elements / (r["ms"] * 1e-3) / 1e9
            others[name] = {"value": gel, "ms_per_step": r["ms"], "bound": orm["bound"],
                            "roofline_gelem_s": orm["roof_gelem"], "frac": gel / orm["roof_gelem"],
                            "clocks": r["clocks"], "plan": r["plan"]}
        line["others"] = others
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
