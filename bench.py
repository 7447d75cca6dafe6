"""Benchmark of the edge-conditioned CG tensor-product convolution on B200.

Metric: TP-conv edges/s (forward, and forward+backward where the workload has a
backward) with the achieved fraction of the roofline. The headline line times
one forward + backward step of the large-graph channelwise fp32 workload (100k
atoms, ~4M edges, 64x(0e+1o+2e) -> 64x(l <= 2, both parities), L_sh 2, K 8),
the largest single-GPU workload, with every input resident in HBM. Its inputs
(~1 GB) are larger than the L2 (126 MB); a 256 MiB write outside the timed events
flushes the L2 between steps anyway.

The same JSON line carries, under "workloads", the forward (and forward +
backward) of every workload, the MACE-like forward among them; under
"workspace", the measured device memory of one forward + backward at E/4, E/2
and E edges on the two largest workloads.

Multi-GPU: the operator has no exchange step for independent batches, so each
rank runs its own replica (weak scaling) and rank 0 reports the max time over
ranks. `--impl reference` times the CPU oracle on the host cores instead.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                       [--config C] [--pass fwd|fwdbwd] [--no-extra] [--no-cpu-baseline]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TP-conv edges/s fwd and fwd+bwd (FP32/FP64) on 1 B200; % of roofline"
SMS, FP32_LANES, FP64_LANES, MAX_MHZ = 148, 128, 64, 1965.0


def alu_peak(dtype: str) -> float:
    """FMA lanes x 2 flops x SMs x max clock (GFLOP/s scale in TFLOP/s)."""
    lanes = FP32_LANES if dtype == "f32" else FP64_LANES
    return SMS * lanes * 2 * MAX_MHZ * 1e6 / 1e12


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, interval_ms: int = 50):
        self.proc = None
        self.lines = []
        self.interval = interval_ms

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.interval)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- setup

def setup(cid: int, dev: str, n_nodes=None, node_order=None):
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    from inputs import CONFIGS, make_workload
    c = CONFIGS[cid]
    plan = tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype, irreps_sh=c.irreps_sh)
    wl = make_workload(cid, plan.n_w, n_nodes=n_nodes, c_out=plan.c_out, node_order=node_order)
    N, E = wl.n_nodes, wl.n_edges
    src = torch.from_numpy(wl.src.astype(np.int32)).to(dev)
    dst = torch.from_numpy(wl.dst.astype(np.int32)).to(dev)
    rowptr, senders, perm = tpc.tp_csr_build(src, dst, N)
    colptr, srcedge, srcrecv = tpc.tp_csr_transpose(rowptr, senders, N)
    p = perm.long()
    d = dict(cfg=c, plan=plan, wl=wl, N=N, E=E, rowptr=rowptr, senders=senders, colptr=colptr,
             srcedge=srcedge, srcrecv=srcrecv, perm=perm,
             x=torch.from_numpy(wl.x).to(dev),
             Y=torch.from_numpy(wl.Y).to(dev)[p].contiguous(),
             phi=torch.from_numpy(wl.phi).to(dev)[p].contiguous(),
             A=torch.from_numpy(wl.A).to(dev),
             gout=torch.from_numpy(wl.grad_out).to(dev))
    d["out"] = torch.empty(N, plan.c_out, dtype=plan.torch_dtype, device=dev)
    d["grads"] = (torch.empty_like(d["x"]), torch.empty_like(d["Y"]), torch.empty_like(d["phi"]),
                  torch.empty_like(d["A"]))
    d["ws_f"] = torch.empty(max(1, plan.workspace_size(N, 0)), dtype=torch.uint8, device=dev)
    d["ws_b"] = torch.empty(max(1, plan.workspace_size(N, 1)), dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    return d


def fwd(d):
    import clebsch_gordan_tensor_node_b200 as tpc
    return tpc.tp_conv_forward(d["plan"], d["x"], d["Y"], d["phi"], d["A"], d["rowptr"], d["senders"],
                               out=d["out"], ws=d["ws_f"])


def bwd(d):
    import clebsch_gordan_tensor_node_b200 as tpc
    return tpc.tp_conv_backward(d["plan"], d["x"], d["Y"], d["phi"], d["A"], d["rowptr"], d["senders"],
                                d["colptr"], d["srcedge"], d["srcrecv"], d["gout"], out=d["grads"],
                                ws=d["ws_b"])


def dbl(d):
    import clebsch_gordan_tensor_node_b200 as tpc
    if "dirs" not in d:
        import torch
        g = torch.Generator(device=d["x"].device).manual_seed(3)
        d["dirs"] = [torch.randn(d[k].shape, generator=g, device=d[k].device, dtype=d[k].dtype)
                     for k in ("x", "Y", "phi", "A")]
        d["dbl_out"] = (torch.empty_like(d["out"]),) + tuple(torch.empty_like(t) for t in d["grads"])
        d["ws_d"] = torch.empty(max(1, d["plan"].workspace_size(d["N"], 2)), dtype=torch.uint8,
                                device=d["x"].device)
    return tpc.tp_conv_double_backward(d["plan"], d["x"], d["Y"], d["phi"], d["A"], d["rowptr"], d["senders"],
                                       d["colptr"], d["srcedge"], d["srcrecv"], d["gout"], *d["dirs"],
                                       out=d["dbl_out"], ws=d["ws_d"])


def time_steps(step, steps: int, warmup: int, flush, sampler=None, dist=None):
    """Per-step CUDA-event times (ms) on the current stream, L2 flushed in
    between. `step(marks)` may append events it records between its passes;
    returns (step times, per-pass times, clocks)."""
    import torch
    for _ in range(warmup):
        flush()
        step([])
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    evs = []
    for _ in range(steps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        marks = []
        a.record()
        step(marks)
        b.record()
        evs.append((a, marks, b))
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    totals = [a.elapsed_time(b) for a, _, b in evs]
    passes = []
    for a, marks, b in evs:
        pts = [a] + marks + [b]
        passes.append([pts[k].elapsed_time(pts[k + 1]) for k in range(len(pts) - 1)])
    return totals, passes, clocks


def roofline_step(d, ms_pass, both: bool) -> dict:
    """Roofline of the timed step: algorithmic flops of every pass over the step
    time, against the derived ALU peak of the dtype; the per-pass numbers use
    the CUDA-event time of each pass (the forward is one kernel launch)."""
    f0, b0 = d["plan"].work_model(d["N"], d["E"], 0)
    ms = sum(ms_pass)
    if both:
        f1, b1 = d["plan"].work_model(d["N"], d["E"], 1)
        flops, nbytes = f0 + f1, b0 + b1
    else:
        flops, nbytes = f0, b0
    r = roofline(d, 0, ms)
    ach = flops / (ms * 1e-3) / 1e12
    key = (d["cfg"].id, "fwdbwd" if both else "fwd")
    t = NCU_TRAFFIC.get(key)
    r.update({"achieved": round(ach, 3), "frac": round(ach / r["peak"], 4), "algorithmic_flops": flops,
              "compulsory_bytes": nbytes, "traffic": None, "traffic_source": None,
              "hbm_frac_of_measured": None,
              "kernel": ("one step = forward (uvu_fwd_kernel) + backward (uvu_edge_kernel, "
                         "uvu_src_kernel, reduce_slots_kernel)") if both and d["cfg"].mode == "uvu" else
                        "one step = " + ("forward + backward" if both else "forward") + " launches"})
    if t is not None:
        hbm = measured_hbm_gbs()
        r["traffic"] = t[0]
        r["traffic_source"] = f"{t[1]}: dram__bytes_read.sum + dram__bytes_write.sum, {t[2]}"
        if hbm:
            r["hbm_frac_of_measured"] = round(t[0] / (ms * 1e-3) / 1e9 / hbm, 4)
    per = {"fwd": {"ms": round(ms_pass[0], 5),
                   "achieved": round(f0 / (ms_pass[0] * 1e-3) / 1e12, 3)}}
    per["fwd"]["frac"] = round(per["fwd"]["achieved"] / r["peak"], 4)
    if both:
        per["bwd"] = {"ms": round(ms_pass[1], 5), "achieved": round(f1 / (ms_pass[1] * 1e-3) / 1e12, 3)}
        per["bwd"]["frac"] = round(per["bwd"]["achieved"] / r["peak"], 4)
    r["passes"] = per
    return r


def tensor_aware_peak_tflops():
    """fp32-exact mixing on the tensor cores: three TF32 products per output
    (3xTF32 split); TF32 runs at half the measured dense bf16 rate (the
    nominal 1.1 vs 2.25 PFLOP/s ratio). From MEASURED_PEAKS.json, else the
    fallback burst figure of 1.59 PFLOP/s bf16."""
    p = measured_peaks()
    bf16 = float(p["bf16_tflops"]) if p and "bf16_tflops" in p else 1590.0
    return bf16 / 2.0 / 3.0


def uvw_mixing_flops(plan, n_nodes: int, pass_: int) -> float:
    """Flops of the channel-mixing products (Sobek Eqs. 34-36): per receiver and
    path 2 (2 l3 + 1) K C_in C_out each; forward one product, backward the
    two of Eq. 36 plus the source mixing of x_bar."""
    r = 0.0
    for p in plan.paths():
        r += 2.0 * (2 * p.l3 + 1) * plan.n_radial * p.mul_in * p.mul_out
        if pass_ == 1:
            r += 2.0 * 2 * (2 * p.l3 + 1) * plan.n_radial * p.mul_in * p.mul_out \
                 + 2.0 * (2 * p.l1 + 1) * plan.n_radial * p.mul_in * p.mul_out
    return r * n_nodes


def tensor_aware_frac(d, pass_: int, ms: float):
    """Roofline fraction of a fully connected pass with the mixing products at
    the 3xTF32 tensor rate and the rest at the FP32 ALU peak."""
    if d["cfg"].mode != "uvw":
        return None
    flops, _ = d["plan"].work_model(d["N"], d["E"], pass_)
    mix = uvw_mixing_flops(d["plan"], d["N"], pass_)
    t = (flops - mix) / (alu_peak("f32") * 1e12) + mix / (tensor_aware_peak_tflops() * 1e12)
    return round(t / (ms * 1e-3), 4)


def roofline_dbl(d, ms: float) -> dict:
    """Roofline of a double-backward step: its algorithmic flops (work model
    pass 2) over the step time against the derived ALU peak."""
    r = roofline(d, 2, ms)
    r["kernel"] = "one step = the second-order program's launches"
    t = NCU_TRAFFIC.get((d["cfg"].id, "dbl"))
    if t is not None:
        r["traffic"] = t[0]
        r["traffic_source"] = f"{t[1]}: dram__bytes_read.sum + dram__bytes_write.sum, {t[2]}"
    return r


# DRAM bytes (read + write) per step (summed over the step's kernels) or per
# launch of a single-kernel pass, from ncu captures of the current kernels (the
# summaries under profiles/ give the commands); absent where no capture of the
# current kernels exists.
NCU_TRAFFIC = {
    (4, "fwdbwd"): (73_558_277_120, "uvu_fwd_kernel + uvu_edge_kernel + uvu_src_kernel + reduce_slots_kernel",
                    "profiles/uvu_step_dram_large_100k.md"),
    (4, "fwd"): (6_989_559_808 + 435_421_440, "uvu_fwd_kernel", "profiles/uvu_step_dram_large_100k.md"),
    (4, "dbl"): (107_987_648_000, "uvu_dbwd_recv_kernel + uvu_dbwd_edge_kernel + uvu_dbwd_src_kernel + "
                 "reduce_slots_kernel", "profiles/uvu_step_dram_large_100k.md"),
}


def roofline(d, pass_: int, ms: float) -> dict:
    flops, nbytes = d["plan"].work_model(d["N"], d["E"], pass_)
    dt = d["cfg"].dtype
    peak = alu_peak(dt)
    ach = flops / (ms * 1e-3) / 1e12
    return {"bound": "alu", "achieved": round(ach, 3), "peak": round(peak, 2), "unit": "TFLOP/s",
            "frac": round(ach / peak, 4), "traffic": None,
            "peak_source": f"derived: {SMS} SMs x {FP32_LANES if dt == 'f32' else FP64_LANES} "
                           f"{'FP32' if dt == 'f32' else 'FP64'} FMA lanes x 2 x {MAX_MHZ:.0f} MHz",
            "algorithmic_flops": flops, "compulsory_bytes": nbytes}


def measured_hbm_gbs():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- CPU oracle

def _cores():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


class OracleSampler:
    """The CPU oracle (forward, or forward + backward) on windows of receivers of
    a workload: each call runs the oracle on the incoming edges of the next
    `n_recv` receivers of a seeded permutation and returns (edges, seconds)."""

    def __init__(self, cid: int, both: bool):
        from inputs import CONFIGS, make_workload
        from oracle import conv as oconv
        self.oconv = oconv
        c = CONFIGS[cid]
        self.cid, self.both = cid, both and c.backward
        self.pr = oconv.Problem(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.irreps_sh)
        self.wl = make_workload(cid, self.pr.n_w, c_out=self.pr.c_out)
        self.order = np.random.default_rng(0).permutation(self.wl.n_nodes)
        self.pos = 0

    def run(self, n_recv: int):
        wl = self.wl
        if self.pos + n_recv > wl.n_nodes:
            self.pos = 0
        recv = self.order[self.pos:self.pos + n_recv]
        self.pos += n_recv
        sel = np.isin(wl.dst, recv)
        args = (wl.x, wl.Y[sel], wl.phi[sel], wl.A, wl.src[sel], wl.dst[sel])
        t0 = time.perf_counter()
        self.oconv.forward(self.pr, *args, wl.n_nodes)
        if self.both:
            self.oconv.backward(self.pr, *args, wl.grad_out, wl.n_nodes)
        return int(sel.sum()), time.perf_counter() - t0

    def calibrate(self, seconds: float) -> int:
        """Receivers per window for about `seconds` of oracle work."""
        self.run(16)                       # first call fills the oracle's CG caches
        e, t = self.run(16)
        return int(max(1, min(self.wl.n_nodes, 16 * seconds / max(t, 1e-3))))

    def label(self):
        return "forward + backward" if self.both else "forward"


def cpu_oracle_sample(cid: int, both: bool, budget_s: float = 15.0):
    """Oracle edges/s on the host cores over a bounded receiver sample."""
    s = OracleSampler(cid, both)
    n_recv = s.calibrate(2.0)
    done_e, t_used, n_done = 0, 0.0, 0
    while t_used < budget_s and n_done < s.wl.n_nodes:
        e, t = s.run(n_recv)
        done_e += e
        t_used += t
        n_done += n_recv
    return {"value": round(done_e / t_used, 1), "unit": "edges/s", "cores": _cores(), "kind": "oracle",
            "sample": f"{s.label()} of {n_done} random receivers ({done_e} edges) of workload {cid}, "
                      f"{t_used:.1f} s", "host_cpus": os.cpu_count(), "workload_edges": len(s.wl.src)}


# ----------------------------------------------------------------------------- ranks

def aggregate_ranks(t_total_ms: float, n_edges: int, steps: int, world: int, dist=None, device="cpu"):
    """Whole-job timing of N replicas: the max over ranks of the timed total
    (ms), and the edges all ranks processed per second of that time."""
    if dist is not None:
        import torch
        tt = torch.tensor([t_total_ms], dtype=torch.float64, device=device)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t_total_ms = float(tt.item())
    return t_total_ms, n_edges * world * steps / (t_total_ms * 1e-3)


# ----------------------------------------------------------------------------- main

def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, timed on the host cores.
    Each step is the oracle on one window of receivers of the workload (sized
    for about 1.5 s of work), so ms_per_step is the wall time of the work that
    actually ran and value = edges of the windows / their time."""
    if rank != 0:
        return
    from inputs import CONFIGS
    c = CONFIGS[args.config]
    both = args.pass_ == "fwdbwd" and c.backward
    s = OracleSampler(args.config, both)
    n_recv = s.calibrate(1.5)
    for _ in range(args.warmup):
        s.run(n_recv)
    edges, secs = 0, 0.0
    for _ in range(args.steps):
        e, t = s.run(n_recv)
        edges += e
        secs += t
    val = round(edges / secs, 1)
    sample = (f"{s.label()} of {args.steps} windows of {n_recv} random receivers ({edges} edges in all) "
              f"of the {len(s.wl.src)}-edge workload, {secs:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": c.name, "pass": s.label(), "sample": sample,
                       "step": f"the oracle on one window of {n_recv} receivers"},
            "cpu_baseline": {"value": val, "unit": "edges/s", "cores": _cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "edges/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, dist):
    import torch
    dev = f"cuda:{int(os.environ.get('LOCAL_RANK', 0))}"
    torch.cuda.set_device(dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.zero_()

    d = setup(args.config, dev)
    c = d["cfg"]
    sampler = ClockSampler() if rank == 0 else None
    both = args.pass_ == "fwdbwd" and c.backward
    second = args.pass_ == "dbl" and c.backward

    def step(marks):
        if second:
            dbl(d)
            return
        fwd(d)
        if both:
            ev = torch.cuda.Event(enable_timing=True)
            ev.record()
            marks.append(ev)
            bwd(d)

    times, passes, clocks = time_steps(step, args.steps, args.warmup, flush, sampler, dist)
    t_total, value = aggregate_ranks(sum(times), d["E"], args.steps, world, dist, dev)
    ms = t_total / args.steps
    ms_pass = [statistics.fmean(p[k] for p in passes) for k in range(len(passes[0]))]
    import clebsch_gordan_tensor_node_b200 as tpc
    assert tpc.tp_get_device_error() == 0
    res = {"metric": METRIC, "value": round(value, 1), "unit": "edges/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": c.dtype,
           "data": "synthetic",
           "config": {"workload": c.name,
                      "pass": "double backward" if second else "forward+backward" if both else "forward",
                      "n_nodes": d["N"], "n_edges": d["E"],
                      "irreps_in": c.irreps_in, "irreps_out": c.irreps_out, "sh_lmax": c.sh_lmax,
                      "n_radial": c.K, "mode": c.mode, "parallelism": f"replicas x{world}",
                      "l2": "inputs larger than L2; also flushed between steps (256 MiB write outside "
                            "the timed events)"},
           "gpu_launches": args.steps * (d["plan"].launch_count(d["N"], 2) if second else
                                         d["plan"].launch_count(d["N"], 0)
                                         + (d["plan"].launch_count(d["N"], 1) if both else 0)),
           "roofline": roofline_dbl(d, ms) if second else roofline_step(d, ms_pass, both), "clocks": clocks}
    # end to end through the public API: pinned host inputs -> device -> passes -> host results
    if not second:
        res["e2e"] = e2e(d, args, both)
    if rank == 0 and not args.no_extra:
        res["workloads"] = extra_workloads(args, dev, flush, d)
        res["workspace"] = workspace_vs_edges(dev, d)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_oracle_sample(args.config, both)
    if rank == 0:
        print(json.dumps(res), flush=True)


def e2e(d, args, both: bool):
    """The metric through the public API with host buffers: every step copies
    its inputs from pinned host memory, runs the passes and copies the results
    (out, and the four gradients for forward + backward) back."""
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    names = ["x", "Y", "phi", "A", "rowptr", "senders"]
    if both:
        names += ["colptr", "srcedge", "srcrecv", "gout"]
    host = {k: d[k].cpu().pin_memory() for k in names}
    devb = {k: torch.empty_like(d[k]) for k in host}
    res_dev = [d["out"]] + (list(d["grads"]) if both else [])
    res_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in res_dev]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in res_host)

    def step():
        for k in host:
            devb[k].copy_(host[k], non_blocking=True)
        tpc.tp_conv_forward(d["plan"], devb["x"], devb["Y"], devb["phi"], devb["A"], devb["rowptr"],
                            devb["senders"], out=d["out"], ws=d["ws_f"])
        if both:
            tpc.tp_conv_backward(d["plan"], devb["x"], devb["Y"], devb["phi"], devb["A"], devb["rowptr"],
                                 devb["senders"], devb["colptr"], devb["srcedge"], devb["srcrecv"],
                                 devb["gout"], out=d["grads"], ws=d["ws_b"])
        for h, t in zip(res_host, res_dev):
            h.copy_(t, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    n = max(5, min(args.steps, 50))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    return {"value": round(d["E"] / (ms * 1e-3), 1), "unit": "edges/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4),
            "pass": "forward+backward" if both else "forward"}


def extra_workloads(args, dev, flush, head):
    """Every workload's forward and (where defined) forward + backward."""
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    out = {}
    for cid in (1, 2, 3, 4, 5, "4-morton"):
        try:
            if cid == "4-morton":
                # the large graph with its nodes numbered along a Z-order curve:
                # the same operator on a spatially sorted node order
                d = setup(4, dev, node_order="morton")
            else:
                d = head if cid == head["cfg"].id else setup(cid, dev)
        except tpc.TpConvError as e:
            out[str(cid)] = {"skipped": str(e)}
            continue
        try:
            k = 20 if d["E"] < 1_000_000 else 8
            tf, _, _ = time_steps(lambda m: fwd(d), k, 3, flush)
            ms_f = statistics.median(tf)
            rf = roofline_step(d, [ms_f], False)
            name = d["cfg"].name + (", nodes in Z-order" if cid == "4-morton" else "")
            rec = {"workload": name, "n_nodes": d["N"], "n_edges": d["E"], "dtype": d["cfg"].dtype,
                   "fwd_ms": round(ms_f, 5), "fwd_edges_per_s": round(d["E"] / (ms_f * 1e-3), 1),
                   "fwd_roofline_frac": rf["frac"], "fwd_traffic": rf["traffic"],
                   "fwd_roofline_frac_tensor_aware": tensor_aware_frac(d, 0, ms_f),
                   "gpu_launches_fwd": d["plan"].launch_count(d["N"], 0)}
            if d["cfg"].mode == "uvu":
                # the receiver-state order (Sobek §4.2 applied to uvu), for comparison
                d["plan"].set_schedule("receiver_state")
                ts, _, _ = time_steps(lambda m: fwd(d), k, 3, flush)
                d["plan"].set_schedule("streamed")
                rec["fwd_receiver_state_ms"] = round(statistics.median(ts), 5)
            if d["cfg"].backward:
                tb, _, _ = time_steps(lambda m: bwd(d), k, 3, flush)
                ms_b = statistics.median(tb)
                rb = roofline_step(d, [ms_f, ms_b], True)
                rec.update({"bwd_ms": round(ms_b, 5),
                            "fwd_bwd_edges_per_s": round(d["E"] / ((ms_f + ms_b) * 1e-3), 1),
                            "bwd_roofline_frac": rb["passes"]["bwd"]["frac"],
                            "bwd_roofline_frac_tensor_aware": tensor_aware_frac(d, 1, ms_b),
                            "fwd_bwd_roofline_frac": rb["frac"],
                            "workspace_bwd_bytes": d["plan"].workspace_size(d["N"], 1),
                            "gpu_launches_bwd": d["plan"].launch_count(d["N"], 1)})
                td, _, _ = time_steps(lambda m: dbl(d), k, 3, flush)
                ms_d = statistics.median(td)
                fd, _ = d["plan"].work_model(d["N"], d["E"], 2)
                rec.update({"dbl_ms": round(ms_d, 5), "dbl_edges_per_s": round(d["E"] / (ms_d * 1e-3), 1),
                            "dbl_roofline_frac": round(fd / (ms_d * 1e-3) / 1e12 / alu_peak(d["cfg"].dtype), 4),
                            "workspace_dbl_bytes": d["plan"].workspace_size(d["N"], 2),
                            "gpu_launches_dbl": d["plan"].launch_count(d["N"], 2)})
            assert tpc.tp_get_device_error() == 0
            out[str(cid)] = rec
        except tpc.TpConvError as e:
            out[str(cid)] = {"skipped": str(e)}
        if d is not head:
            del d
            torch.cuda.empty_cache()
    return out


def _edge_subset(d, keep: float, dev):
    """The workload of `d` with a seeded fraction of its edges (same nodes)."""
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    wl = d["wl"]
    m = np.random.default_rng(1000 + d["cfg"].id).random(len(wl.src)) < keep
    src = torch.from_numpy(wl.src[m].astype(np.int32)).to(dev)
    dst = torch.from_numpy(wl.dst[m].astype(np.int32)).to(dev)
    N = d["N"]
    rowptr, senders, perm = tpc.tp_csr_build(src, dst, N)
    colptr, srcedge, srcrecv = tpc.tp_csr_transpose(rowptr, senders, N)
    p = perm.long()
    return dict(plan=d["plan"], N=N, E=int(m.sum()), x=d["x"], A=d["A"], gout=d["gout"], rowptr=rowptr,
                senders=senders, colptr=colptr, srcedge=srcedge, srcrecv=srcrecv,
                Y=torch.from_numpy(wl.Y[m]).to(dev)[p].contiguous(),
                phi=torch.from_numpy(wl.phi[m]).to(dev)[p].contiguous())


def workspace_vs_edges(dev, head):
    """Device memory of one forward + backward through the public API at E/4,
    E/2 and E edges (same nodes): the allocator's peak above what was allocated
    before the calls (inputs and outputs preallocated, the binding allocates the
    workspace), and the device memory taken outside the allocator."""
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    rec = {}
    for cid in (4, 5):
        d = head if cid == head["cfg"].id else setup(cid, dev)
        row = {"workload": d["cfg"].name, "n_nodes": d["N"], "edges": [], "peak_bytes": [],
               "outside_allocator_bytes": [], "workspace_size_fwd": d["plan"].workspace_size(d["N"], 0),
               "workspace_size_bwd": d["plan"].workspace_size(d["N"], 1)}
        for keep in (0.25, 0.5, 1.0):
            s = _edge_subset(d, keep, dev)
            out = torch.empty_like(d["out"])
            grads = (torch.empty_like(s["x"]), torch.empty_like(s["Y"]), torch.empty_like(s["phi"]),
                     torch.empty_like(s["A"]))

            def step():
                tpc.tp_conv_forward(s["plan"], s["x"], s["Y"], s["phi"], s["A"], s["rowptr"], s["senders"],
                                    out=out)
                tpc.tp_conv_backward(s["plan"], s["x"], s["Y"], s["phi"], s["A"], s["rowptr"], s["senders"],
                                     s["colptr"], s["srcedge"], s["srcrecv"], s["gout"], out=grads)
            step()
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            torch.cuda.reset_peak_memory_stats()
            base = torch.cuda.memory_allocated()
            free0, res0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
            step()
            torch.cuda.synchronize()
            row["edges"].append(s["E"])
            row["peak_bytes"].append(torch.cuda.max_memory_allocated() - base)
            row["outside_allocator_bytes"].append(
                (free0 - torch.cuda.mem_get_info()[0]) - (torch.cuda.memory_reserved() - res0))
            assert tpc.tp_get_device_error() == 0
            del s, out, grads
            torch.cuda.empty_cache()
        row["independent_of_edges"] = len(set(row["peak_bytes"])) == 1
        rec[str(cid)] = row
        if d is not head:
            del d
            torch.cuda.empty_cache()
    return rec


# ----------------------------------------------------------------------------- scaling sweeps

# Sobek §5.1: fully connected profiles, in = out irreps with alternating
# parity, one SH copy per order, K = 16, 128 MiB receiver scratch budget.
SWEEP_PROFILES = ("128/64", "128/64/64", "128/64/64/64")
# Sobek Table 3: the sixteen capacity-matched profiles with OpenEquivariance's
# largest graph counts for forward, backward and double backward (copies of the
# 128-node, degree-32 graph).
TABLE3 = (("32/16", 862, 431, 215), ("32/32", 487, 243, 121), ("32/16/16", 433, 216, 108),
          ("32/32/32", 178, 88, 44), ("32/16/16/16", 244, 121, 60), ("32/32/32/32", 85, 42, 21),
          ("64/32", 217, 108, 54), ("64/64", 122, 61, 30), ("64/32/32", 108, 54, 27),
          ("64/64/64", 44, 22, 11), ("64/32/32/32", 61, 30, 15), ("64/64/64/64", 21, 10, 5),
          ("128/64", 54, 27, 13), ("128/128", 30, 15, 7), ("128/64/64", 27, 13, 6), ("128/64/64/64", 15, 7, 3))


def profile_irreps(profile: str):
    muls = [int(v) for v in profile.split("/")]
    return "+".join(f"{m}x{l}{'e' if l % 2 == 0 else 'o'}" for l, m in enumerate(muls)), len(muls) - 1


def _sweep_point(plan, graph, dev, passes, budget_s=0.25):
    """Median CUDA-event time (ms) and peak allocated memory of each pass on one
    graph: at least 5 warm-up calls and 50 ms, then 10-30 samples totalling at
    least `budget_s` (fewer for calls above a second)."""
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    from inputs import sobek_workload
    irreps = plan.irreps
    w = sobek_workload(graph, irreps, plan.sh_lmax, plan.n_radial, plan.n_w, plan.c_out)
    N, E = w["n_nodes"], len(w["src"])
    src = torch.from_numpy(w["src"].astype(np.int32)).to(dev)
    dst = torch.from_numpy(w["dst"].astype(np.int32)).to(dev)
    rowptr, senders, perm = tpc.tp_csr_build(src, dst, N)
    colptr, srcedge, srcrecv = tpc.tp_csr_transpose(rowptr, senders, N)
    p = perm.long()
    x = torch.from_numpy(w["x"]).to(dev)
    Y = torch.from_numpy(w["Y"]).to(dev)[p].contiguous()
    phi = torch.from_numpy(w["phi"]).to(dev)[p].contiguous()
    A = torch.from_numpy(w["A"]).to(dev)
    g = torch.from_numpy(w["grad_out"]).to(dev)
    del src, dst, p
    calls = {
        "fwd": lambda: tpc.tp_conv_forward(plan, x, Y, phi, A, rowptr, senders),
        "bwd": lambda: tpc.tp_conv_backward(plan, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, g),
        "dbl": lambda: tpc.tp_conv_double_backward(plan, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv,
                                                   g, x, Y, phi, A),
    }
    out = {"nodes": N, "edges": E}
    for name in passes:
        f = calls[name]
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        n = 0
        while n < 5 or time.perf_counter() - t0 < 0.05:
            f()
            torch.cuda.synchronize()
            n += 1
            if time.perf_counter() - t0 > 3.0 and n >= 2:
                break
        torch.cuda.reset_peak_memory_stats()
        times = []
        while len(times) < 30:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            f()
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
            if (len(times) >= 10 and sum(times) >= budget_s * 1e3) or (len(times) >= 3 and sum(times) > 3e3):
                break
        ms = statistics.median(times)
        out[name] = {"ms": round(ms, 4), "M_edges_per_s": round(E / (ms * 1e-3) / 1e6, 2),
                     "peak_GiB": round(torch.cuda.max_memory_allocated() / 2 ** 30, 3), "samples": len(times)}
    assert tpc.tp_get_device_error() == 0
    return out


def _sweep_plan(profile):
    import clebsch_gordan_tensor_node_b200 as tpc
    irreps, L = profile_irreps(profile)
    plan = tpc.Plan(irreps, L, irreps, 16, "uvw", "f32")
    plan.irreps, plan.sh_lmax = irreps, L
    try:
        plan.set_state_budget(128 << 20)
    except tpc.TpConvError:
        pass   # one node's state is larger: keep the default budget
    return plan


def run_sweeps(args):
    """Sobek §5.1-5.4 workloads: degree and graph-count scaling of the three
    scaling profiles, and the capacity-matched sixteen-profile grid of Table 3.
    Prints one JSON line."""
    import torch

    from inputs import SOBEK_COUNTS, SOBEK_DEGREES, sobek_count_graph, sobek_degree_graph
    dev = "cuda:0"
    torch.cuda.set_device(dev)
    res = {"kind": "sobek sweeps", "state_budget_bytes": 128 << 20, "K": 16, "dtype": "f32",
           "degree": {}, "graph_count": {}, "table3": []}
    passes = ("fwd", "bwd", "dbl")
    if "degree" in args.sweeps:
        for prof in SWEEP_PROFILES:
            plan = _sweep_plan(prof)
            res["degree"][prof] = [dict(degree=d, **_sweep_point(plan, sobek_degree_graph(d), dev, passes))
                                   for d in SOBEK_DEGREES]
            torch.cuda.empty_cache()
    if "count" in args.sweeps:
        for prof in SWEEP_PROFILES:
            plan = _sweep_plan(prof)
            res["graph_count"][prof] = [dict(copies=b, **_sweep_point(plan, sobek_count_graph(b), dev, passes))
                                        for b in SOBEK_COUNTS]
            torch.cuda.empty_cache()
    if "table3" in args.sweeps:
        for prof, bf, bb, bd in TABLE3:
            plan = _sweep_plan(prof)
            row = {"profile": prof, "n_w": plan.n_w}
            for name, b in (("fwd", bf), ("bwd", bb), ("dbl", bd)):
                row[name] = dict(copies=b, **_sweep_point(plan, sobek_count_graph(b), dev, (name,))[name])
            res["table3"].append(row)
            torch.cuda.empty_cache()
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--pass", dest="pass_", default="fwdbwd", choices=["fwd", "fwdbwd", "dbl"])
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweeps", nargs="*", default=None, choices=["degree", "count", "table3"],
                    help="run Sobek's scaling workloads instead of the benchmark step")
    args = ap.parse_args()
    if args.sweeps is not None:
        run_sweeps(argparse.Namespace(sweeps=args.sweeps or ["degree", "count", "table3"]))
        return
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
