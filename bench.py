"""Benchmark of the edge-conditioned CG tensor-product convolution on B200.

Metric: TP-conv edges/s (forward, and forward+backward where the workload has a
backward) with the achieved fraction of the roofline. The headline line times
the forward of the MACE-like channelwise fp32 workload (4096 atoms, ~131k
edges, 128x0e+128x1o -> 128x(0e+1o+2e+3o), L_sh 3, K 8). A step is one
forward over that batch with every input resident in HBM. The L2 (126 MB) is
flushed between timed steps by writing a 256 MiB buffer outside the timed
events, because this workload's inputs fit in L2.

Multi-GPU: the operator has no exchange step for independent batches, so each
rank runs its own replica (weak scaling) and rank 0 reports the max time over
ranks. `--impl reference` times the CPU oracle on the host cores instead.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                       [--config C] [--no-extra] [--no-cpu-baseline]
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

def setup(cid: int, dev: str, n_nodes=None):
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    from inputs import CONFIGS, make_workload
    c = CONFIGS[cid]
    plan = tpc.Plan(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode, c.dtype)
    wl = make_workload(cid, plan.n_w, n_nodes=n_nodes)
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


def time_steps(step, steps: int, warmup: int, flush, sampler=None, dist=None):
    """Per-step CUDA-event times (ms) on the current stream, L2 flushed in between."""
    import torch
    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        flush()
        a.record()
        step()
        b.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs], clocks


def roofline_fb(d, ms: float) -> dict:
    f0, b0 = d["plan"].work_model(d["N"], d["E"], 0)
    f1, b1 = d["plan"].work_model(d["N"], d["E"], 1)
    r = roofline(d, 0, ms)
    ach = (f0 + f1) / (ms * 1e-3) / 1e12
    r.update({"achieved": round(ach, 3), "frac": round(ach / r["peak"], 4), "algorithmic_flops": f0 + f1,
              "compulsory_bytes": b0 + b1})
    return r


# DRAM bytes (read + write) per launch of the kernel that a (workload, pass)
# timing is dominated by, from one ncu capture of the current kernel (the
# summary under profiles/ names the command); None where no capture of the
# current kernel exists.
NCU_TRAFFIC = {
    (2, 0): (21_665_024 + 564_480, "uvu_fwd_kernel", "profiles/uvu_fwd_kernel_mace_4096.md"),
}


def roofline(d, pass_: int, ms: float) -> dict:
    flops, nbytes = d["plan"].work_model(d["N"], d["E"], pass_)
    dt = d["cfg"].dtype
    peak = alu_peak(dt)
    ach = flops / (ms * 1e-3) / 1e12
    r = {"bound": "alu", "achieved": round(ach, 3), "peak": round(peak, 2), "unit": "TFLOP/s",
         "frac": round(ach / peak, 4), "traffic": None,
         "peak_source": f"derived: {SMS} SMs x {FP32_LANES if dt == 'f32' else FP64_LANES} "
                        f"{'FP32' if dt == 'f32' else 'FP64'} FMA lanes x 2 x {MAX_MHZ:.0f} MHz",
         "algorithmic_flops": flops, "compulsory_bytes": nbytes,
         "hbm_frac_of_measured": None}
    t = NCU_TRAFFIC.get((d["cfg"].id, pass_))
    if t is not None:
        hbm = measured_hbm_gbs()
        r["traffic"] = t[0]
        r["traffic_source"] = f"{t[1]}: dram__bytes_read.sum + dram__bytes_write.sum, {t[2]}"
        if hbm:
            r["hbm_frac_of_measured"] = round(t[0] / (ms * 1e-3) / 1e9 / hbm, 4)
    return r


def measured_hbm_gbs():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- CPU oracle

def cpu_oracle_sample(cid: int, budget_s: float = 15.0):
    """Oracle forward on a bounded receiver sample of the workload: edges/s on host cores."""
    from inputs import CONFIGS, make_workload
    from oracle import conv as oconv
    c = CONFIGS[cid]
    pr = oconv.Problem(c.irreps_in, c.sh_lmax, c.irreps_out, c.K, c.mode)
    wl = make_workload(cid, pr.n_w)
    rng = np.random.default_rng(0)
    order = rng.permutation(wl.n_nodes)
    done_e, t_used, n_recv = 0, 0.0, 0
    chunk = 64
    while t_used < budget_s and n_recv < wl.n_nodes:
        recv = order[n_recv:n_recv + chunk]
        sel = np.isin(wl.dst, recv)
        t0 = time.perf_counter()
        oconv.forward(pr, wl.x, wl.Y[sel], wl.phi[sel], wl.A, wl.src[sel], wl.dst[sel], wl.n_nodes)
        t_used += time.perf_counter() - t0
        done_e += int(sel.sum())
        n_recv += len(recv)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return {"value": round(done_e / t_used, 1), "unit": "edges/s", "cores": cores, "kind": "oracle",
            "sample": f"forward of {n_recv} random receivers ({done_e} edges) of workload {cid}, "
                      f"{t_used:.1f} s", "host_cpus": os.cpu_count(), "workload_edges": len(wl.src)}


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
    if rank != 0:
        return
    from inputs import CONFIGS
    c = CONFIGS[args.config]
    per_step = []
    for _ in range(args.warmup):
        cpu_oracle_sample(args.config, budget_s=1.0)
    edges = 0
    for _ in range(args.steps):
        r = cpu_oracle_sample(args.config, budget_s=max(1.0, 20.0 / max(1, args.steps)))
        per_step.append(r["value"])
    val = statistics.median(per_step)
    # a step of the workload at the sample's rate
    ms_step = round(1e3 * r["workload_edges"] / val, 3)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "edges/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": c.dtype, "data": "synthetic",
            "config": {"workload": c.name, "pass": "forward"},
            "cpu_baseline": {"value": val, "unit": "edges/s", "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
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
    both = args.pass_ == "fwdbwd"

    def step():
        fwd(d)
        if both:
            bwd(d)

    times, clocks = time_steps(step, args.steps, args.warmup, flush, sampler, dist)
    t_total, value = aggregate_ranks(sum(times), d["E"], args.steps, world, dist, dev)
    ms = t_total / args.steps
    import clebsch_gordan_tensor_node_b200 as tpc
    assert tpc.tp_get_device_error() == 0
    res = {"metric": METRIC, "value": round(value, 1), "unit": "edges/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": c.dtype,
           "data": "synthetic",
           "config": {"workload": c.name, "pass": "forward+backward" if both else "forward",
                      "n_nodes": d["N"], "n_edges": d["E"],
                      "irreps_in": c.irreps_in, "irreps_out": c.irreps_out, "sh_lmax": c.sh_lmax,
                      "n_radial": c.K, "mode": c.mode, "parallelism": f"replicas x{world}",
                      "l2": "flushed between steps (256 MiB write outside the timed events)"},
           "gpu_launches": args.steps * (d["plan"].launch_count(d["N"], 0)
                                         + (d["plan"].launch_count(d["N"], 1) if both else 0)),
           "roofline": roofline(d, 0, ms) if not both else roofline_fb(d, ms), "clocks": clocks}
    # end to end through the public API: pinned host inputs -> device -> forward -> host result
    res["e2e"] = e2e(d, args, dev)
    if rank == 0 and not args.no_extra:
        res["workloads"] = extra_workloads(args, dev, flush)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_oracle_sample(args.config)
    if rank == 0:
        print(json.dumps(res), flush=True)


def e2e(d, args, dev):
    import torch
    host = {k: d[k].cpu().pin_memory() for k in ("x", "Y", "phi", "A", "rowptr", "senders")}
    devb = {k: torch.empty_like(d[k]) for k in host}
    out_h = torch.empty(d["out"].shape, dtype=d["out"].dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()
    import clebsch_gordan_tensor_node_b200 as tpc

    def step():
        for k in host:
            devb[k].copy_(host[k], non_blocking=True)
        o = tpc.tp_conv_forward(d["plan"], devb["x"], devb["Y"], devb["phi"], devb["A"], devb["rowptr"],
                                devb["senders"], out=d["out"], ws=d["ws_f"])
        out_h.copy_(o, non_blocking=True)

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
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4)}


def extra_workloads(args, dev, flush):
    """Every workload's forward and (where defined) forward+backward."""
    import torch

    import clebsch_gordan_tensor_node_b200 as tpc
    out = {}
    for cid in (1, 2, 3, 4, 5):
        try:
            d = setup(cid, dev)
        except tpc.TpConvError as e:
            out[str(cid)] = {"skipped": str(e)}
            continue
        try:
            k = 20 if d["E"] < 1_000_000 else 8
            tf, _ = time_steps(lambda: fwd(d), k, 3, flush)
            ms_f = statistics.median(tf)
            rec = {"workload": d["cfg"].name, "n_nodes": d["N"], "n_edges": d["E"], "dtype": d["cfg"].dtype,
                   "fwd_ms": round(ms_f, 5), "fwd_edges_per_s": round(d["E"] / (ms_f * 1e-3), 1),
                   "fwd_roofline_frac": roofline(d, 0, ms_f)["frac"]}
            if d["cfg"].backward:
                tb, _ = time_steps(lambda: bwd(d), k, 3, flush)
                ms_b = statistics.median(tb)
                rec.update({"bwd_ms": round(ms_b, 5),
                            "fwd_bwd_edges_per_s": round(d["E"] / ((ms_f + ms_b) * 1e-3), 1),
                            "bwd_roofline_frac": roofline(d, 1, ms_b)["frac"],
                            "workspace_bwd_bytes": d["plan"].workspace_size(d["N"], 1)})
            assert tpc.tp_get_device_error() == 0
            out[str(cid)] = rec
        except tpc.TpConvError as e:
            out[str(cid)] = {"skipped": str(e)}
        del d
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "fwdbwd"])
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
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
