"""Benchmark of the quantized gated FFN / MoE layer library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--M M] [--impl ours|reference]

One step = one call of the layer (every kernel of its path) on one batch of M
seeded synthetic token rows, with the weights resident in HBM. The default
workload is the Mixtral-shaped MoE prefill at M = 512 token rows (hidden 4096,
8 experts of intermediate 14336, top-2, INT4-affine group-32 weights, SiLU, raw
residual add), the largest configuration that fits one GPU; ``--config 2 --M 1``
selects the Llama-3-8B-shaped dense decode step, and so on.

Printed: one JSON line (rank 0) with tokens/s over all ranks, weight-stream
GB/s, the roofline of the dominant kernel (CUDA-event durations of its launches
measured in a second pass of the same steps), the end-to-end number through the
C ABI with host buffers, SM clocks sampled during the timed region and the CPU
oracle's throughput on a bounded sample of the same workload.

Multi-GPU (torchrun): replicas only. Every rank runs the same workload on its
own GPU; the time is the max over ranks; value = all ranks' tokens / that time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--config", type=int, default=5)
    p.add_argument("--M", type=int, default=512)
    p.add_argument("--warm-seconds", type=float, default=1.0,
                   help="after the --warmup steps, keep running back-to-back steps for at least this long so "
                        "the GPU clocks have ramped before the timed region")
    p.add_argument("--min-timed-seconds", type=float, default=1.5,
                   help="the K-step timed loop is repeated until this much device time is covered (at least 3 "
                        "repeats); value uses the median repeat, and clocks are sampled over all of them")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--graph", action="store_true",
                   help="time CUDA graph replays of the library calls instead of eager calls (on B200 the replays "
                        "measured 1-3 us per step slower: the captured launches lose part of their programmatic overlap)")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 0)), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------------------- workload accounting


def algorithmic_bytes(c: synth.LayerConfig, w: synth.LayerInputs, M: int, union_size=None):
    """Weight bytes the method must read per call, per kernel role."""
    if c.kind in ("dense", "shared"):
        gu = w.ffn.gate.nbytes + w.ffn.up.nbytes
        dn = w.ffn.down.nbytes
        extra = w.norm_w.nbytes if w.norm_w is not None else 0
        return {"gateup": gu, "down": dn, "total": gu + dn + extra}
    u = union_size if union_size is not None else min(c.E, M * c.k)
    e = w.experts[0]
    gu = u * (e.gate.nbytes + e.up.nbytes)
    dn = u * e.down.nbytes
    if w.shared is not None:
        gu += w.shared.gate.nbytes + w.shared.up.nbytes
        dn += w.shared.down.nbytes
    extra = w.router.nbytes + (w.w_sg.nbytes if w.w_sg is not None else 0)
    return {"gateup": gu, "down": dn, "total": gu + dn + extra}


def algorithmic_flops(c: synth.LayerConfig, M: int):
    """Multiply-add flops (2 per MAC) of the method's contractions per call, per kernel role."""
    if c.kind in ("dense", "shared"):
        return {"gateup": 2.0 * M * 2 * c.I * c.H, "down": 2.0 * M * c.I * c.H}
    P = M * c.k
    gu = 2.0 * P * 2 * c.I * c.H + 2.0 * M * 2 * c.I_s * c.H
    dn = 2.0 * P * c.I * c.H + 2.0 * M * c.I_s * c.H
    return {"gateup": gu, "down": dn}


def max_over_ranks(dist, value: float, device) -> float:
    """The largest of every rank's value (all ranks call this in the same
    order); the value itself without a process group."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, M: int, steps: int, ms_total: float) -> float:
    """Whole-job tokens/s: every rank runs M token rows per step on its own GPU
    (replicas), timed as the slowest rank."""
    return world * M * steps / (ms_total * 1e-3)


def workload_name(c, M):
    return f"cfg{c.cfg} {c.name} M={M}"


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi clock / throttle samples every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# --------------------------------------------------------------------------- our arm


class GpuLayer:
    """Device-resident copies of one configuration's weights (a ring of copies
    so that consecutive steps read weights not left in L2)."""

    def __init__(self, lib, torch, c, w, ring):
        self.lib, self.torch, self.c = lib, torch, c
        self.copies = []

        def clone_qw(q):
            return lib.QWeight(q.format, q.rows, q.cols, q.q.clone(),
                               None if q.scale is None else q.scale.clone(), None if q.min is None else q.min.clone())

        def clone_ffn(f):
            return lib.FFN(clone_qw(f.gate), clone_qw(f.up), clone_qw(f.down))

        if c.kind in ("dense", "shared"):
            base = lib.upload_ffn(w.ffn)
            norm_w = torch.from_numpy(w.norm_w.view(np.int16)).cuda() if c.kind == "shared" else None
            for i in range(ring):
                self.copies.append({"ffn": base if i == 0 else clone_ffn(base), "norm_w": norm_w})
        else:
            r = w.router
            rt = torch.from_numpy(r).cuda() if r.dtype == np.float32 else torch.from_numpy(r.view(np.int16)).cuda()
            router = lib.plain_weight(rt)
            sg = lib.plain_weight(torch.from_numpy(w.w_sg.view(np.int16)).cuda()) if w.w_sg is not None else None
            base_sh = lib.upload_ffn(w.shared) if w.shared is not None else None
            base_ex = [lib.upload_ffn(e) for e in w.experts]
            for i in range(ring):
                ex = base_ex if i == 0 else [clone_ffn(e) for e in base_ex]
                sh = base_sh if (i == 0 or base_sh is None) else clone_ffn(base_sh)
                self.copies.append({"plan": lib.MoePlan(router, ex, c.k, c.act, sh, sg), "keep": (ex, sh)})

    def ws_bytes(self, M):
        c, lib = self.c, self.lib
        if c.kind == "dense":
            return lib.workspace_bytes(lib.KIND_DENSE, M, c.H, c.I)
        if c.kind == "shared":
            return lib.workspace_bytes(lib.KIND_SHARED, M, c.H, c.I)
        return self.copies[0]["plan"].workspace_bytes(M)

    def step(self, i, x, res, out, ws):
        d = self.copies[i % len(self.copies)]
        lib, c = self.lib, self.c
        if c.kind == "dense":
            lib.ffn_dense(d["ffn"], x, res, c.act, ws=ws)
        elif c.kind == "shared":
            lib.ffn_shared_expert(d["ffn"], x, d["norm_w"], out, c.act, c.eps, ws=ws)
        else:
            lib.moe_layer(d["plan"], x, res, ws=ws)


def run_ours(args, rank, world, local_rank):
    import torch
    import moe_expert_layer_dequant_b200 as lib

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    c = synth.CONFIGS[args.config]
    M = args.M
    w = synth.make_weights(c, args.seed)
    inp = synth.make_inputs(c, M, args.seed, weights=w)
    # Ring of device copies of the weights: enough copies that two steps'
    # weight reads exceed twice the L2, so each step reads from HBM.
    per_step = algorithmic_bytes(c, w, M)["total"]
    ring = int(np.ceil(2 * L2_BYTES / max(per_step, 1))) + 1
    ring = max(1, min(ring, 128, int(8e9 // max(w.weight_bytes_total(), 1))))
    layer = GpuLayer(lib, torch, c, w, ring)
    x = torch.from_numpy(inp.x.view(np.int16)).cuda()
    res0 = torch.from_numpy(inp.residual.view(np.int16)).cuda()
    res = res0.clone()
    out = torch.empty_like(x)
    ws = lib.alloc_workspace(layer.ws_bytes(M))
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    # warm-up: the --warmup steps, then back-to-back steps until at least
    # --warm-seconds of device time have passed (a GPU starts a lease at idle
    # clocks; a few steps are not enough for them to ramp)
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    n_warm = 0
    for _ in range(args.warmup):
        layer.step(n_warm, x, res, out, ws)
        n_warm += 1
    torch.cuda.synchronize()
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < args.warm_seconds:
        for _ in range(4):
            layer.step(n_warm, x, res, out, ws)
            n_warm += 1
        torch.cuda.synchronize()
    w1.record(stream)
    torch.cuda.synchronize()
    est_step_ms = w0.elapsed_time(w1) / max(n_warm, 1)
    warm_desc = (f"{args.warmup} counted steps, then back-to-back steps for >= {args.warm_seconds:g} s "
                 f"({n_warm} steps in all)")

    # With --graph: one CUDA graph per weight copy, each holding one step's
    # library calls (kernel parameters, tensor maps included, fixed at
    # capture), replayed in the timed region. Eager calls otherwise, or if a
    # capture fails.
    graphs = []
    graph_error = "default; --graph replays CUDA graphs"
    try:
        if not args.graph:
            raise RuntimeError("eager timing")
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            for i in range(len(layer.copies)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    layer.step(i, x, res, out, ws)
                graphs.append(g)
        torch.cuda.current_stream().wait_stream(cap)
        for i in range(max(args.warmup, len(graphs))):
            graphs[i % len(graphs)].replay()
        torch.cuda.synchronize()
    except Exception as exc:   # noqa: BLE001 - report and time eagerly
        graphs = []
        if args.graph:
            graph_error = f"graph capture failed: {type(exc).__name__}: {exc}"

    def timed_step(i):
        if graphs:
            graphs[i % len(graphs)].replay()
        else:
            layer.step(i, x, res, out, ws)

    # timed region: exactly K steps between events, bracketed by a barrier and
    # a synchronize; the K-step loop is repeated (at least 3 times, until
    # --min-timed-seconds of device time are covered) so that the clock
    # sampler sees the GPU under load, and the median repeat is reported
    reps = max(3, int(np.ceil(args.min_timed_seconds * 1e3 / max(est_step_ms * args.steps, 1e-3))))
    reps = int(max_over_ranks(dist, float(min(reps, 1000)), "cuda"))   # every rank runs the same repeats
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    rep_ms = []
    for _ in range(reps):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            timed_step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        rep_ms.append(e0.elapsed_time(e1))
    clocks = sampler.stop()
    ms_total = max_over_ranks(dist, statistics.median(rep_ms), "cuda")
    ms_step = ms_total / args.steps

    # per-step distribution: events around every call, in a pass of its own
    n_dist = min(args.steps, 500)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_dist)]
    for i in range(n_dist):
        evs[i][0].record(stream)
        layer.step(i, x, res, out, ws)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    st = sorted(a.elapsed_time(b) * 1000.0 for a, b in evs)
    step_us = {"median": round(st[len(st) // 2], 3), "p10": round(st[int(0.1 * (len(st) - 1))], 3),
               "p90": round(st[int(0.9 * (len(st) - 1))], 3), "steps": n_dist,
               "how": "CUDA events around each call in a separate pass (value uses the uninterrupted timed loop)"}

    # second pass of the same steps with per-launch events (roofline)
    lib.profile_enable(True)
    lib.profile_read()
    for i in range(args.steps):
        layer.step(i, x, res, out, ws)
    torch.cuda.synchronize()
    prof = lib.profile_read()
    lib.profile_enable(False)

    # end to end: host (pinned) buffers in, result out, every step
    hx = torch.from_numpy(inp.x.view(np.int16)).pin_memory()
    hres = torch.from_numpy(inp.residual.view(np.int16)).pin_memory()
    hout = torch.empty_like(hres).pin_memory()
    e2e_steps = max(10, args.steps // 4)
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for i in range(e2e_steps):
        x.copy_(hx, non_blocking=True)
        res.copy_(hres, non_blocking=True)
        layer.step(i, x, res, out, ws)
        src = out if c.kind == "shared" else res
        hout.copy_(src, non_blocking=True)
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(dist, f0.elapsed_time(f1), "cuda")

    # union size of the measured batch (MoE), from the library's own router
    union = None
    if c.kind == "moe":
        idx, _ = lib.moe_router_topk(layer.copies[0]["plan"].router, x, c.k)
        union = int(torch.unique(idx).numel())
    ab = algorithmic_bytes(c, w, M, union)

    result = None
    if rank == 0:
        hbm, bf16_tf, bf16_sus, peak_src = measured_peaks()
        tok_s = replica_throughput(world, M, args.steps, ms_total)
        weight_gbs = ab["total"] / (ms_step * 1e-3) / 1e9
        # dominant kernel: largest share of device time in the profiled pass
        dom_name, (dom_n, dom_ms) = max(prof.items(), key=lambda kv: kv[1][1])
        fl = algorithmic_flops(c, M)
        fl["total"] = fl["gateup"] + fl["down"]
        role = "gateup" if "gateup" in dom_name else ("down" if "down" in dom_name else None)
        dom_bytes = ab[role] if role else None
        dom_avg_s = dom_ms / dom_n * 1e-3
        dom_flops = fl[role] if role else None
        # bound: the larger of the weight-stream time and the tensor-core time
        tensor_bound = bool(dom_flops and "gemm_tc" in dom_name and bf16_tf > 0 and
                            dom_flops / (bf16_tf * 1e12) > dom_bytes / (hbm * 1e9))
        # A GEMM timed inside seconds of back-to-back steps runs under the
        # power cap: its denominator is the sustained bf16 figure (a GEMM loop
        # of seconds); the burst figure (a kernel timed alone) is given too.
        long_loop = sum(rep_ms) >= 1000.0 and bf16_sus > 0
        if tensor_bound:
            achieved = dom_flops / dom_avg_s / 1e12
            if long_loop:
                roof_peak, roof_unit = bf16_sus, "TFLOP/s"
                roof_src = (f"{peak_src} bf16 dense GEMM, sustained (the kernel runs inside {sum(rep_ms) / 1e3:.1f} s "
                            f"of back-to-back steps under the power cap)")
            else:
                roof_peak, roof_unit, roof_src = bf16_tf, "TFLOP/s", f"{peak_src} bf16 dense GEMM (burst)"
        else:
            achieved = dom_bytes / dom_avg_s / 1e9 if dom_bytes else None
            roof_peak, roof_unit, roof_src = hbm, "GB/s", f"{peak_src} HBM copy bandwidth"
        traffic = load_traffic(c, M, dom_name)
        launches = sum(n for n, _ in prof.values())     # library launches of one K-step loop
        result = {
            "metric": "FFN/MoE layer tokens/s (weight-stream HBM GB/s and % of B200 roofline alongside)",
            "value": round(tok_s, 2),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 6),
            "step_us": step_us,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": dtype_label(prof, c),
            "data": "synthetic (seeded; shapes and value distributions of the configuration)",
            "config": {
                "workload": workload_name(c, M), "M": M, "H": c.H, "I": c.I, "format": c.fmt,
                "act": c.act, "parallelism": "replicas" if world > 1 else "single-gpu",
                "launch": (f"CUDA graph replay ({len(graphs)} graphs, one per weight copy, each one step of library calls)"
                           if graphs else f"eager library calls ({graph_error})"),
                "warmup": warm_desc,
                "timing": f"median of {reps} repeats of the {args.steps}-step loop (each bracketed by a barrier and "
                          f"a synchronize; device events)",
                "l2": f"weight ring of {ring} device copies; each step reads the next copy "
                      f"({per_step / 1e6:.1f} MB read per step, {ring * per_step / 1e6:.0f} MB per ring turn > 126 MB L2)",
            },
            "weight_bytes_per_step": ab["total"],
            "weight_gbs": round(weight_gbs, 1),
            "weight_frac_of_measured_hbm": round(weight_gbs / hbm, 4),
            "weight_frac_of_8tbs": round(weight_gbs / 8000.0, 4),
            "roofline": {
                "kernel": dom_name, "bound": "tensor" if tensor_bound else "hbm",
                "achieved": round(achieved, 1) if achieved else None,
                "peak": roof_peak, "peak_source": roof_src, "unit": roof_unit,
                "frac": round(achieved / roof_peak, 4) if achieved else None,
                "frac_of_burst_peak": (round(achieved / bf16_tf, 4) if tensor_bound and achieved and bf16_tf > 0 else None),
                "traffic": traffic,
                "algorithmic_bytes_per_launch": dom_bytes, "algorithmic_flops_per_launch": dom_flops,
                "avg_launch_us": round(dom_avg_s * 1e6, 3),
                "timing_note": "per-launch CUDA events on the launching stream; with programmatic dependent "
                               "launch a kernel starts before its predecessor ends and its interval includes that "
                               "wait, so achieved and frac are lower bounds (the per-step value is exact)",
            },
            "kernels": {k: {"launches": n, "avg_us": round(ms / n * 1e3, 3), "share": round(ms / sum(v[1] for v in prof.values()), 4)}
                        for k, (n, ms) in prof.items()},
            "e2e": {
                "value": round(replica_throughput(world, M, e2e_steps, e2e_ms), 2), "unit": "tokens/s",
                "h2d_bytes_per_step": int(inp.x.nbytes + inp.residual.nbytes),
                "d2h_bytes_per_step": int(inp.residual.nbytes),
            },
            "gpu_launches": int(launches),
            "device_faults": lib.device_faults(True),
            "clocks": clocks,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def dtype_label(prof, c):
    """The arithmetic the path computes in, from the kernels that ran."""
    names = list(prof)
    wfmt = "int4-affine" if c.fmt == synth.FMT_INT4_G32 else "int8"
    if any("gemm_tc" in k for k in names):
        return f"bf16 ({wfmt} weights dequantized to bf16 on the tensor cores, fp32 accumulate)"
    return (f"int16 fixed-point x {wfmt} ({wfmt} codes times activations staged as int16 with one power-of-two "
            f"factor per 32-element chunk, exact int32 sums, fp32 scale and accumulate)")


def load_traffic(c, M, kernel_name):
    """dram bytes per launch of the dominant kernel from the committed ncu summary, if it matches."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d.get(f"cfg{c.cfg}-M{M}", {}).get(kernel_name)
    except Exception:
        return None


# --------------------------------------------------------------------------- CPU oracle


def time_oracle(c, M, seed, budget_s=20.0, max_reps=3):
    """The oracle as it stands on this host's cores, on a bounded sample of the workload."""
    import oracle
    w = synth.make_weights(c, seed)
    inp = synth.make_inputs(c, M, seed, weights=w)
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
    except Exception:
        info = []
    tokens = [0]
    done, t0 = 0, time.perf_counter()
    reps = 0
    while True:
        oracle.layer(inp, tokens=tokens)
        reps += 1
        done += len(tokens)
        el = time.perf_counter() - t0
        if el > budget_s * 0.5 or reps >= max_reps:
            break
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
    except Exception:
        pass
    threads = max([i.get("num_threads", 1) for i in info] + [1])
    return {"value": round(done / el, 4), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} oracle call(s) of 1 token row each of {workload_name(c, M)} (full layer incl. "
                      f"dequantization of every weight read), {el:.1f} s; numpy float64, BLAS threads={threads}, "
                      f"elementwise dequant single-threaded"}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    c = synth.CONFIGS[args.config]
    if args.impl == "reference":
        if rank != 0:
            return 0
        cb = time_oracle(c, args.M, args.seed, budget_s=60.0, max_reps=max(1, args.steps))
        line = {"impl": "reference", "metric": "FFN/MoE layer tokens/s (weight-stream HBM GB/s and % of B200 roofline alongside)",
                "value": cb["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded)", "config": {"workload": workload_name(c, args.M), "M": args.M},
                "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    res = run_ours(args, rank, world, local_rank)
    if rank == 0 and res is not None:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = time_oracle(c, args.M, args.seed)
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
