#!/usr/bin/env python3
"""Benchmark: gradient + block-CSR Hessian assembly of the 1000x1000 cloth.

One step = one mad_eval (springs + inertia, fp32) on a fresh perturbation of
the 10^6-vertex cloth: read x and the topology, write g and every Hessian
block.  Prints ONE JSON line (rank 0).  With torchrun (N > 1) every rank runs
its own independent replica (weak scaling, no collective on the data path);
the time is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the fp64 CPU oracle instead (a bounded sample of the
same workload per step, scaled to a full step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mesh_inputs as mi  # noqa: E402

N_GRID = 1000
SEED = 1003
# compulsory bytes of one step (read x + edge list, write g + Hessian values)
V_FULL = N_GRID * N_GRID
E_FULL = 2 * N_GRID * (N_GRID - 1) + (N_GRID - 1) ** 2
NNZB_FULL = V_FULL + 2 * E_FULL
ALGO_BYTES = 4 * (3 * V_FULL) + 8 * E_FULL + 4 * (3 * V_FULL) + 36 * NNZB_FULL
PAGES_MS_1000 = 11.7  # the page's own 1000^2 mass-spring grad+Hessian time (RTX 4090)
FALLBACK_HBM_GBS = 6650.0
METRIC = "grad+Hessian assembly ms/step (1000^2 cloth); achieved HBM GB/s vs ~8 TB/s"
KERNEL = "k_rows_eval_c<float,3> (row-streaming assembly, compact row tables)"
WORKLOAD = ("mass-spring cloth 1000x1000 grid (10^6 vertices, 2,996,001 springs, "
            "6,992,002 3x3 blocks): springs + inertia, g + block-CSR H per step")


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def max_over_ranks(value: float, dist, device) -> float:
    """The largest value over all ranks (the job's time), value itself alone."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_unit(total_ms: float, steps: int, world: int) -> float:
    """Whole-job time per 1000^2 step: every rank assembles its own replica."""
    return total_ms / (steps * world)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic():
    """DRAM bytes per launch of the assembly kernel from the committed ncu
    summary, or None if the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    h = hashlib.sha256()
    for f in d.get("sources", []):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if h.hexdigest() != d.get("sources_sha256"):
        return None
    return d.get("traffic_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, dev_index=0, period=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {}
        for attr in dir(nv):
            if attr.startswith("nvmlClocksEventReason") or attr.startswith("nvmlClocksThrottleReason"):
                v = getattr(nv, attr)
                if isinstance(v, int) and v and (v & (v - 1)) == 0:
                    key = attr.replace("nvmlClocksEventReason", "").replace("nvmlClocksThrottleReason", "")
                    names.setdefault(v, key)
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h) if hasattr(
                    nv, "nvmlDeviceGetCurrentClocksEventReasons") else \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                for bit, nm in names.items():
                    if r & bit and nm not in ("GpuIdle", "ApplicationsClocksSetting"):
                        self.reasons.add(nm)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# --------------------------------------------------------------------- ours


def run_ours(args, rank, world, dist):
    import torch

    import hessian_assembly_b200 as mad

    dev = torch.device("cuda", env_int("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    st = mi.cloth_static(N_GRID, np.float32)
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"],
                      patch_faces=args.patch_faces)
    terms = mad.Terms(mask=mad.MAD_TERM_SPRING | mad.MAD_TERM_INERTIA, flags=args.flags,
                      spring_rest=torch.from_numpy(st["L0"]).to(dev), spring_k=st["k"],
                      inertia_xt=torch.from_numpy(st["xt"]).to(dev), inertia_w=st["w"])
    pool = min(args.steps + args.warmup, args.pool)
    xs = [torch.from_numpy(mi.cloth_x(N_GRID, SEED + 7919 * rank, s, np.float32)).to(dev)
          for s in range(pool)]
    g = torch.empty((st["V"], 3), dtype=torch.float32, device=dev)
    H = torch.empty((ctx.info.capacity_blocks, 3, 3), dtype=torch.float32, device=dev)

    def step(k):
        ctx.mad_eval(xs[k % pool], terms, g, H, None, stream)

    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    # The timed loop has no events between its launches: a step is exactly
    # one launch of the assembly kernel, so the loop's time per step is the
    # kernel's time per launch (an event record between back-to-back
    # launches adds about 2 us of device time).
    clocks = ClockSampler(dev.index)
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(args.warmup + k)
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist:
        dist.barrier()
    own_ms = t0.elapsed_time(t1)
    total_ms = max_over_ranks(own_ms, dist, dev)
    ms_per_step = total_ms / args.steps
    value = job_ms_per_unit(total_ms, args.steps, world)

    # end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        nnzb = ctx.info.nnzb_base
        hx = [torch.from_numpy(mi.cloth_x(N_GRID, SEED + 7919 * rank, 10_000 + s, np.float32)).pin_memory()
              for s in range(2)]
        hg = torch.empty((st["V"], 3), dtype=torch.float32).pin_memory()
        hH = torch.empty((nnzb, 3, 3), dtype=torch.float32).pin_memory()
        he = torch.empty(1, dtype=torch.float64).pin_memory()
        n_e2e = max(3, min(args.steps, 20))
        for k in range(2):
            ctx.mad_eval_host(hx[k % 2], terms, hg, hH, he, stream)
        if dist:
            dist.barrier()
        w0 = time.perf_counter()
        for k in range(n_e2e):
            ctx.mad_eval_host(hx[k % 2], terms, hg, hH, he, stream)
        w_ms = max_over_ranks((time.perf_counter() - w0) * 1e3, dist, dev)
        e2e = {"value": w_ms / (n_e2e * world), "unit": "ms/step",
               "h2d_bytes_per_step": int(hx[0].numel() * 4),
               "d2h_bytes_per_step": int(hg.numel() * 4 + hH.numel() * 4 + 8),
               "steps": n_e2e, "api": "mad_eval_host"}

    hbm, peak_kind = peaks()
    avg_launch_ms = own_ms / args.steps
    achieved = ALGO_BYTES / (avg_launch_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "traffic": kernel_traffic(),
            "kernel": KERNEL,
            "algorithmic_bytes_per_launch": ALGO_BYTES,
            "avg_launch_ms": round(avg_launch_ms, 5), "launches_timed": args.steps,
            "launch_time": "this rank's timed loop / steps (one launch per step, no events "
                           "between launches)",
            "peak_kind": peak_kind}
    out = {
        "metric": METRIC, "value": round(value, 5), "unit": "ms/step", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": False, "scaling": "weak",
        "vs_baseline": round(value / PAGES_MS_1000, 6), "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "n": N_GRID, "seed": SEED, "x_pool": pool,
                   "l2": "inputs + outputs per step 0.36 GB > 126 MB L2; x from a pool of "
                         f"{pool} distinct perturbations", "parallelism": f"replicas x{world}",
                   "assembly": "patch kernel" if args.flags & mad.MAD_EVAL_PATCH_STAGED else
                   "row-streaming kernel", "flags": args.flags},
        "roofline": roof, "e2e": e2e, "gpu_launches": args.steps, "clocks": clk,
        "impl": "ours",
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        with pinned_core() as core:
            out["cpu_baseline"] = cpu_baseline(st)
            if not args.no_extra:
                out["cpu_baseline"]["rows"] = cpu_baseline_rows(st)
        out["cpu_baseline"].update(cpu_info(core))
    if not args.no_extra and rank == 0:
        out["workloads"] = extra_workloads(args)
        out["rooflines"] = rooflines(out["workloads"], ms_per_step, hbm, peak_kind)
    ctx.close()
    return out


class pinned_core:
    """Runs the block on one host core (the process's affinity is restored
    afterwards); yields the core's index."""

    def __enter__(self):
        self.saved = os.sched_getaffinity(0)
        core = max(self.saved)
        os.sched_setaffinity(0, {core})
        return core

    def __exit__(self, *exc):
        os.sched_setaffinity(0, self.saved)
        return False


def cpu_info(core):
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cpu_model": model, "pinned_core": core, "host_cores": os.cpu_count()}


def cloth_bytes(n, esz):
    """Algorithmic bytes of one cloth step (read x and the edge list, write g
    and the Hessian blocks) on the n x n grid, floats of esz bytes."""
    V = n * n
    E = 2 * n * (n - 1) + (n - 1) ** 2
    return esz * 3 * V + 8 * E + esz * 3 * V + esz * 9 * (V + 2 * E)


def param_bytes(n):
    """Algorithmic bytes of the 500^2 parameterization (fp32, dof 2): eval
    reads UV and the face list and writes g and the 2x2 blocks; the product
    reads UV, v and the face list and writes y."""
    V = n * n
    F = 2 * (n - 1) ** 2
    E = 2 * n * (n - 1) + (n - 1) ** 2
    return 8 * V + 12 * F + 8 * V + 16 * (V + 2 * E), 8 * V * 3 + 12 * F


def rooflines(w, headline_ms, hbm, peak_kind):
    """Fraction of the HBM peak per workload: algorithmic bytes / time."""
    V, E, F, P = V_FULL, E_FULL, 2 * (N_GRID - 1) ** 2, 100_000
    pe, ph = param_bytes(500)
    rows = {
        "cloth10": (cloth_bytes(10, 4), w.get("cloth10_graph_eval_ms")),
        "cloth10_call": (cloth_bytes(10, 4), w.get("cloth10_eval_ms")),
        "cloth100": (cloth_bytes(100, 4), w.get("cloth100_graph_eval_ms")),
        "cloth100_call": (cloth_bytes(100, 4), w.get("cloth100_eval_ms")),
        "cloth100_f64": (cloth_bytes(100, 8), w.get("cloth100_f64_eval_ms")),
        "cloth1000": (ALGO_BYTES, headline_ms),
        "cloth1000_generic": (ALGO_BYTES, w.get("cloth1000_generic_eval_ms")),
        "symdir500_generic_eval": (pe, w.get("symdir500_generic_eval_ms")),
        "area1000_generic_eval": (ALGO_BYTES + 16 * F, w.get("area1000_generic_eval_ms")),
        "symdir500_eval": (pe, w.get("symdir500_eval_ms")),
        "symdir500_hvp": (ph, w.get("symdir500_hvp_ms")),
        "arap500_eval": (pe, w.get("arap500_eval_ms")),
        "arap500_hvp": (ph, w.get("arap500_hvp_ms")),
        # pairs: x, edges, pair list, g and the blocks of the pattern with the pairs
        "pairs1000_assembly": (12 * V + 8 * E + 8 * P + 12 * V + 36 * (V + 2 * E + 2 * P),
                               w.get("pairs1000_assembly_ms")),
        # insertion: read the mesh row_ptr and col_idx and the pairs, write the new ones
        "pairs1000_insert": (4 * (V + 1) * 2 + 4 * (V + 2 * E) + 4 * (V + 2 * E + 2 * P) + 8 * P,
                             w.get("pairs1000_insert_ms")),
        "jac1000": (w.get("jac1000_bytes"), w.get("jac1000_ms")),
        # the product: read x, v and the edge list, write y
        "cloth1000_hvp": (12 * V * 3 + 8 * E, w.get("cloth1000_hvp_ms")),
        "area1000_eval": (ALGO_BYTES + 16 * F, w.get("area1000_eval_ms")),
        "area1000_hvp": (12 * V * 3 + 12 * E + 16 * F, w.get("area1000_hvp_ms")),
        "vf1000_eval": (w.get("vf1000_eval_bytes"), w.get("vf1000_eval_ms")),
    }
    out = {}
    for k, (b, ms) in rows.items():
        if not b or not ms:
            continue
        gbs = b / (ms * 1e-3) / 1e9
        out[k] = {"bytes": int(b), "ms": round(ms, 5), "gbs": round(gbs, 1),
                  "frac": round(gbs / hbm, 4)}
    out["peak_gbs"] = hbm
    out["peak_kind"] = peak_kind
    out["note"] = ("algorithmic bytes (read x and topology, write g and the Hessian values "
                   "or y) / median CUDA-event time; *_call rows are single launches, the "
                   "others CUDA-graph replays where named so in workloads")
    return out


def cpu_baseline_rows(st):
    """The oracle beside each secondary workload: one run on one host core,
    on the same seeded inputs as the GPU timings of extra_workloads."""
    import oracle
    orc = oracle.load()
    res = {}
    # SymDir 500^2: pattern + assembly, then the product with the assembled H
    ps = mi.param_static(500, 1004, np.float32)
    t0 = time.perf_counter()
    rp, ci = orc.pattern(ps["V"], ps["F"])
    og, oH, _ = orc.eval(ps["V"], 2, ps["UV"], 4, rp, ci, F=ps["F"], Minv=ps["Minv"],
                         area=ps["area"])
    t1 = time.perf_counter()
    orc.bsr_mv(ps["V"], 2, rp, ci, oH, mi.probe_vector(ps["V"], 2, 1005, np.float32))
    t2 = time.perf_counter()
    res["symdir500_eval_ms"] = round((t1 - t0) * 1e3, 1)
    res["symdir500_hvp_ms"] = round((t2 - t1) * 1e3, 1)
    t0 = time.perf_counter()
    _, oH, _ = orc.eval(ps["V"], 2, ps["UV"], 32, rp, ci, F=ps["F"], Minv=ps["Minv"],
                        area=ps["area"])
    t1 = time.perf_counter()
    orc.bsr_mv(ps["V"], 2, rp, ci, oH, mi.probe_vector(ps["V"], 2, 1005, np.float32))
    t2 = time.perf_counter()
    res["arap500_eval_ms"] = round((t1 - t0) * 1e3, 1)
    res["arap500_hvp_ms"] = round((t2 - t1) * 1e3, 1)
    # cloth 1000^2 + 10^5 pairs (step 0): the pattern with the pairs, then assembly
    xx = mi.cloth_x(N_GRID, 1005, 0, np.float32)
    pp = mi.random_pairs(N_GRID, 100_000, 1005, 0)
    t0 = time.perf_counter()
    rp, ci = orc.pattern(st["V"], st["F"], pp)
    t1 = time.perf_counter()
    orc.eval(st["V"], 3, xx, 11, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"], xt=st["xt"],
             w=st["w"], pairs=pp, prest=mi.pair_rest(xx, pp, np.float32), kp=mi.PAIR_K)
    t2 = time.perf_counter()
    res["pairs1000_insert_ms"] = round((t1 - t0) * 1e3, 1)
    res["pairs1000_assembly_ms"] = round((t2 - t1) * 1e3, 1)
    # residuals + Jacobian of springs + inertia at 1000^2
    xx = mi.cloth_x(N_GRID, 1006, 0, np.float32)
    t0 = time.perf_counter()
    orc.jacobian(st["V"], 3, xx, 3, edges=st["edges"], L0=st["L0"], k=st["k"], xt=st["xt"],
                 w=st["w"])
    res["jac1000_ms"] = round((time.perf_counter() - t0) * 1e3, 1)
    # springs + inertia + area at 1000^2: assembly on the base pattern, then the product
    xx = mi.cloth_x(N_GRID, 1007, 0, np.float32)
    rp, ci = orc.pattern(st["V"], st["F"])
    t0 = time.perf_counter()
    _, oH, _ = orc.eval(st["V"], 3, xx, 19, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"],
                        xt=st["xt"], w=st["w"], F=st["F"],
                        area=cloth_rest_area(st).astype(np.float32), ka=AREA_K)
    t1 = time.perf_counter()
    orc.bsr_mv(st["V"], 3, rp, ci, oH, mi.probe_vector(st["V"], 3, 1008, np.float32))
    t2 = time.perf_counter()
    res["area1000_eval_ms"] = round((t1 - t0) * 1e3, 1)
    res["area1000_hvp_ms"] = round((t2 - t1) * 1e3, 1)
    # springs + inertia + 10^5 vertex-face terms at 1000^2: pattern with their pairs, assembly
    vf = mi.random_vf(N_GRID, N_VF, 1009, 0)
    xx = mi.cloth_x(N_GRID, 1011, 0, np.float32)
    rest = (0.001 * np.random.default_rng(1010).standard_normal(N_VF)).astype(np.float32)
    t0 = time.perf_counter()
    rp, ci = orc.pattern(st["V"], st["F"], mi.vf_pairs(vf, st["F"]))
    t1 = time.perf_counter()
    orc.eval(st["V"], 3, xx, 1 | 2 | 64, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"],
             xt=st["xt"], w=st["w"], F=st["F"], vf=vf, vf_rest=rest, kc=KC)
    t2 = time.perf_counter()
    res["vf1000_insert_ms"] = round((t1 - t0) * 1e3, 1)
    res["vf1000_eval_ms"] = round((t2 - t1) * 1e3, 1)
    res["unit"] = "ms per call, 1 core, one run"
    return res


def cpu_baseline(st):
    import oracle
    orc = oracle.load()
    rp, ci = orc.pattern(st["V"], st["F"])
    times = []
    for s in range(2):
        x = mi.cloth_x(N_GRID, SEED, 20_000 + s, np.float32)
        t0 = time.perf_counter()
        orc.eval(st["V"], 3, x, 3, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"],
                 xt=st["xt"], w=st["w"])
        times.append((time.perf_counter() - t0) * 1e3)
    return {"value": round(statistics.median(times), 1), "unit": "ms/step", "cores": 1,
            "kind": "oracle",
            "sample": "2 full 1000x1000 steps (fp64 closed forms, COO sort + merge), median"}


EXTRA = ("cloth_small", "generic1000", "hvp1000", "symdir500", "pairs1000", "jac1000", "area1000",
         "vf1000", "shard1000")
GENERIC_AD = 8  # MAD_EVAL_GENERIC_AD


def extra_workloads(args, only=None):
    """Secondary workloads (parameterization eval/HVP at 500^2, cloth with 10^5
    runtime pairs at 1000^2, the small grids), CUDA-event timed, median.
    `only` names one of EXTRA to run alone."""
    import torch

    import hessian_assembly_b200 as mad
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    res = {}
    run = lambda name: only is None or only == name  # noqa: E731

    def timeit(fn, n=50, w=5):
        for _ in range(w):
            fn()
        ts = []
        for _ in range(n):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            ts.append((a, b))
        torch.cuda.synchronize()
        return statistics.median([a.elapsed_time(b) for a, b in ts])

    # small cloths (launch-latency bound), fp32 and, at 100^2, fp64
    for n, dt in (((10, "float32"), (100, "float32"), (100, "float64")) if run("cloth_small")
                  else ()):
        npdt = np.dtype(dt)
        tdt = getattr(torch, dt)
        st = mi.cloth_static(n, npdt)
        ctx = mad.Context(st["V"], st["F"], 3, dt, part_xyz=st["X"])
        terms = mad.Terms(mask=3, spring_rest=torch.from_numpy(st["L0"]).to(dev), spring_k=st["k"],
                          inertia_xt=torch.from_numpy(st["xt"]).to(dev), inertia_w=st["w"])
        x = torch.from_numpy(mi.cloth_x(n, 1000 + n, 0, npdt)).to(dev)
        g = torch.empty((st["V"], 3), dtype=tdt, device=dev)
        H = torch.empty((ctx.info.capacity_blocks, 3, 3), dtype=tdt, device=dev)
        key = f"cloth{n}_eval_ms" if dt == "float32" else f"cloth{n}_f64_eval_ms"
        res[key] = round(timeit(lambda: ctx.mad_eval(x, terms, g, H, None, stream)), 5)
        if dt == "float32":  # the same step as a CUDA-graph replay of 20 steps
            reps = 20
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                ctx.mad_eval(x, terms, g, H, None, side)
            stream.wait_stream(side)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(reps):
                    ctx.mad_eval(x, terms, g, H)
            res[f"cloth{n}_graph_eval_ms"] = round(timeit(graph.replay) / reps, 5)
            del graph
        ctx.close()
    if run("generic1000"):
        generic1000(res, mad, torch, dev, stream, timeit)
    if run("hvp1000"):
        hvp1000(res, mad, torch, dev, stream, timeit)
    # parameterization 500^2: eval and HVP
    if run("symdir500"):
        symdir500(res, mad, torch, dev, stream, timeit)
    if run("pairs1000"):
        pairs1000(res, mad, torch, dev, stream)
    if run("jac1000"):
        jac1000(res, mad, torch, dev, stream, timeit)
    if run("area1000"):
        area1000(res, mad, torch, dev, stream, timeit)
    if run("vf1000"):
        vf1000(res, mad, torch, dev, stream, timeit)
    if run("shard1000"):
        shard1000(res, mad, torch, dev, stream, timeit)
    return res


N_VF = 100_000
KC = 50.0


def vf1000(res, mad, torch, dev, stream, timeit):
    """Springs + inertia + 10^5 vertex-face terms on the 1000^2 cloth.  The
    set is installed once (mad_add_vf: its 3 x 10^5 (vertex, corner) pairs
    inserted and the per-row term lists built), then evaluated per row after
    the row kernel (eval and product).  The same terms passed per call
    (t->vf), one thread per term adding with atomics, are timed beside it."""
    st = mi.cloth_static(N_GRID, np.float32)
    vf = mi.random_vf(N_GRID, N_VF, 1009, 0)
    pairs = mi.vf_pairs(vf, st["F"])
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"], max_pairs=len(pairs),
                      slack=0.2)
    dvf = torch.from_numpy(vf).to(dev)
    res["vf1000_insert_ms"] = round(timeit(lambda: ctx.mad_add_vf(dvf, stream), n=16), 5)
    rest = (0.001 * np.random.default_rng(1010).standard_normal(N_VF)).astype(np.float32)
    terms = mad.Terms(mask=1 | 2 | 64, spring_rest=torch.from_numpy(st["L0"]).to(dev),
                      spring_k=st["k"], inertia_xt=torch.from_numpy(st["xt"]).to(dev),
                      inertia_w=st["w"], vf=None, vf_rest=torch.from_numpy(rest).to(dev),
                      vf_k=KC)
    x = torch.from_numpy(mi.cloth_x(N_GRID, 1011, 0, np.float32)).to(dev)
    v = torch.from_numpy(mi.probe_vector(st["V"], 3, 1012, np.float32)).to(dev)
    g = torch.empty((st["V"], 3), device=dev)
    y = torch.empty((st["V"], 3), device=dev)
    H = torch.empty((ctx.info.capacity_blocks, 3, 3), device=dev)
    res["vf1000_eval_ms"] = round(timeit(lambda: ctx.mad_eval(x, terms, g, H, None, stream)), 5)
    res["vf1000_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, terms, v, y, stream)), 5)
    # read x, the edge list, the terms (vertex, face, rest) and their faces'
    # corners; write g and the blocks of the pattern holding the terms' pairs
    _, _, nz = ctx.mad_pattern()
    nnzb = int(nz.cpu()[0])
    V, E = st["V"], len(st["edges"])
    res["vf1000_eval_bytes"] = 12 * V + 8 * E + 24 * N_VF + 12 * V + 36 * nnzb
    # the same terms passed per call: atomics
    ta = mad.Terms(mask=1 | 2 | 64, spring_rest=terms.spring_rest, spring_k=st["k"],
                   inertia_xt=terms.inertia_xt, inertia_w=st["w"], vf=dvf,
                   vf_rest=terms.vf_rest, vf_k=KC)
    res["vf1000_atomic_eval_ms"] = round(timeit(lambda: ctx.mad_eval(x, ta, g, H, None, stream)), 5)
    res["vf1000_atomic_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, ta, v, y, stream)), 5)
    res["vf1000_status"] = ctx.mad_status_sync()
    ctx.close()


def generic1000(res, mad, torch, dev, stream, timeit):
    """The headline step with MAD_EVAL_GENERIC_AD: the spring energy as a plain
    expression, differentiated by the AD number types alone."""
    st = mi.cloth_static(N_GRID, np.float32)
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"])
    terms = mad.Terms(mask=3, flags=GENERIC_AD, spring_rest=torch.from_numpy(st["L0"]).to(dev),
                      spring_k=st["k"], inertia_xt=torch.from_numpy(st["xt"]).to(dev),
                      inertia_w=st["w"])
    xs = [torch.from_numpy(mi.cloth_x(N_GRID, SEED, 40_000 + s, np.float32)).to(dev)
          for s in range(4)]
    g = torch.empty((st["V"], 3), device=dev)
    H = torch.empty((ctx.info.capacity_blocks, 3, 3), device=dev)
    k = [0]

    def step():
        ctx.mad_eval(xs[k[0] % 4], terms, g, H, None, stream)
        k[0] += 1
    res["cloth1000_generic_eval_ms"] = round(timeit(step), 5)
    ctx.close()


def cloth_rest_area(st):
    X, F = st["X"], st["F"]
    return 0.5 * np.linalg.norm(np.cross(X[F[:, 1]] - X[F[:, 0]], X[F[:, 2]] - X[F[:, 0]]), axis=1)


AREA_K = 2.0e3


def area1000(res, mad, torch, dev, stream, timeit):
    """Springs + inertia + area preservation (3-DOF face term) on the 1000^2
    cloth: assembly of g and H, and the matrix-free product.  Compulsory bytes:
    the headline step plus the faces and their rest areas (assembly); x, v,
    edges, L0, faces, rest areas in and y out (product)."""
    st = mi.cloth_static(N_GRID, np.float32)
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"])
    terms = mad.Terms(mask=19, spring_rest=torch.from_numpy(st["L0"]).to(dev), spring_k=st["k"],
                      inertia_xt=torch.from_numpy(st["xt"]).to(dev), inertia_w=st["w"],
                      face_area=torch.from_numpy(cloth_rest_area(st).astype(np.float32)).to(dev),
                      area_k=AREA_K)
    x = torch.from_numpy(mi.cloth_x(N_GRID, 1007, 0, np.float32)).to(dev)
    v = torch.from_numpy(mi.probe_vector(st["V"], 3, 1008, np.float32)).to(dev)
    g = torch.empty((st["V"], 3), device=dev)
    y = torch.empty((st["V"], 3), device=dev)
    H = torch.empty((ctx.info.capacity_blocks, 3, 3), device=dev)
    nF = len(st["F"])
    eb = ALGO_BYTES + 16 * nF
    hb = 12 * V_FULL * 3 + 12 * E_FULL + 16 * nF
    ms = timeit(lambda: ctx.mad_eval(x, terms, g, H, None, stream))
    res["area1000_eval_ms"] = round(ms, 5)
    res["area1000_eval_gbs"] = round(eb / (ms * 1e-3) / 1e9, 1)
    ms = timeit(lambda: ctx.mad_hvp(x, terms, v, y, stream))
    res["area1000_hvp_ms"] = round(ms, 5)
    res["area1000_hvp_gbs"] = round(hb / (ms * 1e-3) / 1e9, 1)
    terms.flags = GENERIC_AD
    res["area1000_generic_eval_ms"] = round(timeit(lambda: ctx.mad_eval(x, terms, g, H, None, stream)), 5)
    res["area1000_generic_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, terms, v, y, stream)), 5)
    ctx.close()


def hvp1000(res, mad, torch, dev, stream, timeit):
    """The matrix-free product y = H v of the 1000^2 cloth (springs +
    inertia), with a seeded N(0,1) direction."""
    st = mi.cloth_static(N_GRID, np.float32)
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"])
    terms = mad.Terms(mask=3, spring_rest=torch.from_numpy(st["L0"]).to(dev), spring_k=st["k"],
                      inertia_xt=torch.from_numpy(st["xt"]).to(dev), inertia_w=st["w"])
    x = torch.from_numpy(mi.cloth_x(N_GRID, SEED, 0, np.float32)).to(dev)
    v = torch.from_numpy(mi.probe_vector(st["V"], 3, 1009, np.float32)).to(dev)
    y = torch.empty((st["V"], 3), device=dev)
    res["cloth1000_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, terms, v, y, stream)), 5)
    ctx.close()


def shard1000(res, mad, torch, dev, stream, timeit):
    """The 1000^2 cloth step split into 2 and 4 owner-computes shards
    (mad_eval_shard), each shard's positions in a buffer of its own, timed
    one shard at a time on this GPU: what each rank's kernel would take on
    its own GPU (the halo read from the other buffers stays on this GPU's
    memory here, not over NVLink)."""
    st = mi.cloth_static(N_GRID, np.float32)
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"])
    terms = mad.Terms(mask=3, spring_rest=torch.from_numpy(st["L0"]).to(dev), spring_k=st["k"],
                      inertia_xt=torch.from_numpy(st["xt"]).to(dev), inertia_w=st["w"])
    x = torch.from_numpy(mi.cloth_x(N_GRID, SEED, 0, np.float32)).to(dev)
    for nranks in (2, 4):
        rb, bb = mad.mad_shard_plan(st["V"], st["F"], nranks)
        parts = [x[rb[r]:rb[r + 1]].clone() for r in range(nranks)]
        ms = []
        for r in range(nranks):
            nr, nb = int(rb[r + 1] - rb[r]), int(bb[r + 1] - bb[r])
            g = torch.empty((max(nr, 1), 3), device=dev)
            H = torch.empty((max(nb, 1), 3, 3), device=dev)
            ms.append(timeit(lambda: ctx.mad_eval_shard(rb, parts, r, terms, g, H, None,
                                                          stream)))
            del g, H
        res[f"shard1000_{nranks}_rank_ms"] = [round(m, 5) for m in ms]
        res[f"shard1000_{nranks}_max_rank_ms"] = round(max(ms), 5)
    ctx.close()


def jac1000(res, mad, torch, dev, stream, timeit):
    """Residuals + sparse Jacobian of springs + inertia on the 1000^2 cloth.
    Algorithmic bytes: read x, edges, L0, xt; write r and the Jacobian values
    (the pattern is written once, outside the timed calls)."""
    st = mi.cloth_static(N_GRID, np.float32)
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"])
    terms = mad.Terms(mask=3, spring_rest=torch.from_numpy(st["L0"]).to(dev), spring_k=st["k"],
                      inertia_xt=torch.from_numpy(st["xt"]).to(dev), inertia_w=st["w"])
    rows, nnz = ctx.mad_jacobian_shape(3)
    rp = torch.empty(rows + 1, dtype=torch.int64, device=dev)
    ci = torch.empty(nnz, dtype=torch.int32, device=dev)
    r = torch.empty(rows, dtype=torch.float32, device=dev)
    J = torch.empty(nnz, dtype=torch.float32, device=dev)
    ctx.mad_jacobian_pattern(3, rp, ci, stream)
    x = torch.from_numpy(mi.cloth_x(N_GRID, 1006, 0, np.float32)).to(dev)
    ms = timeit(lambda: ctx.mad_jacobian(x, terms, r, J, stream))
    E, V = len(st["edges"]), st["V"]
    nbytes = 12 * V + 8 * E + 4 * E + 12 * V + 4 * rows + 4 * nnz
    res["jac1000_ms"] = round(ms, 5)
    res["jac1000_bytes"] = int(nbytes)
    res["jac1000_gbs"] = round(nbytes / (ms * 1e-3) / 1e9, 1)
    ctx.close()


def symdir500(res, mad, torch, dev, stream, timeit):
    ps = mi.param_static(500, 1004, np.float32)
    ctx = mad.Context(ps["V"], ps["F"], 2, "float32", part_xyz=ps["X"])
    terms = mad.Terms(mask=4, face_Minv=torch.from_numpy(ps["Minv"].reshape(-1, 4)).to(dev),
                      face_area=torch.from_numpy(ps["area"]).to(dev))
    x = torch.from_numpy(ps["UV"]).to(dev)
    v = torch.from_numpy(mi.probe_vector(ps["V"], 2, 1005, np.float32)).to(dev)
    g = torch.empty((ps["V"], 2), device=dev)
    y = torch.empty((ps["V"], 2), device=dev)
    H = torch.empty((ctx.info.capacity_blocks, 2, 2), device=dev)
    res["symdir500_eval_ms"] = round(timeit(lambda: ctx.mad_eval(x, terms, g, H, None, stream)), 5)
    res["symdir500_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, terms, v, y, stream)), 5)
    tg = mad.Terms(mask=4, flags=GENERIC_AD, face_Minv=terms.face_Minv, face_area=terms.face_area)
    res["symdir500_generic_eval_ms"] = round(timeit(lambda: ctx.mad_eval(x, tg, g, H, None, stream)), 5)
    res["symdir500_generic_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, tg, v, y, stream)), 5)
    # the same term set through the patch-staged kernel, for comparison
    tp = mad.Terms(mask=4, flags=mad.MAD_EVAL_PATCH_STAGED, face_Minv=terms.face_Minv,
                   face_area=terms.face_area)
    res["symdir500_patch_eval_ms"] = round(timeit(lambda: ctx.mad_eval(x, tp, g, H, None, stream)), 5)
    res["symdir500_patch_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, tp, v, y, stream)), 5)
    # ARAP on the same faces and inputs
    ta = mad.Terms(mask=32, face_Minv=terms.face_Minv, face_area=terms.face_area)
    res["arap500_eval_ms"] = round(timeit(lambda: ctx.mad_eval(x, ta, g, H, None, stream)), 5)
    res["arap500_hvp_ms"] = round(timeit(lambda: ctx.mad_hvp(x, ta, v, y, stream)), 5)
    ctx.close()


def pairs1000(res, mad, torch, dev, stream):
    """Cloth 1000^2 + 10^5 fresh pairs per step: insertion, assembly."""
    st = mi.cloth_static(N_GRID, np.float32)
    ctx = mad.Context(st["V"], st["F"], 3, "float32", part_xyz=st["X"])
    terms = mad.Terms(mask=11, spring_rest=torch.from_numpy(st["L0"]).to(dev), spring_k=st["k"],
                      inertia_xt=torch.from_numpy(st["xt"]).to(dev), inertia_w=st["w"],
                      pair_k=mi.PAIR_K)
    nst = 8
    xs, ps_, rs = [], [], []
    for s in range(nst):
        xx = mi.cloth_x(N_GRID, 1005, s, np.float32)
        pp = mi.random_pairs(N_GRID, 100_000, 1005, s)
        xs.append(torch.from_numpy(xx).to(dev))
        ps_.append(torch.from_numpy(pp).to(dev))
        rs.append(torch.from_numpy(mi.pair_rest(xx, pp, np.float32)).to(dev))
    g = torch.empty((st["V"], 3), device=dev)
    H = torch.empty((ctx.info.capacity_blocks, 3, 3), device=dev)
    ins, asm = [], []
    for s in range(3 * nst):
        k = s % nst
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        ctx.mad_add_pairs(ps_[k], rs[k], stream)
        b.record(stream)
        ctx.mad_eval(xs[k], terms, g, H, None, stream)
        c.record(stream)
        if s >= nst:
            ins.append((a, b))
            asm.append((b, c))
    torch.cuda.synchronize()
    res["pairs1000_insert_ms"] = round(statistics.median([a.elapsed_time(b) for a, b in ins]), 5)
    res["pairs1000_assembly_ms"] = round(statistics.median([a.elapsed_time(b) for a, b in asm]), 5)
    res["pairs1000_status"] = ctx.mad_status_sync(stream)
    ctx.close()


# ---------------------------------------------------------------- reference


# Whole 1000^2 oracle steps take about 2 s each on one host core; runs of
# more steps than this time a bounded sample per step instead.
REF_FULL_STEPS_MAX = 40


def run_reference(args):
    """The oracle on one pinned host core.  Each step is a whole 1000^2 cloth
    step (fp64 closed forms, COO sort + merge) on a fresh perturbation, when
    warm-up + timed steps <= REF_FULL_STEPS_MAX; otherwise each step is the
    same workload on the 250x250 grid, scaled to a 1000^2 step by the ratio
    of term counts (stated in `sample`)."""
    import oracle
    orc = oracle.load()
    full = args.steps + args.warmup <= REF_FULL_STEPS_MAX
    ns = N_GRID if full else args.ref_sample_n
    st = mi.cloth_static(ns, np.float32)
    rp, ci = orc.pattern(st["V"], st["F"])
    terms_s = st["edges"].shape[0] + st["V"]
    scale = (E_FULL + V_FULL) / terms_s
    xs = [mi.cloth_x(ns, SEED, 30_000 + s, np.float32) for s in range(2)]

    def step(k):
        orc.eval(st["V"], 3, xs[k % 2], 3, rp, ci, edges=st["edges"], L0=st["L0"], k=st["k"],
                 xt=st["xt"], w=st["w"])

    with pinned_core() as core:
        for k in range(args.warmup):
            step(k)
        t0 = time.perf_counter()
        for k in range(args.steps):
            step(k)
        ms = (time.perf_counter() - t0) * 1e3 / args.steps * scale
    if full:
        sample = f"whole {N_GRID}x{N_GRID} steps ({terms_s} terms), two perturbations alternating"
    else:
        sample = (f"{ns}x{ns} grid per step ({terms_s} terms), scaled by {scale:.3f} to a "
                  f"{N_GRID}x{N_GRID} step")
    cpu = {"value": round(ms, 3), "unit": "ms/step", "cores": 1, "kind": "oracle",
           "sample": sample}
    cpu.update(cpu_info(core))
    return {"metric": METRIC, "value": round(ms, 3), "unit": "ms/step", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": round(ms / PAGES_MS_1000, 4),
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "n": N_GRID, "sample": sample},
            "cpu_baseline": cpu,
            "e2e": {"value": round(ms, 3), "unit": "ms/step", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--pool", type=int, default=32)
    ap.add_argument("--patch-faces", type=int, default=512)
    ap.add_argument("--flags", type=int, default=0, help="MAD_EVAL_* bits for the timed step")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--ref-sample-n", type=int, default=250)
    ap.add_argument("--only", choices=EXTRA, default=None,
                    help="run one secondary workload alone and print its timings")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.only:
        if rank == 0:
            import torch
            torch.cuda.init()
            print(json.dumps({"workloads": extra_workloads(args, args.only)}), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(env_int("LOCAL_RANK", 0))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    out = run_ours(args, rank, world, dist)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
