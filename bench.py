#!/usr/bin/env python
"""Benchmark: gated RMSNorm forward + backward on B200, through librn's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = rmsnorm_fwd + rmsnorm_bwd (the backward kernel and its dw fold)
with the workload's gate activation and weight offset; by default the gated
operator (silu, offset 0: the kernels gated_norm_fwd / gated_norm_bwd run) over
one batch of 262144 rows (8192 tokens x 32 heads) x 128, bf16, with 1% of
channels scaled x50 in x, z and dy (seeded synthetic data).  --workload picks
another configuration or a variant (sigmoid gate, fp16, offset).  Prints one
JSON line on rank 0.

value     = algorithmic HBM bytes of all steps on all ranks / max-over-ranks time
            (GB/s); the byte model counts each tensor once: forward reads x, z
            and writes y, rstd; backward reads x, z, dy, rstd and writes dx,
            dz; w once per call, dw once.
L2        = four buffer sets rotate (forward on set k%4, backward on set
            (k+2)%4), so a buffer is touched again only after two steps over
            other buffers (>= 512 MB, more than the 126 MB L2).
roofline  = the backward call (k_bwd + its fold launches), the dominant one:
            its algorithmic bytes / its mean CUDA-event duration, against the
            measured HBM copy bandwidth.
e2e       = the same metric through the public Python API with host buffers:
            every step copies x, z, dy, w from pinned host memory and y, rstd,
            dx, dz, dw back.
--impl reference times the fp64 CPU oracle (the repository's checker) on
every host core (one worker process per core, each on its own block of
rows), one bounded row sample per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rollout_parity_b200 import workloads  # noqa: E402

METRIC = "gated RMSNorm fwd+bwd HBM GB/s (% of B200 peak), rows/s; invariance pass"
WORKLOAD = "gated_262144x128_bf16_outliers"
FALLBACK_HBM_GBS = 6650.0
SETS = 4


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-invariance", action="store_true")
    ap.add_argument("--buffer-sets", type=int, default=SETS,
                    help="rotating input sets (fewer only for profiler captures)")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(workloads.ALL),
                    help="which synthetic workload one step runs (default: the headline)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every call from Python instead of replaying a CUDA graph")
    return ap.parse_args()


def bytes_model(rows, width, esize=2, gated=True):
    """Algorithmic bytes of one forward call and one backward call."""
    t = 3 if gated else 2            # forward: x, (z), y
    b = 5 if gated else 3            # backward: x, (z), dy, dx, (dz)
    fwd = rows * (t * width * esize + 4) + width * 4
    bwd = rows * (b * width * esize + 4) + 2 * width * 4
    return fwd, bwd


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def src_sha():
    """Digest of the kernel sources (csrc/*.cu, *.cuh) and the C header."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "rollout_parity_b200", "csrc")
    files = sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for f in [os.path.join(csrc, f) for f in files] + [os.path.join(ROOT, "include", "rn.h")]:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:12]


def op_name(wl):
    if wl.act == "none":
        return ("zero-centred RMSNorm fwd+bwd" if wl.weight_offset == 1.0 else
                f"RMSNorm (weight offset {wl.weight_offset:g}) fwd+bwd")
    if wl.act == "silu" and wl.weight_offset == 0.0:
        return "gated RMSNorm fwd+bwd"
    return f"gated RMSNorm ({wl.act} gate, weight offset {wl.weight_offset:g}) fwd+bwd"


def esize_of(wl):
    return 4 if wl.dtype == "f32" else 2


def profiled_traffic(workload):
    """DRAM bytes per backward call of this workload from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    want = src_sha()
    for ln in open(p):
        kv = dict(t.split("=", 1) for t in ln.split() if "=" in t)
        if (kv.get("workload") == workload and kv.get("unit") == "bwd_call"
                and kv.get("source_sha1") == want):
            return int(kv["dram_bytes_per_call"])
    return None


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons in the background."""

    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.t0 = self.t1 = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *self.sel, "--query-gpu=timestamp," + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for ln in out.strip().splitlines():
            f = [s.strip() for s in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                ts += float("0." + f[0].split(".")[1]) if "." in f[0] else 0.0
            except Exception:
                ts = None
            rows.append((ts, f))
        inside = [f for ts, f in rows if ts is not None and self.t0 - 0.05 <= ts <= self.t1 + 0.05]
        use = inside or [f for _, f in rows]
        sm = [float(f[1]) for f in use if f[1].replace(".", "").isdigit()]
        mx = [float(f[2]) for f in use if f[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for f in use for n, v in zip(names, f[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(inside), "samples_outside_window": len(rows) - len(inside)}


def graph_steps(k):
    """Steps per captured graph: a divisor of k (so exactly k steps run), at most
    256, preferring multiples of the buffer rotation (4)."""
    divs = [d for d in range(1, min(k, 256) + 1) if k % d == 0]
    rot = [d for d in divs if d % SETS == 0]
    return max(rot) if rot else max(divs)


def dist_setup(n):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if n > 1 or world > 1:
        import datetime
        import torch.distributed as dist
        rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", str(rank)))
        return rank, local, world, dist, datetime
    return 0, 0, 1, None, None


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(a):
    import rollout_parity_b200 as rn
    from rollout_parity_b200._lib import DType, check
    from rollout_parity_b200.ops import act_code

    rank, local, world, dist, dt_mod = dist_setup(a.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist is not None:
        dist.init_process_group("nccl", timeout=dt_mod.timedelta(seconds=120),
                                device_id=dev)
    lib = rn.load()

    nsets = max(1, a.buffer_sets)
    make = workloads.ALL[a.workload]
    host = [make(seed=1000 * rank + s) for s in range(nsets)]
    wl0 = host[0]
    R, H, eps = wl0.rows, wl0.width, wl0.eps
    gated = wl0.gated
    dtc = int({"bf16": DType.BF16, "f16": DType.F16, "f32": DType.F32}[wl0.dtype])
    actc, woff = int(act_code(wl0.act)), wl0.weight_offset
    esize = esize_of(wl0)
    fwd_b, bwd_b = bytes_model(R, H, esize=esize, gated=gated)
    step_b = fwd_b + bwd_b
    nws = lib.norm_bwd_workspace_bytes(R, H)
    sets = []
    for wl in host:
        d = wl.to(dev)
        sets.append(dict(x=d.x, z=d.z, w=d.w, dy=d.dy, y=torch.empty_like(d.x),
                         rstd=torch.empty(R, dtype=torch.float32, device=dev),
                         dx=torch.empty_like(d.x), dz=torch.empty_like(d.x) if gated else None,
                         dw=torch.empty(H, dtype=torch.float32, device=dev),
                         ws=torch.empty(nws, dtype=torch.uint8, device=dev)))
    P = [{k: (None if v is None else v.data_ptr()) for k, v in s.items()} for s in sets]
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def fwd(p, stp=sp):
        return lib.rmsnorm_fwd(R, H, eps, woff, actc, dtc, p["x"], p["z"], p["w"], p["y"],
                               p["rstd"], stp)

    exchange = None
    if world > 1:
        # data parallel: every rank returns its 256-row chunk partials of dw; they
        # are all-gathered in rank order and folded with the declared tree every
        # step, so the step's dw is that of the whole N-rank batch, bitwise
        from rollout_parity_b200 import parallel
        from rollout_parity_b200.ops import rn_fold_tree
        rows_per_rank = parallel.check_chunk_split(R, device=dev)
        nch = int(lib.rmsnorm_bwd_chunk_count(R))
        n_all = sum(-(-r // 256) for r in rows_per_rank)
        fold_ws = torch.empty(max(16, int(lib.rn_fold_tree_workspace_bytes(n_all, H))),
                              dtype=torch.uint8, device=dev)
        for s_, p_ in zip(sets, P):
            s_["chunks"] = torch.empty(nch, H, dtype=torch.float32, device=dev)
            p_["chunks"] = s_["chunks"].data_ptr()

        def exchange(s_):
            parallel.chunk_split_dw(
                s_["chunks"], R, rows_per_rank=rows_per_rank,
                fold=lambda g: rn_fold_tree(g, out=s_["dw"], ws=fold_ws))
        a.no_graph = True      # NCCL calls stay outside graph capture

    def bwd(p, stp=sp):
        if exchange is not None:
            return lib.rmsnorm_bwd_chunks(R, H, eps, woff, actc, dtc, p["x"], p["z"], p["w"],
                                          p["dy"], p["rstd"], None, p["dx"], p["dz"],
                                          p["chunks"], p["ws"], nws, stp)
        return lib.rmsnorm_bwd(R, H, eps, woff, actc, dtc, p["x"], p["z"], p["w"], p["dy"],
                               p["rstd"], None, p["dx"], p["dz"], p["dw"], p["ws"], nws, stp)

    for p in P:                       # every set gets its rstd before any backward
        check("rmsnorm_fwd", fwd(p))
    n_launch = None                   # our kernels per step, counted by the library
    for k in range(max(1, a.warmup)):
        check("rmsnorm_fwd", fwd(P[k % nsets]))
        nl = lib.rn_last_launches()
        check("rmsnorm_bwd", bwd(P[(k + 2) % nsets]))
        nl += lib.rn_last_launches()
        if exchange is not None:
            exchange(sets[(k + 2) % nsets])
            nl += lib.rn_last_launches()
        n_launch = nl
    torch.cuda.synchronize()

    K = a.steps
    G = K if a.no_graph else graph_steps(K)
    # per-call events for the roofline: G steps recorded in a separate graph (or,
    # without graphs, every step of the timed loop)
    ev = [[torch.cuda.Event(enable_timing=True, external=not a.no_graph) for _ in range(3)]
          for _ in range(G)]
    graph = graph_ev = graph_fwd_only = graph_bwd_only = None
    if not a.no_graph:
        # graph: G steps of calls only; it is what the timed region replays K / G times.
        # graph_ev: the same G steps with event records between the calls.
        cap = torch.cuda.Stream(dev)

        def capture(with_events):
            g = torch.cuda.CUDAGraph()
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap):
                csp = cap.cuda_stream
                for j in range(G):
                    if with_events:
                        ev[j][0].record(cap)
                    s1 = fwd(P[j % nsets], csp)
                    if with_events:
                        ev[j][1].record(cap)
                    s2 = bwd(P[(j + 2) % nsets], csp)
                    if with_events:
                        ev[j][2].record(cap)
                    if s1 or s2:
                        raise RuntimeError(f"capture failed: status {s1}, {s2}")
            stream.wait_stream(cap)
            return g

        graph = capture(False)
        graph_ev = capture(True)

        def capture_one(call, off):
            # G calls of one direction back to back, buffer sets rotating
            g = torch.cuda.CUDAGraph()
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap):
                for j in range(G):
                    st_ = call(P[(j + off) % nsets], cap.cuda_stream)
                    if st_:
                        raise RuntimeError(f"capture failed: status {st_}")
            stream.wait_stream(cap)
            return g

        graph_fwd_only = capture_one(fwd, 0)
        graph_bwd_only = capture_one(bwd, 2)
        for _ in range(max(1, a.warmup // G)):
            graph.replay()
        torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(dev)
    clocks.start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark("t0")
    t_start.record(stream)
    if graph is not None:
        for _ in range(K // G):
            graph.replay()
    else:
        for k in range(K):
            e = ev[k]
            e[0].record(stream)
            s1 = fwd(P[k % nsets])
            e[1].record(stream)
            s2 = bwd(P[(k + 2) % nsets])
            if exchange is not None:
                exchange(sets[(k + 2) % nsets])
            e[2].record(stream)
            if s1 or s2:
                check("rmsnorm_fwd", s1)
                check("rmsnorm_bwd", s2)
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.mark("t1")
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    if graph_ev is not None:   # per-call timings, right after the timed region
        for _ in range(2):
            graph_ev.replay()
        torch.cuda.synchronize()
    fwd_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(G)]
    bwd_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(G)]
    # each direction alone, G calls back to back (launches overlap as in the
    # step): mean time per call without an event between calls
    streamed = {}
    for name, g in (("fwd", graph_fwd_only), ("bwd", graph_bwd_only)):
        if g is None:
            continue
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        streamed[name] = e0.elapsed_time(e1) / G
    if dist is not None:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_step = ms / K
    value = world * step_b * K / (ms / 1e3) / 1e9
    # our kernels per step: the forward, the backward and its fold passes, and
    # with N ranks the rn_fold_tree passes of the dw exchange
    launches = K * n_launch

    inv = invariance_checks(rn, sets[0], R, H, eps, wl0) \
        if rank == 0 and not a.no_invariance else None
    e2e = run_e2e(rn, host[0], dev, a.e2e_steps, step_b, world, dist) if a.e2e_steps > 0 \
        else None
    cpu = acc = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(host[0], fwd_b, bwd_b)
        # the oracle as the checker of set 0's outputs (its inputs are host[0])
        acc = accuracy(host[0], sets[0])

    if rank == 0:
        peak, src = peaks()
        bwd_mean = float(np.mean(bwd_ms))
        fwd_mean = float(np.mean(fwd_ms))
        achieved = bwd_b / (bwd_mean / 1e3) / 1e9
        # the roofline's time per call: G calls back to back (as the timed
        # region runs them: no event between calls), else the per-call events
        if "bwd" in streamed:
            rl_gbs = bwd_b / (streamed["bwd"] / 1e3) / 1e9
            rl_timing = (f"{G} calls back to back in one graph, buffer sets rotating, one "
                         "event pair around them")
        else:
            rl_gbs, rl_timing = achieved, "CUDA events around each call in the timed loop"
        traffic = profiled_traffic(a.workload)
        desc = {WORKLOAD: {"layout": "8192 tokens x 32 heads, row = token*32 + head",
                           "outliers": "1% of channels x50 in x, z, dy"}}.get(a.workload, {})
        opname = op_name(wl0)
        iod = wl0.dtype
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": K, "warmup": a.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": iod,
            "data": "synthetic (seeded; no dataset or checkpoint)",
            "config": {"workload": a.workload, "op": opname, "rows": R, "width": H, **desc,
                       "activation": wl0.act, "weight_offset": woff,
                       "eps": eps, "io_dtype": (f"{iod} x/z/dy/y/dx/dz" if gated else
                                                f"{iod} x/dy/y/dx") + ", fp32 w/rstd/dw",
                       "accumulate": "fp32",
                       "bytes_per_step": step_b,
                       "parallelism": (f"data parallel x{world}: rows split across ranks, dw "
                                       "chunk partials all-gathered and folded each step"
                                       if world > 1 else "one GPU"),
                       "launch": ("python loop" if a.no_graph else
                                  f"CUDA graph of {G} steps replayed {K // G} times"),
                       "per_call_timing": ("events in the timed loop" if a.no_graph else
                                           f"events in a copy of the graph replayed after "
                                           f"the timed region ({G} steps)"),
                       "l2": (f"{nsets} rotating buffer sets (fwd on k%{nsets}, bwd on "
                              f"(k+2)%{nsets}): every buffer is re-touched only after >= 512 MB "
                              "of other traffic (L2 is 126 MB); no flush kernel")
                       if nsets == SETS else f"{nsets} buffer set(s): profiling layout"},
            "rows_per_s": round(world * R * K / (ms / 1e3), 1),
            "pct_of_peak": round(100.0 * value / world / peak, 2),
            "fwd_us": round(1e3 * fwd_mean, 2), "bwd_us": round(1e3 * bwd_mean, 2),
            "fwd_gbs": round(fwd_b / (fwd_mean / 1e3) / 1e9, 1),
            "bwd_gbs": round(achieved, 1),
            "back_to_back": ({"fwd_us": round(1e3 * streamed["fwd"], 2),
                              "bwd_us": round(1e3 * streamed["bwd"], 2),
                              "fwd_gbs": round(fwd_b / streamed["fwd"] / 1e6, 1),
                              "bwd_gbs": round(bwd_b / streamed["bwd"] / 1e6, 1),
                              "timing": f"{G} calls of one direction in one graph, buffer sets "
                                        "rotating, one event pair around the replay"}
                             if streamed else None),
            "invariance": inv,
            "roofline": {"bound": "hbm",
                         "kernel": "rmsnorm_bwd call (backward kernel + dw fold pass)",
                         "timing": rl_timing,
                         "achieved": round(rl_gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(rl_gbs / peak, 4), "peak_source": src,
                         "per_call": {"achieved": round(achieved, 1),
                                      "frac": round(achieved / peak, 4),
                                      "timing": "CUDA events around each call (bwd_us)"},
                         "traffic": traffic, "algorithmic_bytes": bwd_b},
            "cpu_baseline": cpu, "accuracy": acc, "e2e": e2e, "gpu_launches": launches,
            "clocks": clk,
            "source_sha1": src_sha(),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def invariance_checks(rn, s, R, H, eps, wl):
    """Bitwise: rows inside the full batch vs the same rows as their own batch,
    and dw across repeats and launch geometries."""
    gated = wl.gated

    def fb(x, z, dy):
        y, r = rn.rmsnorm_fwd(x, s["w"], eps, wl.weight_offset, z, wl.act)
        dx, dz, dw = rn.rmsnorm_bwd(x, s["w"], dy, r, eps, wl.weight_offset, z, wl.act)
        return ([y, r, dx, dz] if gated else [y, r, dx]), dw

    bits = lambda t: t.view(torch.int32 if t.dtype == torch.float32 else torch.int16)
    cl = lambda t, sl: None if t is None else t[sl].clone()
    full, dw = fb(s["x"], s["z"], s["dy"])
    checks, bad = 0, 0
    for st, n in ((R // 3, 1), (R // 5, 7), (R // 2 - 5, min(4099, R // 2)), (R - 33, 33)):
        if st < 0 or st + n > R:
            continue
        sl = slice(st, st + n)
        part, _ = fb(cl(s["x"], sl), cl(s["z"], sl), cl(s["dy"], sl))
        for a_, b_ in zip([t[sl] for t in full], part):
            checks += 1
            bad += int(not torch.equal(bits(a_), bits(b_)))
    for geo in ((0, 0, 0), (148, 1, 8), (7, 2, 64), (0, 0, 0)):
        rn.rn_test_set_geometry(*geo)
        _, dw2 = fb(s["x"], s["z"], s["dy"])
        checks += 1
        bad += int(not torch.equal(bits(dw), bits(dw2)))
    rn.rn_test_set_geometry(0, 0, 0)
    torch.cuda.synchronize()
    return {"result": "pass" if bad == 0 else "fail", "bitwise_checks": checks, "failed": bad}


def run_e2e(rn, wl, dev, steps, step_b, world, dist):
    """Steps through the public API with every step's inputs copied in from
    pinned host memory and its results copied out, inside the timed region.
    On one GPU two device buffer sets alternate, so step k's inputs go in (on
    one stream) while step k-1's results come out (on another): the host link
    carries both directions at once.  With N ranks each step runs in order."""
    R, H, eps = wl.rows, wl.width, wl.eps
    gated = wl.gated
    pin = lambda t: t.pin_memory()
    hx, hdy, hw = pin(wl.x), pin(wl.dy), pin(wl.w)
    hz = pin(wl.z) if gated else None
    oy, ors = torch.empty_like(hx).pin_memory(), torch.empty(R, dtype=torch.float32).pin_memory()
    odx, odz = torch.empty_like(hx).pin_memory(), torch.empty_like(hx).pin_memory()
    odw = torch.empty(H, dtype=torch.float32).pin_memory()
    nbuf = 2 if dist is None else 1

    def dev_set():
        d = {"x": torch.empty_like(hx, device=dev), "dy": torch.empty_like(hx, device=dev),
             "w": torch.empty_like(hw, device=dev), "rstd": torch.empty(R, dtype=torch.float32,
                                                                        device=dev),
             "dw": torch.empty(H, dtype=torch.float32, device=dev),
             "z": torch.empty_like(hx, device=dev) if gated else None,
             "ws": rn.workspace(R, H, dev)}
        d["y"], d["dx"] = torch.empty_like(d["x"]), torch.empty_like(d["x"])
        d["dz"] = torch.empty_like(d["x"]) if gated else None
        return d

    bufs = [dev_set() for _ in range(nbuf)]
    h2d = sum(t.numel() * t.element_size() for t in (hx, hz, hdy, hw) if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in ((oy, ors, odx, odz, odw) if gated else
                                                     (oy, ors, odx, odw)))
    if dist is not None:
        from rollout_parity_b200.parallel import check_chunk_split, chunk_split_dw
        rows_per_rank = check_chunk_split(R, device=dev)
    main = torch.cuda.current_stream(dev)
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3)) if dist is None else \
        (main, main, main)
    ev = lambda: torch.cuda.Event()
    computed = [ev() for _ in range(nbuf)]       # the set's compute is done (inputs free)
    outputs_free = [ev() for _ in range(nbuf)]   # the copy-out that read the set is done
    copied_in = [ev() for _ in range(nbuf)]
    for e_ in computed + outputs_free:
        e_.record(main)

    def step(k):
        b = k % nbuf
        d = bufs[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(computed[b])
            d["x"].copy_(hx, non_blocking=True)
            if gated:
                d["z"].copy_(hz, non_blocking=True)
            d["dy"].copy_(hdy, non_blocking=True)
            d["w"].copy_(hw, non_blocking=True)
            copied_in[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(copied_in[b])
            s_cmp.wait_event(outputs_free[b])
            zz = d["z"]
            rn.rmsnorm_fwd(d["x"], d["w"], eps, wl.weight_offset, zz, wl.act, y=d["y"],
                           rstd=d["rstd"])
            if dist is None:
                rn.rmsnorm_bwd(d["x"], d["w"], d["dy"], d["rstd"], eps, wl.weight_offset, zz,
                               wl.act, dx=d["dx"], dz=d["dz"], dw=d["dw"], ws=d["ws"])
                dw_out = d["dw"]
            else:   # with N ranks the step's dw is the whole batch's (chunk partials folded)
                _, _, ch = rn.rmsnorm_bwd_chunks(d["x"], d["w"], d["dy"], d["rstd"], eps,
                                                 wl.weight_offset, zz, wl.act, dx=d["dx"],
                                                 dz=d["dz"], ws=d["ws"])
                dw_out = chunk_split_dw(ch, R, rows_per_rank=rows_per_rank)
            computed[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            odw.copy_(dw_out, non_blocking=True)
            oy.copy_(d["y"], non_blocking=True)
            ors.copy_(d["rstd"], non_blocking=True)
            odx.copy_(d["dx"], non_blocking=True)
            if gated:
                odz.copy_(d["dz"], non_blocking=True)
            outputs_free[b].record(s_out)

    def join():
        for s_ in (s_in, s_cmp, s_out):
            main.wait_stream(s_)

    for k in range(3):
        step(k)
    join()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
        torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(main)
    for s_ in (s_in, s_cmp, s_out):
        s_.wait_stream(main)
    for k in range(steps):
        step(k)
    join()
    e.record(main)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e)
    if dist is not None:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return {"value": round(world * step_b * steps / (ms / 1e3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4),
            "overlap": ("inputs of step k copied in while step k-1's results are copied out "
                        "(two device buffer sets, three streams)" if dist is None else
                        "none: copy in, compute, copy out in order"),
            "api": "rollout_parity_b200.rmsnorm_fwd/rmsnorm_bwd" if dist is None else
                   "rollout_parity_b200.rmsnorm_fwd/rmsnorm_bwd_chunks + parallel.chunk_split_dw"}


# ---------------------------------------------------------------------------
# the fp64 oracle on the host cores
# ---------------------------------------------------------------------------
def _oracle_step(orc, wl, x, z, w, dy):
    orc.rmsnorm_fwd(x, w, wl.eps, wl.weight_offset, z, wl.act)
    orc.rmsnorm_bwd(x, w, dy, wl.eps, wl.weight_offset, z, wl.act)


def host_info():
    """The host's usable cores and CPU model (recorded beside every CPU figure)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": cores, "cpu_model": model}


# Worker side of OraclePool.  A worker is a fresh interpreter (the pool is
# started with "spawn": nothing of the parent's CUDA state is inherited, and
# spawn is safe after the parent has used the GPU, where fork is not).
_POOL = {}


def _pool_init(names, shapes, eps, weight_offset, act):
    from multiprocessing import shared_memory
    import oracle
    _POOL["orc"] = oracle
    _POOL["shm"] = [shared_memory.SharedMemory(name=n) for n in names]
    _POOL["arr"] = [np.ndarray(sh, dtype=np.float64, buffer=m.buf)
                    for m, sh in zip(_POOL["shm"], shapes)]
    _POOL["p"] = (eps, weight_offset, act)


def _pool_rows(block):
    a, b = block
    x, dy, w = _POOL["arr"][0], _POOL["arr"][1], _POOL["arr"][2]
    z = _POOL["arr"][3] if len(_POOL["arr"]) > 3 else None
    eps, off, act = _POOL["p"]
    orc = _POOL["orc"]
    zz = None if z is None else z[a:b]
    orc.rmsnorm_fwd(x[a:b], w, eps, off, zz, act)
    _, _, dw = orc.rmsnorm_bwd(x[a:b], w, dy[a:b], eps, off, zz, act)
    return dw


class OraclePool:
    """The fp64 oracle over rows [0, n) of a workload on every host core: one
    worker process per core, each running the unmodified oracle on its own
    contiguous block of rows, read from shared memory.  pass_() runs one
    forward + backward over all n rows."""

    def __init__(self, wl, n, procs=None):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        f = workloads.as_f64
        arrays = [f(wl.x[:n]), f(wl.dy[:n]), f(wl.w)]
        if wl.z is not None:
            arrays.append(f(wl.z[:n]))
        self.shm = []
        for a in arrays:
            m = shared_memory.SharedMemory(create=True, size=max(8, a.nbytes))
            np.ndarray(a.shape, dtype=np.float64, buffer=m.buf)[...] = a
            self.shm.append(m)
        self.procs = procs or host_info()["nproc"]
        step = -(-n // self.procs)
        self.blocks = [(i, min(n, i + step)) for i in range(0, n, step)]
        self.pool = mp.get_context("spawn").Pool(
            self.procs, initializer=_pool_init,
            initargs=([m.name for m in self.shm], [a.shape for a in arrays], wl.eps,
                      wl.weight_offset, wl.act))
        self.pass_()                      # workers started and warm

    def pass_(self):
        return self.pool.map(_pool_rows, self.blocks, chunksize=1)

    def close(self):
        self.pool.close()
        self.pool.join()
        for m in self.shm:
            m.close()
            m.unlink()


def _time_passes(fn, min_s, max_s):
    reps, t0 = 0, time.perf_counter()
    while True:
        fn()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_s or el * (reps + 1) / reps > max_s:
            return reps, el


def accuracy(wl, out, max_elems=1 << 26):
    """Parity statistics of one step's outputs against the fp64 oracle, over
    the workload's rows (its first rows when it has more than ``max_elems``
    elements): for 16-bit outputs the fraction of y elements correctly rounded
    (equal to the oracle's value rounded once), the fraction within the plain
    2-ulp bound, the elements that pass only through the cancellation floor
    (dx, dz: 2^-16 times the oracle's cancellation scale), those out of
    tolerance and the largest error in ulps; relative L2 for fp32 tensors.
    ``out`` holds the device outputs for ``wl``'s inputs."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import numerics
    import oracle
    f = workloads.as_f64
    R, H = wl.rows, wl.width
    n = R if R * H <= max_elems else max(32, max_elems // H)
    fmt = {"bf16": numerics.BF16, "f16": numerics.F16}.get(wl.dtype)
    off, act, eps = wl.weight_offset, wl.act, wl.eps
    names = ["y", "dx"] + (["dz"] if wl.gated else [])
    cnt = {k: {} for k in names}
    l2 = {k: [0.0, 0.0] for k in names + ["rstd"]}
    dw_ref = np.zeros(H)
    w = f(wl.w)
    step = max(1, (1 << 21) // H)
    for a in range(0, n, step):
        b = min(n, a + step)
        x, dy = f(wl.x[a:b]), f(wl.dy[a:b])
        z = None if wl.z is None else f(wl.z[a:b])
        ref = {}
        ref["y"], rho = oracle.rmsnorm_fwd(x, w, eps, off, z, act)
        ref["dx"], ref["dz"], dw = oracle.rmsnorm_bwd(x, w, dy, eps, off, z, act)
        dw_ref += dw
        scale = {"y": None, "dx": oracle.rmsnorm_dx_scale(x, w, dy, eps, off, z, act)}
        if wl.gated:
            scale["dz"] = oracle.rmsnorm_dz_scale(x, w, dy, eps, off, z, act)
        for k in names:
            g = f(out[k][a:b])
            if fmt is not None:
                c = numerics.counts_16(g, ref[k], fmt, scale[k])
                for key, v in c.items():
                    cnt[k][key] = max(cnt[k].get(key, 0.0), v) if key == "max_err_ulps" \
                        else cnt[k].get(key, 0) + v
            l2[k][0] += float(np.sum((g - ref[k]) ** 2))
            l2[k][1] += float(np.sum(ref[k] ** 2))
        gr = f(out["rstd"][a:b])
        l2["rstd"][0] += float(np.sum((gr - rho) ** 2))
        l2["rstd"][1] += float(np.sum(rho ** 2))
    rel = lambda k: round(float(np.sqrt(l2[k][0] / l2[k][1])), 9) if l2[k][1] > 0 else 0.0
    res = {"rows_checked": n, "of_rows": R,
           "tolerance": ("16-bit: |gpu - oracle| <= 2 ulp (+ 2^-16 x cancellation scale "
                         "for dx, dz); fp32: relative L2 <= 1e-4")}
    for k in names:
        e = {"rel_l2": rel(k)}
        if fmt is not None:
            c, m = cnt[k], max(1, cnt[k]["n"])
            e.update({"correctly_rounded_pct": round(100.0 * c["correctly_rounded"] / m, 5),
                      "plain_2ulp_pct": round(100.0 * c["plain_pass"] / m, 5),
                      "floor_hits": c["floor_hits"], "out_of_tolerance": c["out_of_tolerance"],
                      "max_err_ulps": round(c["max_err_ulps"], 3), "elements": c["n"]})
        res[k] = e
    res["rstd"] = {"rel_l2": rel("rstd")}
    if n == R:
        g = f(out["dw"])
        den = float(np.linalg.norm(dw_ref))
        res["dw"] = {"rel_l2": round(float(np.linalg.norm(g - dw_ref)) / den, 9) if den else 0.0}
    return res


def cpu_baseline(wl, fwd_b, bwd_b, min_s=10.0, max_s=30.0):
    """The fp64 oracle, as it stands, over (a bounded sample of) the workload's
    rows: on every host core (the reported figure) and on one thread."""
    import oracle
    f = workloads.as_f64
    n = wl.rows
    if wl.rows * wl.width > (1 << 26):        # bound host memory and time: a row sample
        n = max(32, (1 << 26) // wl.width)
        fwd_b, bwd_b = bytes_model(n, wl.width, esize_of(wl), wl.gated)
    x, dy, w = f(wl.x[:n]), f(wl.dy[:n]), f(wl.w)
    z = None if wl.z is None else f(wl.z[:n])
    reps1, el1 = _time_passes(lambda: _oracle_step(oracle, wl, x, z, w, dy), min_s, max_s)
    one = round((fwd_b + bwd_b) * reps1 / el1 / 1e9, 4)
    host = host_info()
    pool = OraclePool(wl, n)
    try:
        reps, el = _time_passes(pool.pass_, min_s, max_s)
    finally:
        pool.close()
    return {"value": round((fwd_b + bwd_b) * reps / el / 1e9, 4), "unit": "GB/s",
            "cores": pool.procs, "kind": "oracle",
            "sample": f"fp64 numpy oracle fwd+bwd over rows [0, {n}) of the {wl.rows}-row "
                      f"workload, split in {len(pool.blocks)} row blocks over {pool.procs} "
                      f"worker processes (one per core), {reps} passes in {el:.1f} s",
            "single_thread": {"value": one, "unit": "GB/s", "cores": 1,
                              "sample": f"same rows, one thread, {reps1} passes in {el1:.1f} s"},
            "host": host}


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(max(1, a.gpus))))
    if rank != 0:
        return
    import oracle
    wl = workloads.ALL[a.workload]()
    R, H = wl.rows, wl.width
    f = workloads.as_f64
    fz = (lambda t: None) if not wl.gated else f
    host = host_info()
    # size the per-step row sample so the whole run stays near a minute on the
    # host's cores (a single-thread probe, scaled by the core count)
    probe = min(R, max(32, 4096 * 128 // H))
    t0 = time.perf_counter()
    _oracle_step(oracle, wl, f(wl.x[:probe]), fz(wl.z[:probe] if wl.gated else None), f(wl.w),
                 f(wl.dy[:probe]))
    per_row = (time.perf_counter() - t0) / probe / host["nproc"]
    n = int(60.0 / per_row / max(1, a.steps + a.warmup))
    n = max(32, min(R, (1 << 26) // H, n // 32 * 32))
    pool = OraclePool(wl, n)
    try:
        for _ in range(a.warmup):
            pool.pass_()
        t0 = time.perf_counter()
        for _ in range(a.steps):
            pool.pass_()
        el = time.perf_counter() - t0
    finally:
        pool.close()
    fwd_b, bwd_b = bytes_model(n, H, esize_of(wl), wl.gated)
    value = (fwd_b + bwd_b) * a.steps / el / 1e9
    sample = (f"fp64 numpy oracle fwd+bwd on rows [0, {n}) of the {R}-row workload per step, "
              f"split in {len(pool.blocks)} row blocks over {pool.procs} worker processes "
              f"(one per core)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(1e3 * el / a.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no dataset or checkpoint)",
        "config": {"workload": a.workload,
                   "op": op_name(wl),
                   "rows": R, "width": H, "sample_rows_per_step": n},
        "rows_per_s": round(n * a.steps / el, 1),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": pool.procs,
                         "kind": "oracle", "sample": sample, "host": host},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
