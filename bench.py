#!/usr/bin/env python
"""Benchmark of the GSPN line scan (libgspn) on B200.

One step = one pass of the whole hot path over one batch: the forward
(gate normalisation, four-direction line scan, summed merge) followed by the
backward (reverse adjoint scans, dx / dlambda / dlogits), through the C ABI.
Default workload: compact (channel-shared taps) 4-direction global scan, bf16
storage, fp32 arithmetic, B=32, C=1152, H=W=64 -- the 1K foundation shape.

Metric: achieved HBM GB/s = compulsory bytes / time, where the compulsory
bytes are every input read once and every output written once
(forward: x, lambda, logits, out; backward: x, lambda, logits, dout, dx,
dlambda, dlogits).  Also reported: % of the measured HBM copy peak and
Gpixel*channel/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libgspn|reference]

For N > 1 it runs under torch.distributed.run, one rank per GPU; each rank
processes its own batch (weak scaling, no collective on the data path) and
rank 0 prints one JSON line with the max-over-ranks time.
--impl reference times the CPU oracle (plain double-precision C) on the host
cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "GSPN scan achieved HBM GB/s (% of B200 peak) and Gpixel·ch/s, fwd and fwd+bwd"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libgspn", choices=["libgspn", "reference"])
    ap.add_argument("--workload", default=synth.HEADLINE,
                    choices=list(synth.WORKLOADS) + list(synth.EXTRA_WORKLOADS) + list(synth.BLOCK_WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target length of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="passes", default="both", choices=["both", "fwd", "bwd"],
                    help="profiling aid: time only one pass (the JSON line then covers that pass)")
    ap.add_argument("--batch", type=int, default=0, help="profiling aid: override B (0 = the workload's)")
    ap.add_argument("--channels", type=int, default=0, help="profiling aid: override C (0 = the workload's)")
    ap.add_argument("--graph", action="store_true",
                    help="replay each pass from a CUDA graph captured once (no per-call host work in the timed loop)")
    return ap.parse_args()


def pass_bytes(w: synth.Workload):
    """Compulsory bytes of one forward and one backward pass."""
    e = w.elt_bytes
    n = w.B * w.C * w.H * w.W
    lam = w.D * n
    lg = w.D * w.B * w.Cw * 3 * w.H * w.W
    fwd = e * (n + lam + lg + n)
    bwd = e * (n + lam + lg + n + n + lam + lg)
    return fwd, bwd


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# sources of the kernel each pass's traffic figure was taken on
KERNEL_SOURCES = {
    "fwd": ("gspn_compact64.cu", "gspn_tma.cuh", "gspn_lane.cuh", "gspn_tmem.cuh", "gspn_common.cuh", "gspn_internal.h"),
    "bwd": ("gspn_compact64_bwd.cu", "gspn_tma.cuh", "gspn_lane.cuh", "gspn_tmem.cuh", "gspn_common.cuh", "gspn_internal.h"),
}


def csrc_hash(kernel_pass: str) -> str:
    h = hashlib.sha256()
    d = os.path.join(ROOT, "linear_spatial_propagation_b200", "csrc")
    for f in KERNEL_SOURCES[kernel_pass]:
        h.update(f.encode())
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_pass: str, w: synth.Workload):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summary, if it was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None
    ent = d.get(w.name, {}).get(kernel_pass)
    if not ent or ent.get("csrc_hash") != csrc_hash(kernel_pass):
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9:
                    rows.append(f)
        except Exception:
            return None
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        load = [s for s in sm if mx and s > 0.3 * max(mx)] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------
# CPU oracle (baseline / reference arm)
# ------------------------------------------------------------------------------
def oracle_sample(w: synth.Workload, target_s: float, nthreads: int):
    """Time the oracle's forward + backward on a sample of w's planes: as many
    channels of one batch image as fit in about target_s seconds, then, when
    all of an image's channels fit, as many whole images (each its own seeded
    B=1 problem, drawn before its timing starts) as fit."""
    import oracle

    def draw(cs, i):
        sw = w.replace(B=1, C=cs, seed=w.seed + 7 + i)
        return sw, synth.make_inputs(sw, with_dout=True)

    def timed(sw, inp):
        t0 = time.perf_counter()
        oracle.fwd_workload(sw, inp, nthreads=nthreads)
        oracle.bwd_workload(sw, inp, nthreads=nthreads)
        return time.perf_counter() - t0

    probe_c = min(w.C, max(1, nthreads))
    sw, inp = draw(probe_c, 0)
    t = timed(sw, inp)
    cs = int(min(w.C, max(1, probe_c * target_s / max(t, 1e-6))))
    if cs > probe_c:
        sw, inp = draw(cs, 0)
        t = timed(sw, inp)
    images = [(sw, inp)]
    if cs == w.C and w.B > 1:
        n_img = int(min(w.B, max(1, target_s / max(t, 1e-6))))
        for i in range(1, n_img):
            sw_i, inp_i = draw(cs, i)
            t += timed(sw_i, inp_i)
            images.append((sw_i, inp_i))
    f, b = pass_bytes(sw)
    n = len(images)
    return {"seconds": t, "bytes": (f + b) * n, "pixch": n * sw.C * sw.H * sw.W, "channels": sw.C,
            "images": n, "sw": sw, "inputs": images}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    nthreads = os.cpu_count() or 1
    steps, warm = max(1, args.steps), max(0, args.warmup)
    per_step = max(0.5, min(args.cpu_seconds, 150.0 / (steps + warm)))
    cal = oracle_sample(w, per_step, nthreads)
    import oracle
    images = cal["inputs"]

    def step():
        for sw, inp in images:
            oracle.fwd_workload(sw, inp, nthreads=nthreads)
            oracle.bwd_workload(sw, inp, nthreads=nthreads)

    for _ in range(warm):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = (time.perf_counter() - t0) / steps
    val = cal["bytes"] / dt / 1e9
    sample = (f"{cal['images']} batch image(s) x C={cal['channels']} of {w.name} (fwd+bwd, B=1 each), "
              f"{nthreads} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": warm, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
        "config": config_of(w, args.gpus),
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": nthreads, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_block_reference(args, w):
    """The block oracle as the reference arm, on whole batch images."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    nthreads = os.cpu_count() or 1
    steps, warm = max(1, args.steps), max(0, args.warmup)
    per_step = max(0.5, min(args.cpu_seconds, 150.0 / (steps + warm)))
    for _ in range(warm):
        block_oracle_sample(w, per_step, nthreads)
    tot_b, tot_s, imgs = 0, 0.0, 0
    for _ in range(steps):
        smp = block_oracle_sample(w, per_step, nthreads)
        tot_b += smp["bytes"]
        tot_s += smp["seconds"]
        imgs = smp["images"]
    val = tot_b / tot_s / 1e9
    line = {
        "impl": "reference", "metric": BLOCK_METRIC, "value": val, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": warm, "ms_per_step": tot_s / steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
        "config": block_config(w, args.gpus),
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{imgs} batch image(s) of {w.name} per step, B=1 each"},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(dist, v: float, device) -> float:
    """The maximum of v over the ranks of the process group (v itself when
    there is none); every rank calls it at the same point."""
    if dist is None:
        return v
    import torch

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_rank: int, n_ranks: int, ms: float) -> float:
    """Whole-job GB/s: the bytes every rank moved over the slowest rank's time."""
    return bytes_per_rank * n_ranks / (ms * 1e-3) / 1e9


L2_BYTES = 126 * 2**20  # B200 L2


def config_of(w, n, passes="both", graph=False, flushed=False):
    return {"workload": w.name, "B": w.B, "C": w.C, "H": w.H, "W": w.W,
            "directions": "+".join(n_ for b, n_ in ((1, "T2B"), (2, "B2T"), (4, "L2R"), (8, "R2L")) if w.dir_mask & b),
            "groups": w.groups, "shared_taps": w.shared, "io_dtype": w.dtype,
            "pass": {"both": "fwd+bwd", "fwd": "fwd", "bwd": "bwd"}[passes],
            "launch": "cuda_graph" if graph else "direct",
            "l2": "flushed before every timed pass (a pass's bytes fit in L2)" if flushed
            else "inputs larger than L2 (no flush needed)",
            "parallelism": f"replicas x{n}" if n > 1 else "1 GPU"}


# ------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------
def run_gpu(args, w):
    import torch

    import linear_spatial_propagation_b200 as lsp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    lsp.load(build_if_missing=False)

    wr = w.replace(seed=w.seed + 1000 * rank)
    inp = synth.make_inputs(wr, with_dout=True)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def pinned(a):
        t = torch.from_numpy(a)
        if w.dtype == "bf16":
            t = t.view(torch.bfloat16)
        return t.pin_memory()

    h = {k: pinned(v) for k, v in inp.items()}
    del inp
    d = {k: v.to(dev) for k, v in h.items()}
    out = torch.empty_like(d["x"])
    grads = (torch.empty_like(d["x"]), torch.empty_like(d["logits"]), torch.empty_like(d["lam"]))
    desc = lsp.make_desc(w.B, w.C, w.H, w.W, w.dir_mask, w.groups, w.shared, w.dtype)
    wsf = lsp.workspace(desc, 0, dev)
    wsb = lsp.workspace(desc, 1, dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def fwd(din=d, o=None, strm=None):
        o = out if o is None else o
        st = lsp.gspn_fwd(desc, din["x"].data_ptr(), din["logits"].data_ptr(), din["lam"].data_ptr(), o.data_ptr(),
                          wsf.data_ptr() if wsf is not None else 0, wsf.numel() if wsf is not None else 0,
                          sp if strm is None else strm)
        if st:
            raise lsp.GspnError(st, "gspn_fwd")

    def bwd(din=d, g=None, strm=None):
        g = grads if g is None else g
        st = lsp.gspn_bwd(desc, din["x"].data_ptr(), din["logits"].data_ptr(), din["lam"].data_ptr(),
                          din["dout"].data_ptr(), g[0].data_ptr(), g[1].data_ptr(), g[2].data_ptr(),
                          wsb.data_ptr() if wsb is not None else 0, wsb.numel() if wsb is not None else 0,
                          sp if strm is None else strm)
        if st:
            raise lsp.GspnError(st, "gspn_bwd")

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def rank_max(v):
        return max_over_ranks(dist, v, dev)

    do_f = args.passes in ("both", "fwd")
    do_b = args.passes in ("both", "bwd")
    for _ in range(max(3, args.warmup)):
        if do_f:
            fwd()
        if do_b:
            bwd()
    barrier()
    # --graph: each pass is captured once into a CUDA graph (the library's calls
    # only enqueue work on the given stream) and the timed loop replays them
    fwd_t, bwd_t = fwd, bwd
    graphs = []
    if args.graph:
        gs = torch.cuda.Stream(dev)
        gs.wait_stream(stream)
        with torch.cuda.stream(gs):
            for fn in (fwd, bwd):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=gs):
                    fn(strm=gs.cuda_stream)
                graphs.append(g)
        stream.wait_stream(gs)
        fwd_t, bwd_t = graphs[0].replay, graphs[1].replay
        for _ in range(max(3, args.warmup)):
            if do_f:
                fwd_t()
            if do_b:
                bwd_t()
        barrier()
    # A pass whose compulsory bytes fit in L2 (126 MB) could find its
    # inputs there from the step before: then every timed pass starts after a
    # write of a buffer twice the size of L2, outside the pass's own events,
    # and the step time is the sum of the passes.
    fb0, bb0 = pass_bytes(w)
    flush = (do_f and fb0 < L2_BYTES) or (do_b and bb0 < L2_BYTES)
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e_start.record(stream)
    for k in range(K):
        if flush:
            flush_buf.zero_()
        ev[k][0].record(stream)
        if do_f:
            fwd_t()
        ev[k][1].record(stream)
        if flush:
            flush_buf.zero_()
        ev[k][2].record(stream)
        if do_b:
            bwd_t()
        ev[k][3].record(stream)
    e_end.record(stream)
    barrier()
    clk = clocks.stop()
    total_ms = rank_max(e_start.elapsed_time(e_end))
    fwd_ms = rank_max(sum(e[0].elapsed_time(e[1]) for e in ev) / K)
    bwd_ms = rank_max(sum(e[2].elapsed_time(e[3]) for e in ev) / K)
    ms = fwd_ms + bwd_ms if flush else total_ms / K

    # end to end: pinned host inputs -> device -> fwd + bwd -> results back to pinned
    # host, every step.  The copies run on their own streams so that step k+1's
    # inputs go up and step k-1's results come down while step k computes (two
    # device buffer sets; events order each buffer's reuse).
    E = args.e2e_steps
    hout = torch.empty(out.shape, dtype=tdt).pin_memory()
    hgrads = [torch.empty(g.shape, dtype=tdt).pin_memory() for g in grads]
    h2d = sum(t.numel() * t.element_size() for t in h.values())
    d2h = out.numel() * out.element_size() + sum(g.numel() * g.element_size() for g in grads)
    e2e_ms = None
    if E > 0:
        dins = [d, {k: torch.empty_like(v) for k, v in d.items()}]
        outs = [out, torch.empty_like(out)]
        gset = [grads, tuple(torch.empty_like(g) for g in grads)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        in_ready, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        used = [False, False]
        barrier()
        e2 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e2[0].record(s_in)
        for k in range(E):
            j = k % 2
            if used[j]:
                s_in.wait_event(comp_done[j])    # step k-2 has finished reading this input set
                stream.wait_event(out_done[j])   # and its results have left this output set
            for name in ("x", "lam", "logits", "dout"):
                with torch.cuda.stream(s_in):
                    dins[j][name].copy_(h[name], non_blocking=True)
            in_ready[j].record(s_in)
            stream.wait_event(in_ready[j])
            if do_f:
                fwd(dins[j], outs[j])
            if do_b:
                bwd(dins[j], gset[j])
            comp_done[j].record(stream)
            s_out.wait_event(comp_done[j])
            with torch.cuda.stream(s_out):
                hout.copy_(outs[j], non_blocking=True)
                for hg, g in zip(hgrads, gset[j]):
                    hg.copy_(g, non_blocking=True)
            out_done[j].record(s_out)
            used[j] = True
        e2[1].record(s_out)
        barrier()
        e2e_ms = rank_max(e2[0].elapsed_time(e2[1]) / E)

    fb, bb = pass_bytes(w)
    if not do_f:
        fb = 0
    if not do_b:
        bb = 0
    peak, peak_src = measured_peaks()
    n_gpu = world
    value = job_gbs(fb + bb, n_gpu, ms)
    pixch = w.B * w.C * w.H * w.W
    fwd_gbs = fb / (fwd_ms * 1e-3) / 1e9 if fb else 0.0
    bwd_gbs = bb / (bwd_ms * 1e-3) / 1e9 if bb else 0.0
    dom = "bwd" if bwd_ms >= fwd_ms else "fwd"
    dom_gbs = bwd_gbs if dom == "bwd" else fwd_gbs
    launches = K * (lsp.gspn_launches_per_call(desc, 0) * do_f + lsp.gspn_launches_per_call(desc, 1) * do_b)

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            try:
                s = oracle_sample(w, args.cpu_seconds, os.cpu_count() or 1)
                cpu = {"value": s["bytes"] / s["seconds"] / 1e9, "unit": "GB/s", "cores": os.cpu_count() or 1,
                       "kind": "oracle",
                       "sample": f"fwd+bwd of {s['images']} batch image(s) x C={s['channels']} planes of "
                                 f"{w.name}, B=1 each ({s['seconds']:.1f} s)"}
                # the same oracle on one thread, on a smaller sample of the same workload
                s1 = oracle_sample(w, args.cpu_seconds / 3.0, 1)
                cpu["single_thread"] = {
                    "value": s1["bytes"] / s1["seconds"] / 1e9, "unit": "GB/s", "cores": 1,
                    "sample": f"fwd+bwd of {s1['images']} batch image(s) x C={s1['channels']} planes of "
                              f"{w.name}, B=1 each ({s1['seconds']:.1f} s)"}
            except Exception as ex:  # the baseline must not sink the GPU line
                cpu = {"value": None, "unit": "GB/s", "cores": os.cpu_count() or 1, "kind": "oracle",
                       "sample": f"failed: {ex!r}"[:200]}
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": n_gpu, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded numpy PCG64, per-rank seed)",
            "config": config_of(w, n_gpu, args.passes, args.graph, flush),
            "pct_of_peak": 100.0 * value / n_gpu / peak,
            "gpix_ch_per_s": pixch * n_gpu / (ms * 1e-3) / 1e9,
            "fwd": {"ms": fwd_ms, "GB/s": fwd_gbs, "pct_of_peak": 100.0 * fwd_gbs / peak,
                    "gpix_ch_per_s": pixch / (fwd_ms * 1e-3) / 1e9 if fb else 0.0, "bytes": fb,
                    "kernel": lsp.gspn_variant_name(desc, 0)},
            "bwd": {"ms": bwd_ms, "GB/s": bwd_gbs, "pct_of_peak": 100.0 * bwd_gbs / peak,
                    "gpix_ch_per_s": pixch / (bwd_ms * 1e-3) / 1e9 if bb else 0.0, "bytes": bb,
                    "kernel": lsp.gspn_variant_name(desc, 1)},
            "roofline": {"bound": "hbm", "achieved": dom_gbs, "peak": peak, "unit": "GB/s",
                         "frac": dom_gbs / peak, "peak_source": f"{peak_src} copy bandwidth",
                         "kernel": lsp.gspn_variant_name(desc, 1 if dom == "bwd" else 0),
                         "traffic": ncu_traffic(dom, w)},
            "e2e": ({"value": job_gbs(fb + bb, n_gpu, e2e_ms), "unit": "GB/s",
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
                    if e2e_ms else None),
            "gpu_launches": launches,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------------------
# Compressed propagation block (gspn_block_fwd)
# ------------------------------------------------------------------------------
BLOCK_METRIC = "GSPN compressed block forward: achieved HBM GB/s (x, y, lambda and logits at the proxy width)"


def block_bytes(w) -> int:
    """Compulsory bytes of one block forward: x read and y written once,
    lambda and the tap logits at the proxy width read once, the projection
    matrices and the merger and norm weights read once."""
    n = w.B * w.C * w.H * w.W
    return (2 * n * 2 + 4 * w.B * w.Cp * w.H * w.W * 2 + 4 * w.B * 3 * w.H * w.W * 2 + 2 * w.C * w.Cp * 2
            + 5 * w.Cp * 4)


def block_config(w, n):
    return {"workload": w.name, "B": w.B, "C": w.C, "H": w.H, "W": w.W, "C_proxy": w.Cp, "groups": w.groups,
            "norm": "rms" if w.norm else "none", "io_dtype": "bf16", "pass": "fwd",
            "l2": "inputs larger than L2 (no flush needed)", "parallelism": f"replicas x{n}" if n > 1 else "1 GPU"}


def block_oracle_sample(w, target_s: float, nthreads: int):
    """The block oracle on as many whole batch images (each a B = 1 problem
    drawn before its timing) as fit in about target_s seconds."""
    import oracle
    imgs, t = 0, 0.0
    while imgs < w.B and (imgs == 0 or t < target_s):
        sw = w.replace(B=1, seed=w.seed + 7 + imgs)
        inp = synth.make_block_inputs(sw)
        t0 = time.perf_counter()
        oracle.block_fwd(inp["x"], inp["v_proj"], inp["logits"], inp["lam"], inp["alpha"], inp["gamma"],
                         inp["u_proj"], groups=sw.groups, norm=sw.norm, eps=sw.eps, dtype="bf16", nthreads=nthreads)
        t += time.perf_counter() - t0
        imgs += 1
    return {"seconds": t, "bytes": block_bytes(w.replace(B=1)) * imgs, "images": imgs}


def run_block(args, w):
    import torch

    import linear_spatial_propagation_b200 as lsp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    dev = torch.device("cuda", local)
    lsp.load(build_if_missing=False)
    inp = synth.make_block_inputs(w.replace(seed=w.seed + 1000 * rank))

    def pinned(a):
        t = torch.from_numpy(a)
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).pin_memory()

    h = {k: pinned(v) for k, v in inp.items()}
    d = {k: v.to(dev) for k, v in h.items()}
    y = torch.empty_like(d["x"])
    desc = lsp.make_block_desc(w.B, w.C, w.H, w.W, w.Cp, w.groups, w.norm, w.eps)
    ws = torch.empty(lsp.gspn_block_workspace_size(desc), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(din=d, yo=None):
        yo = y if yo is None else yo
        st = lsp.gspn_block_fwd(desc, din["x"].data_ptr(), din["v_proj"].data_ptr(), din["logits"].data_ptr(),
                                din["lam"].data_ptr(), din["alpha"].data_ptr(), din["gamma"].data_ptr(),
                                din["u_proj"].data_ptr(), yo.data_ptr(), ws.data_ptr(), ws.numel(),
                                stream.cuda_stream)
        if st:
            raise lsp.GspnError(st, "gspn_block_fwd")

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step()
    barrier()
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks(dist, e0.elapsed_time(e1) / K, dev)
    # end to end through the same entry point: every step copies its inputs up
    # from pinned host memory and y back down (serialised on the stream)
    E = args.e2e_steps
    e2e_ms = None
    h2d = sum(t.numel() * t.element_size() for t in h.values())
    d2h = y.numel() * y.element_size()
    if E > 0:
        hy = torch.empty(y.shape, dtype=y.dtype).pin_memory()
        barrier()
        e2 = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e2[0].record(stream)
        for _ in range(E):
            for k in d:
                d[k].copy_(h[k], non_blocking=True)
            step()
            hy.copy_(y, non_blocking=True)
        e2[1].record(stream)
        barrier()
        e2e_ms = max_over_ranks(dist, e2[0].elapsed_time(e2[1]) / E, dev)
    nb = block_bytes(w)
    peak, peak_src = measured_peaks()
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            try:
                smp = block_oracle_sample(w, args.cpu_seconds, os.cpu_count() or 1)
                cpu = {"value": smp["bytes"] / smp["seconds"] / 1e9, "unit": "GB/s", "cores": os.cpu_count() or 1,
                       "kind": "oracle", "sample": f"{smp['images']} batch image(s) of {w.name}, B=1 each "
                                                   f"({smp['seconds']:.1f} s)"}
            except Exception as ex:
                cpu = {"value": None, "unit": "GB/s", "cores": os.cpu_count() or 1, "kind": "oracle",
                       "sample": f"failed: {ex!r}"[:200]}
        gbs = nb / (ms * 1e-3) / 1e9
        line = {
            "metric": BLOCK_METRIC, "value": job_gbs(nb, world, ms), "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded numpy PCG64, per-rank seed)",
            "config": block_config(w, world), "bytes_per_step": nb,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "peak_source": f"{peak_src} copy bandwidth", "kernel": "gspn_block_fwd (4 launches)",
                         "traffic": None},
            "e2e": ({"value": job_gbs(nb, world, e2e_ms), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                     "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms} if e2e_ms else None),
            "gpu_launches": 4 * K, "clocks": clk, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.workload in synth.BLOCK_WORKLOADS:
        bw = synth.BLOCK_WORKLOADS[args.workload]
        if args.batch:
            bw = bw.replace(B=args.batch, name=f"{bw.name}@B{args.batch}")
        if args.impl == "reference":
            return run_block_reference(args, bw)
        return run_block(args, bw)
    w = synth.WORKLOADS.get(args.workload) or synth.EXTRA_WORKLOADS[args.workload]
    if not w.backward:
        w = w.replace(backward=True)
    if args.batch:
        w = w.replace(B=args.batch, name=f"{w.name}@B{args.batch}")
    if args.channels:
        w = w.replace(C=args.channels, name=f"{w.name}@C{args.channels}")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
