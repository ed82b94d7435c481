#!/usr/bin/env python
"""LAPLEX benchmark: symmetric matvec throughput at n = 2^30 (fp32) on B200.

Workload (the headline): y = K x with K_ij = exp(-|a_i - a_j|), n = 2^30
anchors a ~ U(0, 2^30) generated already ascending (pre-sorted path), x ~ N(0,1),
B = 1, fp32.  One step = one laplex_matvec_sym call.  Inputs (12.9 GB moved per
step) are far larger than the 126 MB L2, so no L2 flush is needed between steps.

Printed (rank 0, one JSON line): metric/value (Gelem/s, whole job), roofline of
the step against the measured HBM copy peak, the other hot-path rows measured on
the same data (sort of the unsorted anchors, the permuted product, the backward
pass), the end-to-end number through host buffers, the fp64 oracle timed on the
host cores as a CPU baseline, SM clocks sampled during the timed region, and the
number of this library's kernels launched in the timed region.

--impl reference times the fp64 CPU oracle (the method's plain statement) on a
bounded sample of the same workload on the host cores.
Multi-GPU (torchrun): every rank runs an independent replica of the workload
(weak scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LAPLEX sym matvec Gelem/s at n=2^30 fp32; achieved HBM GB/s vs B200 peak"
BYTES_PER_ELEM_SYM = 12  # read s (4) + x (4), write y (4): the minimum the product moves
# launches of this library per pre-sorted single-column laplex_matvec_sym call:
# k_tile_local (first pass), k_carry_blocks, k_carry_tiles, k_tile_local (redo pass)
KERNELS_PER_SYM_CALL = 4


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--n", type=int, default=1 << 30)
    p.add_argument("--rows", default="sort,perm,carry,noalloc,backward,c2,c3,c4",
                   help="extra hot-path rows to time (comma list; empty for none)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def src_sha(*names):
    h = hashlib.sha256()
    for nm in names:
        with open(os.path.join(ROOT, "exact_laplace_b200", "csrc", nm), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel_key, sha, n):
    """dram read+write bytes per launch from profiles/traffic.txt, if the record was
    taken on the current kernel source (sha) at this n; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        if line.startswith("#") or not line.strip():
            continue
        kv = dict(tok.split("=", 1) for tok in line.split())
        if kv.get("key") == kernel_key and kv.get("src_sha") == sha and int(kv.get("n", -1)) == n:
            return float(kv["bytes_per_launch"])
    return None


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons (background process)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons, samples = [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f:
            parts = [t.strip() for t in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                if int(parts[0]) != self.idx:
                    continue
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            samples += 1
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.f.name)
        # samples taken while the GPU was busy (the timed loop) sit near the top clock
        busy = [c for c in sm if c > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": samples}


def cpu_baseline(n_total, seed, budget_s=10.0, m=1 << 24):
    """The fp64 oracle (sort-free sequential recurrences, plain C, one thread) on
    contiguous m-element samples of the same pre-sorted workload."""
    import oracle as O
    from exact_laplace_b200 import synth
    s, x = synth.sym_uniform(m, 0.0, float(1 << 30) * m / n_total, seed=seed, presorted=True)
    done, t0 = 0, time.perf_counter()
    while True:
        O.sym_sorted(s, x)
        done += m
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": done / el / 1e9, "unit": "Gelem/s", "cores": 1, "of": os.cpu_count(),
            "kind": "oracle",
            "sample": f"{done // m} x {m} contiguous anchors (same density as the n=2^30 "
                      f"workload), fp64 sequential recurrences, {el:.1f} s"}


def crow(ms, bytes_per_call, hbm):
    """Compact row: time per call (ms) and roofline fraction (algorithmic bytes
    per call / time / HBM peak), 4 and 3 significant digits."""
    return {"ms": float(f"{ms:.4g}"), "frac": float(f"{bytes_per_call / (ms * 1e-3) / 1e9 / hbm:.3g}")}


def reduce_max(v, world, device):
    """v on one rank; over several (torchrun replicas), the maximum over the
    ranks: the slowest replica decides the job's time."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, ms):
    """Whole-job throughput in units/s: every rank processes units_per_rank in
    the (max-over-ranks) time ms."""
    return world * units_per_rank / (ms * 1e-3)


def workload_config(n, world):
    """The config of the headline workload, the same for both arms."""
    e = int(round(math.log2(n))) if n > 0 and (n & (n - 1)) == 0 else None
    size = f"2^{e}" if e is not None else str(n)
    return {"workload": f"symmetric LAPLEX matvec y=Kx, K_ij=exp(-|a_i-a_j|), n={size} anchors "
                        f"U(0,{size}) pre-sorted, x~N(0,1), B=1, fp32",
            "n": n, "B": 1, "seed": "rank", "parallelism": f"replicas x{world}",
            "l2": f"inputs {12 * n / 1e9:.1f} GB per step vs 126 MB L2 (no flush needed above it)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as O
    from exact_laplace_b200 import synth
    m = 1 << 22
    s, x = synth.sym_uniform(m, 0.0, float(1 << 30) * m / args.n, seed=0, presorted=True)
    for _ in range(args.warmup):
        O.sym_sorted(s, x)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.sym_sorted(s, x)
    el = time.perf_counter() - t0
    val = args.steps * m / el / 1e9
    line = {"metric": METRIC, "value": val, "unit": "Gelem/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": workload_config(args.n, args.gpus),
            "cpu_baseline": {"value": val, "unit": "Gelem/s", "cores": 1, "of": os.cpu_count(),
                             "kind": "oracle",
                             "sample": f"{m} contiguous anchors of the workload's density per "
                                       "step, fp64 sequential recurrences on one host core"},
            "e2e": {"value": val, "unit": "Gelem/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    from exact_laplace_b200 import laplex as X
    from exact_laplace_b200 import synth

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        return reduce_max(v, world, dev)

    n = args.n
    hi = float(1 << 30)
    s_h, x_h = synth.sym_uniform(n, 0.0, hi * n / (1 << 30), seed=rank, presorted=True)
    s_p = torch.from_numpy(s_h).pin_memory()
    x_p = torch.from_numpy(x_h).pin_memory()
    del s_h, x_h
    s_d = s_p.to(dev)
    x_d = x_p.to(dev)
    y_d = torch.empty_like(x_d)
    stream = torch.cuda.current_stream(dev)

    def timed(fn, steps, warmup):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        return max_over_ranks(e0.elapsed_time(e1))

    # ---------------- headline: pre-sorted symmetric product
    def sym_call():
        X.matvec_sym(s_d, x_d, out=y_d)

    clk = Clocks(local)
    ms = timed(sym_call, args.steps, args.warmup)
    clocks = clk.stop()
    # then, in a separate run of calls, events around the dominant kernel
    # (k_tile_local) of every call, recorded by the library on the call's stream
    # (laplex_set_profile_events); kept out of the timed loop above
    kn = min(args.steps, 50)
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(kn)]
    for b, a in kev:  # torch creates the CUDA events at their first record
        b.record(stream)
        a.record(stream)
    torch.cuda.synchronize(dev)
    for b, a in kev:
        X.set_profile_events(b, a)
        sym_call()
    torch.cuda.synchronize(dev)
    X.set_profile_events(None, None)
    X.device_status(dev)
    kernel_ms = max_over_ranks(sum(b.elapsed_time(a) for b, a in kev) / len(kev))
    ms_step = ms / args.steps
    value = job_throughput(n, world, ms_step) / 1e9
    hbm, peak_kind = peaks()
    achieved = BYTES_PER_ELEM_SYM * n / (kernel_ms * 1e-3) / 1e9
    sha = src_sha("sym_stream.cu", "scan_core.cuh", "common.cuh", "bulk.cuh")
    traffic = traffic_from_profile("k_tile_local_presorted_b1", sha, n)
    roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": traffic,
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
            else "fallback 6650 GB/s",
            "kernel": "k_tile_local (dominant kernel of laplex_matvec_sym)",
            "kernel_ms": kernel_ms,
            "algorithmic_bytes_per_launch": BYTES_PER_ELEM_SYM * n,
            "whole_call": {"ms": ms_step, "achieved_GB_s": BYTES_PER_ELEM_SYM * n / (ms_step * 1e-3) / 1e9,
                           "frac": BYTES_PER_ELEM_SYM * n / (ms_step * 1e-3) / 1e9 / hbm,
                           "kernels": "memset + k_tile_local (first pass) + k_carry_blocks + k_carry_tiles + k_tile_local (redo pass)"}}

    # ---------------- other rows on the same data
    rows = {}
    wanted = [r for r in args.rows.split(",") if r]
    rsteps = max(3, min(20, args.steps // 10))
    if wanted:
        a_h = synth.uniform(n, 0.0, hi * n / (1 << 30), seed=rank, stream="a")
        a_d = torch.from_numpy(a_h).to(dev)
        del a_h
        s2 = torch.empty_like(a_d)
        p2 = torch.empty(n, dtype=torch.int32, device=dev)
        try:
            if "sort" in wanted:
                ms_s = timed(lambda: X.sort_anchors(a_d, s2, p2), rsteps, 1) / rsteps
                X.device_status(dev)
                rows["c5_sort"] = crow(ms_s, 12 * n, hbm)
            if "perm" in wanted:
                X.sort_anchors(a_d, s2, p2)
                ms_p = timed(lambda: X.matvec_sym(s2, x_d, p2, out=y_d), rsteps, 1) / rsteps
                X.device_status(dev)
                rows["c5_matvec_perm"] = crow(ms_p, 16 * n, hbm)
                # the plan: inverse permutation once per sort, then products whose
                # vectors move into and out of sorted order by bucketed scatters
                inv = torch.empty_like(p2)
                ms_i = timed(lambda: X.invert_perm(p2, out=inv), rsteps, 1) / rsteps
                rows["c5_invert_perm"] = crow(ms_i, 8 * n, hbm)
                ms_q = timed(lambda: X.matvec_sym_planned(s2, p2, inv, x_d, out=y_d), rsteps, 1) / rsteps
                X.device_status(dev)
                rows["c5_matvec_planned"] = crow(ms_q, 16 * n, hbm)
                del inv
            if "carry" in wanted:
                # anchors that change every step: the sort carrying x, then the
                # one-call product (sort carrying x, product, y back to caller order)
                xs = torch.empty_like(x_d)
                ms_c = timed(lambda: X.sort_anchors_carry(a_d, x_d, s2, p2, xs), rsteps, 1) / rsteps
                X.device_status(dev)
                rows["c5_sort_carry"] = crow(ms_c, 20 * n, hbm)
                del xs
                ms_u = timed(lambda: X.matvec_sym_unsorted(a_d, x_d, out=y_d, sorted_out=s2, perm_out=p2),
                             rsteps, 1) / rsteps
                X.device_status(dev)
                rows["c5_matvec_unsorted"] = crow(ms_u, 20 * n, hbm)
        except X.LaplexError as e:
            rows["sort_error"] = str(e)
        del a_d, s2, p2
        if "noalloc" in wanted:
            # the allocation-free entry point on the headline's data
            ms_n = timed(lambda: X.matvec_sym_noalloc(s_d, x_d, out=y_d), rsteps, 1) / rsteps
            X.device_status(dev)
            rows["c5_matvec_noalloc"] = crow(ms_n, BYTES_PER_ELEM_SYM * n, hbm)
        if "backward" in wanted:
            try:
                g_d = torch.from_numpy(synth.normal(n, seed=rank, stream="g")).to(dev)
                dx = torch.empty_like(x_d)
                da = torch.empty_like(x_d)
                ms_b = timed(lambda: X.backward(s_d, x_d, g_d, dx_out=dx, da_out=da), rsteps, 1) / rsteps
                X.device_status(dev)
                rows["c5_backward"] = crow(ms_b, 20 * n, hbm)
                del g_d, dx, da
            except X.LaplexError as e:
                rows["backward_error"] = str(e)
        torch.cuda.empty_cache()

    # ---------------- the other workloads (inputs near or below L2 size: flushed)
    flush_buf = torch.ones(64 << 20, dtype=torch.float32, device=dev)  # 256 MB

    def timed_flush(fn, steps):
        """Sum of per-call device times, the 126 MB L2 flushed (a 256 MB read)
        before every call and outside the timed events.  A spin kernel queued
        first keeps the device behind the host, so the events time the call's
        kernels and not the host's launch latency."""
        fn()
        torch.cuda.synchronize(dev)
        evs = []
        for _ in range(steps):
            torch.cuda._sleep(1_000_000)
            flush_buf.sum()  # read: leaves L2 holding clean lines of another buffer
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize(dev)
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in evs)) / steps

    def timed_warm(fn, steps):
        """Mean device time of back-to-back calls (inputs left in L2 by the
        previous call where they fit)."""
        return timed(fn, steps, 2) / steps

    def graphed(fn):
        """fn captured once into a CUDA graph (after an eager call on the
        capture stream, which sizes its workspace); returns the replay."""
        s_cap = torch.cuda.Stream(dev)
        s_cap.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s_cap):
            fn()
        torch.cuda.current_stream(dev).wait_stream(s_cap)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s_cap):
            fn()
        return g

    def frow(fn, bytes_per, steps):
        """A row timed both with L2 flushed before every call (ms, frac) and
        warm (warm_ms); frac = algorithmic bytes / time / HBM peak."""
        r = crow(timed_flush(fn, steps), bytes_per, hbm)
        r["warm_ms"] = crow(timed_warm(fn, steps), bytes_per, hbm)["ms"]
        return r

    fsteps = max(10, min(20, args.steps))  # calls per C2-C4 row (each well under a millisecond)
    try:
        if "c2" in wanted:
            n2 = 1 << 24
            for B in (1, 8):
                a2, x2 = synth.sym_normal(n2, 2000.0, B=B, seed=rank)
                a2d = torch.from_numpy(a2).to(dev)
                x2d = torch.from_numpy(x2).to(dev)
                y2d = torch.empty_like(x2d)
                s2d = torch.empty_like(a2d)
                p2d = torch.empty(n2, dtype=torch.int32, device=dev)

                def c2_full():
                    X.sort_anchors(a2d, s2d, p2d)
                    X.matvec_sym(s2d, x2d, p2d, out=y2d)
                rows[f"c2_sort_and_matvec_B{B}"] = frow(c2_full, n2 * (12 + 16 + 8 * B), fsteps)
                X.sort_anchors(a2d, s2d, p2d)
                xs = x2d[p2d.long()].contiguous()
                rows[f"c2_presorted_B{B}"] = frow(lambda: X.matvec_sym(s2d, xs, out=y2d), n2 * (4 + 8 * B), fsteps)
                del a2d, x2d, y2d, s2d, p2d, xs
            X.device_status(dev)
        if "c3" in wanted:
            a3, b3, x3, w3 = synth.general_ties(1 << 22, 1 << 20, -1000.0, 1000.0, seed=rank)
            a3d, b3d = torch.from_numpy(a3).to(dev), torch.from_numpy(b3).to(dev)
            sa, pa = X.sort_anchors(a3d)
            sb, pb = X.sort_anchors(b3d)
            x3d, w3d = torch.from_numpy(x3).to(dev), torch.from_numpy(w3).to(dev)
            xs3 = x3d[pb.long()].contiguous()
            ws3 = w3d[pa.long()].contiguous()
            y3 = torch.empty_like(ws3)
            z3 = torch.empty_like(xs3)
            nn, kk = 1 << 22, 1 << 20
            rows["c3_general_Kx"] = frow(lambda: X.matvec_general(sa, sb, xs3, out=y3), 8 * nn + 8 * kk, fsteps)
            # the same call replayed from a CUDA graph (no per-kernel launch from the host)
            g3 = graphed(lambda: X.matvec_general(sa, sb, xs3, out=y3))
            rows["c3_general_Kx_graph"] = frow(g3.replay, 8 * nn + 8 * kk, fsteps)
            del g3
            rows["c3_general_KTw"] = frow(lambda: X.matvec_general(sa, sb, ws3, transpose=True, out=z3), 8 * nn + 8 * kk, fsteps)
            # anchor gradients of <w, K x> (sorted order): reads a, b, x, w; writes dx, da, db
            rows["c3_backward_general"] = frow(lambda: X.backward_general(sa, sb, xs3, ws3), 16 * nn + 16 * kk, fsteps)
            # weighted Gram matrix of 4096 a-points over the 2^20 b-points (output 64 MB)
            sa4 = sa[:: (nn // 4096)].contiguous()
            rows["gram_matrix_4096x2^20"] = frow(lambda: X.gram_matrix(sa4, sb, xs3.abs()), 4 * 4096 * 4096 + 12 * kk, fsteps)
            # phased anchor and phase gradients (phases ~ U(0, 2 pi), sorted order):
            # reads a, phi, w, b, psi, x; writes dphi, da, dx, dpsi, db
            phi3 = torch.from_numpy(synth.uniform(nn, 0.0, 2 * math.pi, seed=rank, stream="phi")).to(dev)
            psi3 = torch.from_numpy(synth.uniform(kk, 0.0, 2 * math.pi, seed=rank, stream="psi")).to(dev)
            rows["c3_backward_phased"] = frow(lambda: X.backward_phased(sa, phi3, xs3, ws3, sb=sb, psi=psi3), 20 * nn + 24 * kk, fsteps)
            X.device_status(dev)
            del a3d, b3d, sa, pa, sb, pb, x3d, w3d, xs3, ws3, y3, z3, phi3, psi3
        if "c4" in wanted:
            a4, phi4, v4 = synth.phased_image(seed=rank)
            n4 = a4.size
            a4d = torch.from_numpy(a4).to(dev)
            s4, p4 = X.sort_anchors(a4d)
            phis = torch.from_numpy(phi4).to(dev)[p4.long()].contiguous()
            vs = torch.from_numpy(v4).to(dev)[p4.long()].contiguous()
            y4 = torch.empty_like(vs)
            rows["c4_phased_Kv"] = frow(lambda: X.matvec_phased(s4, phis, vs, out=y4), 16 * n4, fsteps)
            g4 = graphed(lambda: X.matvec_phased(s4, phis, vs, out=y4))
            rows["c4_phased_Kv_graph"] = frow(g4.replay, 16 * n4, fsteps)
            del g4
            rows["c4_gram_KTKv"] = frow(lambda: X.gram(s4, vs, phi=phis, out=y4), 32 * n4, fsteps)
            gs4 = torch.from_numpy(synth.normal(n4, seed=rank, stream="g")).to(dev)
            rows["c4_backward_phased"] = frow(lambda: X.backward_phased(s4, phis, vs, gs4), 28 * n4, fsteps)
            X.device_status(dev)
            del a4d, s4, p4, phis, vs, y4, gs4
    except X.LaplexError as e:
        rows["rows_error"] = str(e)
    del flush_buf
    torch.cuda.empty_cache()

    # ---------------- end to end through host buffers (pinned)
    e2e = None
    if not args.no_e2e:
        # whole steps through host buffers: every step copies its s and x from
        # pinned host memory and its y back; the streamer overlaps step k's
        # copy in with step k-1's product and step k-2's copy out (12 steps:
        # the last copy out, not overlapped, weighs 1/12 of a step)
        y_p = torch.empty(n, dtype=torch.float32).pin_memory()
        esteps = max(3, min(12, args.steps))
        hs = X.HostStreamer(n, device=dev)
        hs.submit(s_p, x_p, y_p)  # warm-up step
        hs.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(hs.h2d)
        for _ in range(esteps):
            hs.submit(s_p, x_p, y_p)
        e1.record(hs.d2h)
        hs.synchronize()
        barrier()
        ms_e = max_over_ranks(e0.elapsed_time(e1))
        del hs
        torch.cuda.empty_cache()
        e2e = {"value": world * n / (ms_e / esteps * 1e-3) / 1e9, "unit": "Gelem/s",
               "h2d_bytes_per_step": s_p.numel() * 4 + x_p.numel() * 4,
               "d2h_bytes_per_step": y_p.numel() * 4, "steps": esteps,
               "path": "exact_laplace_b200.laplex.HostStreamer: pinned host -> device, "
                       "laplex_matvec_sym, device -> pinned host, overlapped across steps"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(n, 0)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic",
                "config": workload_config(n, world),
                "roofline": roof, "e2e": e2e, "cpu_baseline": cpu,
                "clocks": clocks, "gpu_launches": KERNELS_PER_SYM_CALL * args.steps,
                # last, so that a tail of the line keeps them; the n = 2^30 rows at the very end
                "rows": {**{k: v for k, v in rows.items() if not k.startswith("c5")},
                         **{k: v for k, v in rows.items() if k.startswith("c5")}}}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
