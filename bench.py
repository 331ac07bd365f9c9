"""Benchmark of the MC-Sparse hot path on B200: reuse-step throughput at ~5% KV density.

    python bench.py [--gpus N --steps K --warmup W] [--workload I] [--impl ours|reference]

One step = one anchor period of the workload's schedule, i.e. every stage of
the path once: PDDP grouping, the anchor step (dense attention, exact group
scores, top-k selection, sparse pass + residual) and one reuse step (sparse
pass over the cached selection + residual) on drifted inputs. Inputs are
seeded synthetic fields resident in HBM before timing. `value` is the
executed tensor throughput of the reuse step (4 * n_q * k * d flops per head),
the headline of the workload; the line also carries the anchor-step and
dense-pass times, the reuse-vs-dense speedup, the roofline of the reuse
kernel, an end-to-end figure through the C ABI with host buffers, and the
fp64 CPU oracle timed on a bounded sample as a reported baseline.

With --gpus N > 1 (launched by torchrun) rank r runs batch elements
r*B .. r*B + B - 1 of a global batch of N * B (the path shards by batch with
no exchange), timings are the max over ranks, and `value` aggregates all
ranks ("weak" scaling); with --shard heads the ranks split the workload's
heads instead ("strong" scaling: the same job on more GPUs).
`--impl reference` times the oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import dataclasses
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "reuse-step ms & executed TFLOP/s at 5% KV density (% bf16 TC peak) vs dense"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with only this many heads (smaller case for profiling)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-flush", action="store_true",
                    help="do not flush L2 before each timed reuse / dense repetition")
    ap.add_argument("--shard", choices=["batch", "heads"], default="batch",
                    help="multi-GPU split: each rank its own batch element(s) (weak scaling) "
                         "or the workload's heads split over the ranks (strong scaling)")
    return ap.parse_args()


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples (every 50 ms) while the GPU is
    timed: from before the timed steps to after the last timed call (the steps,
    the separate reuse and dense timings and the end-to-end loop)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines: list[str] = []
        self.reader = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def start(self, wait_s: float = 5.0):
        """Starts the sampler and returns once its first sample has arrived
        (or after `wait_s`), so the timed region is covered from its start."""
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        import atexit
        atexit.register(self._kill)  # an error between start and stop ends the sampler too
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        t0 = time.perf_counter()
        while not self.lines and time.perf_counter() - t0 < wait_s and self.proc.poll() is None:
            time.sleep(0.01)

    def _kill(self):
        if self.proc is not None and self.proc.poll() is None:
            self.proc.kill()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.reader.join(timeout=5)
        rows = [r for r in csv.reader(io.StringIO("".join(self.lines))) if len(r) >= 9]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "sm_mhz_min": min(sm) if sm else None}


# ----------------------------------------------------------------- CPU oracle leg

def oracle_reuse_sample(wl, seconds: float, Q, K, V, idx_by_group, R_by_group, groups_h0):
    """Times the fp64 oracle's reuse step (sparse attention over the cached
    selection + residual) on whole groups of head 0 for about `seconds`.
    Returns (TFLOP/s, groups done, elapsed, threads)."""
    from oracle import oracle as orc
    Xq, Xk, Xv = (T[0, 0].double().numpy() for T in (Q, K, V))
    done, flops = 0, 0.0
    t0 = time.perf_counter()
    g = 0
    G = len(idx_by_group)
    while time.perf_counter() - t0 < seconds or done == 0:
        rows = orc.group_rows(groups_h0, wl.group_size, g % G)
        _ = orc.sparse(Xq[rows], Xk, Xv, idx_by_group[g % G]) + R_by_group[g % G]
        flops += 4.0 * len(rows) * wl.k * wl.head_dim
        done += 1
        g += 1
    el = time.perf_counter() - t0
    return flops / el / 1e12, done, el


def omp_threads() -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (os.cpu_count() or 1)


def synthetic_selection(wl, G, seed=0):
    """Ascending random k-subsets standing in for cached selections (CPU leg only)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    return [np.sort(rng.choice(wl.n_kv, size=wl.k, replace=False)).astype(np.int32)
            for _ in range(G)]


def reference_arm(args, wl):
    """The fp64 oracle timed on the host cores, same metric/unit/config."""
    import numpy as np
    from oracle import oracle as orc
    from token_level_sparse_pddp_b200.synthetic import InputStream
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    it = iter(InputStream(wl, head_ids=[0], steps=2))
    _, _, Q0, K0, V0 = next(it)
    _, _, Q1, K1, V1 = next(it)
    gs = wl.group_size
    G = wl.num_groups
    groups = np.concatenate([np.arange(wl.n_q), -np.ones(G * gs - wl.n_q)]).astype(np.int32)
    sel = synthetic_selection(wl, min(G, 4))
    Rg = [np.zeros((len(orc.group_rows(groups, gs, g)), wl.head_dim)) for g in range(len(sel))]
    per_step = max(0.5, min(5.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_reuse_sample(wl, per_step / 4, Q1, K1, V1, sel, Rg, groups)
    vals, ms = [], []
    for _ in range(args.steps):
        v, done, el = oracle_reuse_sample(wl, per_step, Q1, K1, V1, sel, Rg, groups)
        vals.append(v)
        ms.append(el * 1e3 / done)
    value = statistics.median(vals)
    sample = (f"reuse-step sparse attention + residual, fp64, on whole {gs}-query groups of "
              f"head 0 over random ascending k={wl.k} subsets standing in for the cached "
              f"selection, ~{per_step:.1f} s per step; TFLOP/s = executed flops / time; "
              f"ms_per_step is extrapolated from the sample's time per group to all "
              f"{wl.num_groups * wl.heads} groups of the workload")
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "TFLOP/s (executed, reuse step)", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": statistics.median(ms) * wl.num_groups * wl.heads,
        "ms_per_step_extrapolated": True,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s (executed, reuse step)",
                         "cores": omp_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s (executed, reuse step)",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(wl):
    return {"workload": wl.name, "batch": wl.batch, "heads": wl.heads, "n_q": wl.n_q,
            "n_kv": wl.n_kv, "head_dim": wl.head_dim, "group_size": wl.group_size, "k": wl.k,
            "kv_density": round(wl.k / wl.n_kv, 4), "input_dtype": wl.dtype,
            "step": "PDDP grouping + anchor step + one reuse step (drifted inputs)",
            "l2": "inputs larger than L2 (Q,K,V %.0f MB + R %.0f MB per step); the reuse and "
                  "dense timings also flush L2 (write of a 512 MB buffer) before each "
                  "repetition, medians reported"
                  % (3 * wl.batch * wl.heads * wl.n_kv * wl.head_dim * 2 / 1e6,
                     wl.batch * wl.heads * wl.n_q * wl.head_dim * 4 / 1e6)}


# ----------------------------------------------------------------- GPU arm

def main():
    args = parse()
    from token_level_sparse_pddp_b200.synthetic import InputStream, workload
    wl = workload(args.workload)
    if args.heads:
        wl = dataclasses.replace(wl, heads=args.heads, name=f"{wl.name}-H{args.heads}")
    if args.impl == "reference":
        os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))
        reference_arm(args, wl)
        return

    import torch
    from token_level_sparse_pddp_b200 import multi, tlsp

    info = multi.rank_info()
    world, rank, local = info.world, info.rank, info.local_rank
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    multi.init(info, "nccl", device=dev)

    def barrier():
        multi.barrier(info)

    def max_over_ranks(vals):
        return multi.max_over_ranks(info, vals, device=dev)

    peaks, peak_kind = load_peaks()
    full_wl = wl
    if args.shard == "heads":
        # rank r holds its contiguous share of the heads of one fixed batch
        my_heads = list(multi.head_shard(wl.heads, world, rank))
        it = iter(InputStream(wl, head_ids=my_heads, steps=2))
        wl = dataclasses.replace(wl, heads=len(my_heads))
    else:
        # rank r holds batch elements r*B .. r*B + B - 1 of a global batch of world * B
        it = iter(InputStream(wl, steps=2, batch_offset=multi.batch_offset(wl.batch, rank)))
    _, _, Qa, Ka, Va = next(it)
    _, _, Qr, Kr, Vr = next(it)
    Qa, Ka, Va = (t.to(dev) for t in (Qa, Ka, Va))
    Qr_h, Kr_h, Vr_h = (t.pin_memory() for t in (Qr, Kr, Vr))
    Qr, Kr, Vr = (t.to(dev) for t in (Qr_h, Kr_h, Vr_h))
    gs, k = wl.group_size, wl.k
    ws = tlsp.Workspace(tlsp.dims_of(Qa, Ka), gs, k, device=dev)
    G = wl.num_groups
    groups = torch.empty((wl.batch, wl.heads, G * gs), dtype=torch.int32, device=dev)
    O_full = torch.empty_like(Qa)
    idx = torch.empty((wl.batch, wl.heads, G, k), dtype=torch.int32, device=dev)
    R = torch.empty(Qa.shape, dtype=torch.float32, device=dev)
    O = torch.empty_like(Qr)

    def one_step(ev=None):
        if ev: ev[0].record()
        tlsp.group_queries(Qa, gs, ws, out=groups)
        if ev: ev[1].record()
        tlsp.anchor_attention(Qa, Ka, Va, groups, gs, k, ws, out=(O_full, idx, R))
        if ev: ev[2].record()
        tlsp.reuse_attention(Qr, Kr, Vr, groups, gs, k, idx, R, ws, out=O)
        if ev: ev[3].record()

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    if ws.status() != 0:
        raise RuntimeError(f"device status {tlsp.status_string(ws.status())} after warm-up")

    clocks = ClockSampler(local)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    launches0 = tlsp.launch_count()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for s in range(args.steps):
        one_step(events[s])
    t_end.record()
    torch.cuda.synchronize()
    barrier()
    launches = tlsp.launch_count() - launches0
    total_ms = t_start.elapsed_time(t_end)
    group_ms = [e[0].elapsed_time(e[1]) for e in events]
    anchor_ms = [e[1].elapsed_time(e[2]) for e in events]
    step_reuse_ms = [e[2].elapsed_time(e[3]) for e in events]
    if ws.status() != 0:
        raise RuntimeError(f"device status {tlsp.status_string(ws.status())} after timing")

    # The reuse step and the dense pass alone (the comparison point), each
    # repetition after an L2 flush (a 512 MB write) so K/V come from HBM as
    # they would on a fresh step.
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def timed(fn, reps, flush):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        for _ in range(2):
            fn()
        for r in range(reps):
            if flush:
                flush_buf.fill_(r & 0xff)
            ev[r][0].record()
            fn()
            ev[r][1].record()
        torch.cuda.synchronize()
        return [e[0].elapsed_time(e[1]) for e in ev]

    flush = not args.no_flush
    reuse_call = lambda: tlsp.reuse_attention(Qr, Kr, Vr, groups, gs, k, idx, R, ws, out=O)
    launches_r0 = tlsp.launch_count()
    reuse_ms = timed(reuse_call, args.steps, flush)
    reuse_launches = (tlsp.launch_count() - launches_r0) // (args.steps + 2)
    reuse_warm_ms = timed(reuse_call, args.steps, False)
    O_dense = torch.empty_like(Qa)
    dense_ms = timed(lambda: tlsp.dense_attention(Qa, Ka, Va, ws, out=O_dense), args.steps, flush)
    del flush_buf

    # End to end through the C ABI with host buffers: pinned inputs in,
    # result out, copies inside the timed region (reuse steps). The step is cut
    # into head chunks on three streams (host-to-device copies, reuse calls,
    # device-to-host copies), so chunk c's upload, chunk c-1's compute and
    # chunk c-2's download overlap; every call is the library's own reuse call
    # on a chunk of heads (per-head work, contiguous when the batch is 1).
    O_h = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    Qe, Ke, Ve = torch.empty_like(Qr), torch.empty_like(Kr), torch.empty_like(Vr)
    n_chunk = min(16, wl.heads) if wl.batch == 1 else 1
    bounds = [(c * wl.heads // n_chunk, (c + 1) * wl.heads // n_chunk) for c in range(n_chunk)]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]

    def e2e_step():
        main = torch.cuda.current_stream()
        for st in (s_in, s_cmp, s_out):
            st.wait_stream(main)
        for h0, h1 in bounds:
            hs = slice(h0, h1)
            with torch.cuda.stream(s_in):
                Qe[:, hs].copy_(Qr_h[:, hs], non_blocking=True)
                Ke[:, hs].copy_(Kr_h[:, hs], non_blocking=True)
                Ve[:, hs].copy_(Vr_h[:, hs], non_blocking=True)
            s_cmp.wait_stream(s_in)
            with torch.cuda.stream(s_cmp):
                tlsp.reuse_attention(Qe[:, hs], Ke[:, hs], Ve[:, hs], groups[:, hs], gs, k,
                                     idx[:, hs], R[:, hs], ws, out=O[:, hs])
            s_out.wait_stream(s_cmp)
            with torch.cuda.stream(s_out):
                O_h[:, hs].copy_(O[:, hs], non_blocking=True)
        main.wait_stream(s_out)

    for s in range(args.steps + 2):
        if s >= 2:
            e2e_ev[s - 2][0].record()
        e2e_step()
        if s >= 2:
            e2e_ev[s - 2][1].record()
    torch.cuda.synchronize()
    e2e_ms = [e[0].elapsed_time(e[1]) for e in e2e_ev]
    clk = clocks.stop()
    h2d = sum(t.numel() * t.element_size() for t in (Qr_h, Kr_h, Vr_h))
    d2h = O_h.numel() * O_h.element_size()

    med = statistics.median
    mx = max_over_ranks([total_ms, med(reuse_ms), med(anchor_ms), med(group_ms), med(dense_ms),
                         med(e2e_ms), med(reuse_warm_ms), med(step_reuse_ms)])
    (total_ms, reuse_mean, anchor_mean, group_mean, dense_mean, e2e_mean, reuse_warm,
     reuse_in_step) = mx
    flops = wl.reuse_flops()  # this rank's work
    # the whole job's work: world copies of the batch shard, or the full workload split by heads
    strong = args.shard == "heads"
    job_flops = full_wl.reuse_flops() if strong else world * flops
    job_dense = full_wl.dense_flops() if strong else world * wl.dense_flops()
    value = job_flops / (reuse_mean * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (reuse_mean * 1e-3) / 1e12
    traffic = None
    tr_path = os.path.join(ROOT, "profiles", "reuse_traffic.json")
    if os.path.exists(tr_path):
        tr = json.load(open(tr_path))
        if tr.get("workload") == wl.name and tr.get("kernel_rev") == tlsp_kernel_rev():
            traffic = tr.get("bytes_per_launch")

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s (executed, reuse step)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "strong" if strong else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded smooth field + noise)",
        "config": dict(config_of(full_wl),
                       global_batch=full_wl.batch if strong else world * wl.batch,
                       parallelism=f"heads{world}" if strong else f"dp{world}"),
        "reuse_ms": reuse_mean, "reuse_ms_warm_l2": reuse_warm, "reuse_ms_in_step": reuse_in_step,
        "reuse_launches": reuse_launches,
        "anchor_ms": anchor_mean, "group_queries_ms": group_mean,
        "dense_pass_ms": dense_mean, "reuse_vs_dense_speedup": dense_mean / reuse_mean,
        "reuse_dense_equiv_tflops": job_dense / (reuse_mean * 1e-3) / 1e12,
        "dense_pass_tflops": wl.dense_flops() / (dense_mean * 1e-3) / 1e12,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "reuse sparse attention (gathered QK^T, PV, +R epilogue)",
                     "peak_kind": f"bf16 dense burst, {peak_kind}",
                     "frac_of_sustained": achieved / float(peaks["bf16_tflops_sustained"])},
        "e2e": {"value": job_flops / (e2e_mean * 1e-3) / 1e12,
                "unit": "TFLOP/s (executed, reuse step)", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms": e2e_mean, "head_chunks": n_chunk},
        "gpu_launches": launches, "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import numpy as np
        from oracle import oracle as orc
        os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))
        g_h0 = groups[0, 0].cpu().numpy()
        sel = [idx[0, 0, g].cpu().numpy() for g in range(min(G, 8))]
        Rg = [R[0, 0, orc.group_rows(g_h0, gs, g)].double().cpu().numpy() for g in range(len(sel))]
        v, done, el = oracle_reuse_sample(wl, args.cpu_seconds, Qr[:, :1].cpu(), Kr[:, :1].cpu(),
                                          Vr[:, :1].cpu(), sel, Rg, g_h0)
        line["cpu_baseline"] = {
            "value": v, "unit": "TFLOP/s (executed, reuse step)", "cores": omp_threads(),
            "kind": "oracle",
            "sample": f"{done} groups x {gs} queries of head 0 (reuse step: sparse attention over "
                      f"the GPU's cached k={k} selection + R, fp64) in {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    multi.finish(info)


def tlsp_kernel_rev() -> str:
    """Hash of the sources of the sparse attention kernel: counters taken on
    other sources are stale."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "token_level_sparse_pddp_b200", "csrc")
    for f in ("attn_tc.cu", "tc_ptx.cuh", "common.cuh", "kernels.h"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
