#!/usr/bin/env python
"""Benchmark of one clustered sparse attention layer call on B200.

A step is one pass of the whole hot path over one layer's synthetic inputs:
k-means on Q and on K (k-means++ seeding + ``iters`` rounds, the permutation
and segment offsets), the permuted values and their per-cluster means, the
compensation-error probe with greedy routing, and the attention pass with
centroid compensation that writes O in the original token order.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan720p]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun, one rank per GPU): every rank runs its own layer call
(its own batch element, no exchange), so the scaling is weak and
``value`` = slowest rank's ms per step / N (ms per layer call for the job).
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

from clustered_sparse_attention_b200 import synth  # noqa: E402

METRIC = "sparse-attn layer ms & effective TFLOPS at Wan 720p shape; % of tensor/HBM peak"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="wan720p", choices=sorted(synth.WORKLOADS))
    p.add_argument("--density", type=float, default=None)
    p.add_argument("--var-lambda", type=float, default=0.0,
                   help="strength of the variance-corrected compensation (0: plain)")
    p.add_argument("--topp", type=float, default=None,
                   help="routing budget per query cluster from the key clusters holding this "
                        "share of the estimated weight (instead of a fixed density)")
    p.add_argument("--iters", type=int, default=None)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--cpu-sample-seconds", type=float, default=15.0)
    p.add_argument("--heads", type=int, default=None,
                   help="override the head count (smaller profiling cases)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        # nvidia-smi's first query initialises NVML, which on a fresh machine
        # takes a while and disturbs the GPU: let it finish before any timing
        t0 = time.time()
        while not self.lines and time.time() - t0 < 15.0 and self.proc.poll() is None:
            time.sleep(0.05)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def window(self, t0, t1):
        """Keep only the samples taken inside [t0, t1] (the timed region)."""
        inside = [x for x in self.lines if t0 <= x[0] <= t1]
        if inside:
            self.lines = inside

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for _, ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# Algorithmic work of one layer call (what the method computes)
# ---------------------------------------------------------------------------
def attention_work(q_off, k_off, pair_off, pair_kc, d):
    """FLOPs of the attention pass: 4 d per (query row, key) of the selected
    blocks plus 4 d per (query row, skipped non-empty key cluster)."""
    flops_sel = 0.0
    flops_comp = 0.0
    pairs_sel = 0.0
    BH = q_off.shape[0]
    for bh in range(BH):
        qo, ko, po = q_off[bh], k_off[bh], pair_off[bh]
        nk = np.diff(ko)
        nonempty = int((nk > 0).sum())
        nq = np.diff(qo)
        for i in range(len(nq)):
            if nq[i] == 0:
                continue
            sel = pair_kc[bh][po[i]:po[i + 1]]
            keys = float(nk[sel].sum())
            pairs_sel += nq[i] * keys
            flops_sel += 4.0 * d * nq[i] * keys
            flops_comp += 4.0 * d * nq[i] * (nonempty - len(sel))
    return flops_sel, flops_comp, pairs_sel


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample, extrapolated to one layer call
# ---------------------------------------------------------------------------
def oracle_sample_ms(w, seconds=15.0, density=None, iters=None, topp=None):
    """Time the oracle's steps on one head's data with reduced counts, each
    scaled by the ratio of full to sampled work, and return (ms per layer
    call, threads, description).  Setup (inputs, one clustering) is untimed."""
    import oracle
    density = w.density if density is None else density
    iters = w.iters if iters is None else iters
    frac = max(0.05, min(1.0, seconds / 15.0))
    Q = synth.head_tensor(w, "q", 0, 0).astype(np.float64)
    K = synth.head_tensor(w, "k", 0, 0).astype(np.float64)
    V = synth.head_tensor(w, "v", 0, 0).astype(np.float64)
    N, d = Q.shape
    g = np.random.default_rng(0)
    # untimed setup: clusters from one assignment against sampled tokens
    cq0 = Q[g.choice(N, w.Cq, replace=False)]
    ck0 = K[g.choice(N, w.Ck, replace=False)]
    lq, _, _, _ = oracle.assign(Q, cq0)
    lk, _, _, _ = oracle.assign(K, ck0)
    timings = {}

    def timed(fn):
        t = time.perf_counter()
        r = fn()
        return time.perf_counter() - t, r

    # k-means++: C sequential passes; time a prefix of the passes
    npp = max(4, int(24 * frac))
    t, _ = timed(lambda: oracle.kmeanspp(K, npp, 1, 0))
    per_pass = t / npp
    timings["kmeanspp"] = per_pass * (w.Cq + w.Ck) if iters and w.iters else 0.0
    # assign: cost per (token x centroid); time a token subset against all centroids
    nt = max(256, int(2048 * frac))
    t_q, _ = timed(lambda: oracle.assign(Q[:nt], cq0))
    t_k, _ = timed(lambda: oracle.assign(K[:nt], ck0))
    timings["assign"] = (t_q + t_k) * (N / nt) * iters
    t, cent_q = timed(lambda: oracle.update(Q, lq, cq0))
    t2, cent_k = timed(lambda: oracle.update(K, lk, ck0))
    timings["update"] = (t + t2) * iters
    t, (pq, oq) = timed(lambda: oracle.stable_sort(lq, w.Cq))
    t2, (pk, ok) = timed(lambda: oracle.stable_sort(lk, w.Ck))
    timings["sort"] = (t + t2) * iters
    Qp, Kp, Vp = Q[pq], K[pk], V[pk]
    t, vbar = timed(lambda: oracle.segment_mean(Vp, ok))
    timings["centroids"] = t
    npr = max(1, int(4 * frac))
    t, Es = timed(lambda: oracle.probe(cent_q[:npr], Kp, Vp, cent_k, vbar, ok, w.scale))
    timings["probe"] = t * w.Cq / npr
    E = np.concatenate([Es, np.tile(Es, (w.Cq // npr + 1, 1))[:w.Cq - npr]], 0)
    if topp is None:
        t, (po, pkc) = timed(lambda: oracle.route(E.astype(np.float32), oq, ok, N, density))
    else:
        def topp_route():
            b, _ = oracle.topp_budget(cent_q, cent_k, oq, ok, topp, w.scale)
            return oracle.route(E.astype(np.float32), oq, ok, N, 1.0, budgets=b)
        t, (po, pkc) = timed(topp_route)
    timings["route"] = t
    nr = max(32, int(256 * frac))
    rows = g.choice(N, nr, replace=False)
    t, _ = timed(lambda: oracle.attend(Qp, Kp, Vp, oq, ok, po, pkc, cent_k, vbar, pq, w.scale,
                                       rows=rows))
    timings["attend"] = t * N / nr
    per_head = sum(timings.values())
    total_ms = per_head * w.B * w.H * 1e3
    desc = ("oracle on head (0,0) of %s, extrapolated x%d heads: k-means++ %d of %d passes, "
            "assign %d of %d tokens x %d iters, probe %d of %d probes, attend %d of %d rows; "
            "update/sort/centroids/route full" % (w.name, w.B * w.H, npp, w.Cq + w.Ck, nt, N,
                                                   iters, npr, w.Cq, nr, N))
    return total_ms, oracle.num_threads(), desc, {k: v * 1e3 for k, v in timings.items()}


# ---------------------------------------------------------------------------
def dist_setup(args):
    import torch

    from clustered_sparse_attention_b200 import ranks
    ws, rank, local = ranks.setup("nccl")
    if ws == 1:
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    from clustered_sparse_attention_b200 import ranks
    ranks.barrier(ws)


def max_over_ranks(x, ws):
    from clustered_sparse_attention_b200 import ranks
    return ranks.max_over_ranks(x, ws, device="cuda")


def run_reference(args, w):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.lib()
    secs = min(args.cpu_sample_seconds, 8.0)
    for _ in range(args.warmup):
        oracle_sample_ms(w, seconds=secs * 0.3, density=args.density, iters=args.iters,
                         topp=args.topp)
    vals = []
    desc = ""
    cores = 1
    for _ in range(args.steps):
        v, cores, desc, _ = oracle_sample_ms(w, seconds=secs, density=args.density, topp=args.topp,
                                             iters=args.iters)
        vals.append(v)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "ms",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": value,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, args),
        "cpu_baseline": {"value": value, "unit": "ms", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, args):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "Cq": w.Cq, "Ck": w.Ck,
            "iters": args.iters or w.iters,
            "compensation": ("variance-corrected, lambda %g" % args.var_lambda if args.var_lambda
                             else "plain (n e^{score of the centroid})"),
            "budget": ("top-p %g of the estimated weight per query cluster" % args.topp
                       if args.topp else "density %g (floor(density * N) keys per query cluster)"
                       % (args.density or w.density)),
            "kmeans_init": ("warm: one round from the previous step's centroids (step 0 cold, "
                            "40 rounds); inputs drift by %g N(0,1) per step" % w.drift
                            if w.warm_steps else "k-means++ (cold)"),
            "inputs": "%s, seeded Gaussian mixtures" % w.dtype,
            "l2": "inputs larger than L2 (3 x %.0f MB)" % (w.B * w.H * w.N * w.d * 2 / 1e6),
            "parallelism": "one independent layer call per GPU (no exchange)"}


# DRAM bytes (read + write) of one attend_sm100_kernel launch, from the ncu
# capture of the 8-head Wan 720p case (profiles/attend_sm100_wan720p_h8.md);
# traffic grows with the heads of a launch (same per-head routing), so other
# head counts of that shape scale it.  None for shapes not captured, and None
# while the kernel has changed since the capture.
ATTEND_TRAFFIC_H8_WAN720P = 561.704960e6 + 139.453696e6


def attend_traffic(w):
    if (ATTEND_TRAFFIC_H8_WAN720P is not None and w.name.startswith("wan720p") and w.N == 75600
            and w.d == 128 and w.Ck == 500):
        return ATTEND_TRAFFIC_H8_WAN720P * (w.B * w.H) / 8.0
    return None


def main():
    args = parse()
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name="%s_h%d" % (w.name, args.heads))
    if args.impl == "reference":
        return run_reference(args, w)

    import torch

    import clustered_sparse_attention_b200 as csa
    from clustered_sparse_attention_b200 import ranks as ranks_mod
    ws, rank, local = dist_setup(args)
    iters = args.iters or w.iters
    density = args.density or w.density
    dev = torch.device("cuda", torch.cuda.current_device())

    # inputs: this rank's own batch element (weak scaling), resident in HBM
    def host_tensor(name):
        if w.dtype == "f32":   # the small fp32 workload: every rank draws batch 0
            return torch.from_numpy(synth.layer_tensor(w, name, threads=min(16, os.cpu_count() or 1)))
        from clustered_sparse_attention_b200 import ranks
        bits = synth.layer_tensor_bits(w, name, threads=min(16, os.cpu_count() or 1),
                                       batch_offset=ranks.batch_offset(rank))
        return torch.from_numpy(bits).view(torch.bfloat16)

    host = {n: host_tensor(n).pin_memory() for n in ("q", "k", "v")}
    Q, K, V = (host[n].to(dev) for n in ("q", "k", "v"))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    ev_names = ("cluster_q", "cluster_k", "values", "route", "attend")

    # Warm-start workload (centroid cache, SVG2 section 3.4): step 0 is a cold
    # clustering (untimed) that fills the cache; every later step drifts the
    # inputs by drift * N(0, 1) per element (drawn on the device, before the
    # timed region) and clusters with one round from the previous centroids.
    warm = {"q": None, "k": None}
    if w.warm_steps:
        cold = csa.svgear_cluster(Q, w.Cq, 40, seed=2 * rank)
        warm["q"] = cold.centroids
        cold = csa.svgear_cluster(K, w.Ck, 40, seed=2 * rank + 1)
        warm["k"] = cold.centroids
        gen = torch.Generator(device=dev)
        n_inputs = max(3, args.warmup) + args.steps
        inputs, cur = [], [Q, K, V]
        for t in range(n_inputs):
            nxt = []
            for i, X in enumerate(cur):
                gen.manual_seed(1000003 * (t + 1) + 7919 * i + 104729 * rank)
                nxt.append((X.float() + w.drift * torch.randn(X.shape, generator=gen, device=dev,
                                                              dtype=torch.float32)).to(X.dtype))
            inputs.append(tuple(nxt))
            cur = nxt
        del cur
        torch.cuda.synchronize()
    step_no = [0]

    def next_inputs(Q, K, V):
        if not w.warm_steps:
            return Q, K, V
        t = step_no[0]
        step_no[0] += 1
        return inputs[t]

    def step(Q, K, V, events=None):
        def mark(i):
            if events is not None:
                events[i].record(stream)
        mark(0)
        cq = csa.svgear_cluster(Q, w.Cq, iters, warm_centroids=warm["q"], seed=2 * rank)
        mark(1)
        ck = csa.svgear_cluster(K, w.Ck, iters, warm_centroids=warm["k"], seed=2 * rank + 1)
        mark(2)
        if w.warm_steps:
            warm["q"], warm["k"] = cq.centroids, ck.centroids
        Vp = csa.svgear_permute(V, ck.perm)
        vbar = csa.svgear_centroids(Vp, ck.offsets, w.Ck)
        mark(3)
        if args.topp:
            po, pk, _ = csa.svgear_route_topp(cq.centroids, cq.offsets, ck.centroids, vbar,
                                              ck.offsets, ck.Xp, Vp, args.topp, w.scale)
        else:
            po, pk = csa.svgear_route(cq.centroids, cq.offsets, ck.centroids, vbar, ck.offsets,
                                      ck.Xp, Vp, density, w.scale)
        mark(4)
        kvar = csa.svgear_key_variance(ck.Xp, ck.offsets, w.Ck) if args.var_lambda else None
        O = csa.svgear_attend(cq.Xp, ck.Xp, Vp, cq.offsets, ck.offsets, po, pk, ck.centroids,
                              vbar, cq.perm, w.scale, kvar=kvar, lam=args.var_lambda)
        mark(5)
        return O, (cq, ck, po, pk, Vp)

    # the clock sampler starts (and finishes initialising) before the warm-up
    clocks = ClockSampler(local if ws > 1 else torch.cuda.current_device())
    clocks.start()
    for _ in range(max(3, args.warmup)):
        step(*next_inputs(Q, K, V))
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_inputs = [next_inputs(Q, K, V) for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    l0 = csa.kernel_launches()
    t_begin = time.time()
    start.record(stream)
    for s in range(args.steps):
        O, state = step(*step_inputs[s], evs[s])
    end.record(stream)
    torch.cuda.synchronize()
    t_end = time.time()
    barrier(ws)
    launches = csa.kernel_launches() - l0
    clocks.window(t_begin, t_end)
    clk = clocks.stop()
    ms_step = start.elapsed_time(end) / args.steps
    ms_step_max = max_over_ranks(ms_step, ws)
    stage_ms = {n: float(np.mean([evs[s][i].elapsed_time(evs[s][i + 1]) for s in range(args.steps)]))
                for i, n in enumerate(ev_names)}

    # algorithmic work of the attention pass (from the last step's routing)
    cq, ck, po, pk, Vp_last = state
    BH = w.B * w.H
    q_off = cq.offsets.view(BH, -1).cpu().numpy()
    k_off = ck.offsets.view(BH, -1).cpu().numpy()
    pair_off = po.view(BH, -1).cpu().numpy()
    pair_kc = pk.view(BH, -1).cpu().numpy()
    f_sel, f_comp, pairs = attention_work(q_off, k_off, pair_off, pair_kc, w.d)
    density_real = pairs / (float(w.N) * w.N * BH)
    peaks = load_peaks()
    attend_ms = stage_ms["attend"]
    achieved = (f_sel + f_comp) / (attend_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    if w.dtype == "bf16":
        roofline = {"kernel": "attend_sm100_kernel (svgear_attend, bf16)", "bound": "tensor",
                    "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak,
                    "peak_kind": "bf16 dense, sustained, %s" % (
                        "of measured" if peaks["source"] == "measured" else "of fallback"),
                    "traffic": attend_traffic(w), "flops_per_launch": f_sel + f_comp}
    else:
        # fp32 SIMT attention: FMA units, 148 SMs x 128 lanes x 2 flops x 1.965 GHz
        alu_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roofline = {"kernel": "attend_simt_kernel (svgear_attend, fp32)", "bound": "alu",
                    "achieved": achieved, "peak": alu_peak, "unit": "TFLOP/s",
                    "frac": achieved / alu_peak,
                    "peak_kind": "fp32 FMA, from unit counts and the 1965 MHz clock",
                    "traffic": None, "flops_per_launch": f_sel + f_comp}

    # quality of the timed configuration (not timed): attention recall and the
    # output error against dense attention on 64 sampled query rows per head
    g = np.random.default_rng(1234)
    R = min(64, w.N)
    rows = np.stack([np.sort(g.choice(w.N, R, replace=False)) for _ in range(BH)])
    rec, e2, r2 = csa.svgear_diagnostics(
        cq.Xp, ck.Xp, Vp_last, cq.offsets, ck.offsets, po, pk, O, cq.perm, w.scale,
        torch.from_numpy(rows.astype(np.int32)).view(w.B, w.H, R).to(dev))
    rec, e2, r2 = (t.double().cpu().numpy() for t in (rec, e2, r2))
    quality = {"rows_per_head": R, "recall_mean": float(rec.mean()),
               "recall_min": float(rec.min()),
               "relative_mse": float(e2.sum() / max(r2.sum(), 1e-300))}

    # end to end through the public host-buffer call: every step copies its
    # pinned host inputs to the device (overlapped with the stages that do not
    # read them yet) and reads O back into pinned host memory
    e2e = None
    if not args.no_e2e:
        Od_host = torch.empty((w.B, w.H, w.N, w.d), dtype=Q.dtype).pin_memory()

        def e2e_step():
            res = csa.layer_host(host["q"], host["k"], host["v"], w.Cq, w.Ck, iters, density,
                                 scale=w.scale, seed=rank, warm_q=warm["q"], warm_k=warm["k"],
                                 topp=args.topp, var_lambda=args.var_lambda, out=Od_host)
            if w.warm_steps:
                warm["q"], warm["k"] = res["q"].centroids, res["k"].centroids

        e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        e2e_ms = max_over_ranks(a.elapsed_time(b) / args.steps, ws)
        nbytes = w.B * w.H * w.N * w.d * 2
        e2e = {"value": ranks_mod.job_ms_per_call(e2e_ms, ws), "unit": "ms",
               "h2d_bytes_per_step": 3 * nbytes,
               "d2h_bytes_per_step": nbytes}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, cores, desc, parts = oracle_sample_ms(w, seconds=args.cpu_sample_seconds,
                                                 density=density, iters=iters, topp=args.topp)
        cpu = {"value": v, "unit": "ms", "cores": cores, "kind": "oracle", "sample": desc,
               "stages_ms": parts}

    if rank == 0:
        line = {
            "metric": METRIC, "value": ranks_mod.job_ms_per_call(ms_step_max, ws), "unit": "ms",
            "n_gpus": ws,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step_max,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic: seeded patch-coherent Gaussian mixtures at the %s shape" % w.name,
            "config": {**workload_config(w, args), "density_selected": density_real},
            "effective_tflops": (f_sel + f_comp) / (ms_step * 1e-3) / 1e12,
            "attention_tflops": achieved,
            "stages_ms": stage_ms,
            "roofline": roofline,
            "quality": quality,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clk,
            "gpu_launches": int(launches),
        }
        print(json.dumps(line), flush=True)
    ranks_mod.teardown(ws)


if __name__ == "__main__":
    main()
