#!/usr/bin/env python
"""Benchmark of one clustered sparse attention layer call on B200.

A step is one pass of the whole hot path over one layer's synthetic inputs,
one svgear_layer call through the C ABI: k-means on Q and on K (k-means++
seeding + ``iters`` rounds, the permutation and segment offsets), the
permuted values and their per-cluster means, the compensation-error probe
with greedy routing, and the attention pass with centroid compensation that
writes O in the original token order.  CUDA events recorded by the call at
its stage boundaries give the per-stage times.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan720p]
    python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Multi-GPU (torchrun, one rank per GPU): by default the ranks split the heads
of one layer call (rank r takes a contiguous head range, no data moves
between ranks), so the scaling is strong and ``value`` = the slowest rank's
ms per call; ``--split batch`` instead gives every rank its own batch element
(weak scaling, ``value`` = slowest rank's ms per step / N).
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
    p.add_argument("--heads", type=int, default=None,
                   help="override the head count (smaller profiling cases)")
    p.add_argument("--split", choices=["heads", "batch"], default="heads",
                   help="multi-GPU: split one call's heads (strong) or one batch element per "
                        "rank (weak)")
    p.add_argument("--cpu-samples", type=int, default=3,
                   help="runs of the oracle's sample behind cpu_baseline (the median is kept)")
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
class OracleSample:
    """The CPU oracle on head (0, 0) of a workload, from that head's own
    clustered state, timed on a fixed sample and extrapolated to one layer
    call.  The same sample serves the bench's cpu_baseline and every step of
    the reference arm, so the two agree up to timing noise.

    Untimed set-up: the head's inputs and its clustering by the oracle itself
    (k-means++, then Lloyd rounds until no label moves -- the fixed point, at
    which further rounds repeat the same result -- or ``iters`` rounds), the
    permuted tensors, value centroids, errors and pairs.

    Timed sample, in the layer's order: k-means++ on Q and on K in full (all
    Cq + Ck passes); one full round of assign + update + stable sort for Q
    and for K, counted ``iters`` times (every round does the same work); the
    value permutation and centroids; the probe for every query cluster and
    the routing; attention for every ROW_STRIDE-th permuted query row,
    counted ROW_STRIDE times.  The head's time times B*H is the layer's."""

    ROW_STRIDE = 64

    def __init__(self, w, density=None, iters=None, topp=None, var_lambda=0.0):
        import oracle
        self.oracle = oracle
        self.w = w
        self.density = w.density if density is None else density
        self.iters = w.iters if iters is None else iters
        self.topp = topp
        self.lam = var_lambda
        f64 = lambda a: np.ascontiguousarray(a, np.float64)  # noqa: E731
        self.Q, self.K, self.V = (f64(synth.head_tensor(w, t, 0, 0)) for t in ("q", "k", "v"))
        self.cq = self._cluster(self.Q, w.Cq, 0)
        self.ck = self._cluster(self.K, w.Ck, 1)
        self.pq, self.oq = oracle.stable_sort(self.cq[1], w.Cq)
        self.pk, self.ok = oracle.stable_sort(self.ck[1], w.Ck)
        self.Qp, self.Kp, self.Vp = self.Q[self.pq], self.K[self.pk], self.V[self.pk]
        self.vbar = oracle.segment_mean(self.Vp, self.ok)
        self.rows = np.arange(0, w.N, self.ROW_STRIDE)

    def _cluster(self, X, C, seed):
        o = self.oracle
        idx, _ = o.kmeanspp(X, C, seed, 0)
        cent, labels = X[idx].copy(), None
        for _ in range(self.iters):
            lab, _, _, _ = o.assign(X, cent)
            if labels is not None and np.array_equal(lab, labels):
                break
            labels = lab
            cent = o.update(X, labels, cent)
        return cent, labels

    def run(self):
        """(ms per layer call, per-stage ms of the whole call)."""
        o, w = self.oracle, self.w
        t = {}

        def timed(name, fn, times=1.0):
            t0 = time.perf_counter()
            r = fn()
            t[name] = t.get(name, 0.0) + (time.perf_counter() - t0) * times
            return r

        timed("kmeanspp", lambda: o.kmeanspp(self.Q, w.Cq, 0, 0))
        timed("kmeanspp", lambda: o.kmeanspp(self.K, w.Ck, 1, 0))
        for X, (cent, lab), C in ((self.Q, self.cq, w.Cq), (self.K, self.ck, w.Ck)):
            timed("assign", lambda: o.assign(X, cent), self.iters)
            timed("update", lambda: o.update(X, lab, cent), self.iters)
            timed("sort", lambda: o.stable_sort(lab, C), self.iters)
        timed("values", lambda: o.segment_mean(self.V[self.pk], self.ok))
        E = timed("probe", lambda: o.probe(self.cq[0], self.Kp, self.Vp, self.ck[0], self.vbar,
                                           self.ok, w.scale))
        if self.topp is None:
            po, pkc = timed("route", lambda: o.route(E.astype(np.float32), self.oq, self.ok,
                                                     w.N, self.density))
        else:
            def topp_route():
                b, _ = o.topp_budget(self.cq[0], self.ck[0], self.oq, self.ok, self.topp,
                                     w.scale)
                return o.route(E.astype(np.float32), self.oq, self.ok, w.N, 1.0, budgets=b)
            po, pkc = timed("route", topp_route)
        kvar = None
        if self.lam:
            kvar = timed("values", lambda: o.segment_var(self.Kp, self.ok))
        timed("attend", lambda: o.attend(self.Qp, self.Kp, self.Vp, self.oq, self.ok, po, pkc,
                                         self.ck[0], self.vbar, self.pq, w.scale, rows=self.rows,
                                         kvar=kvar, lam=self.lam),
              w.N / len(self.rows))
        heads = w.B * w.H
        return sum(t.values()) * heads * 1e3, {k: v * heads * 1e3 for k, v in t.items()}

    def describe(self):
        w = self.w
        return ("oracle on head (0,0) of %s from its own clustering, x%d heads: k-means++ in full "
                "(%d passes), one full assign/update/sort round of Q and K x %d rounds, value "
                "centroids, probe and routing in full, attention on every %dth permuted row "
                "(%d of %d) x %d" % (w.name, w.B * w.H, w.Cq + w.Ck, self.iters, self.ROW_STRIDE,
                                     len(self.rows), w.N, self.ROW_STRIDE))


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
    sample = OracleSample(w, density=args.density, iters=args.iters, topp=args.topp,
                          var_lambda=args.var_lambda)
    for _ in range(args.warmup):
        sample.run()
    vals = [sample.run()[0] for _ in range(args.steps)]
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "ms",
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": value,
        "higher_is_better": False, "scaling": "strong" if args.split == "heads" else "weak",
        "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, args, ws),
        "cpu_baseline": {"value": value, "unit": "ms", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample.describe(),
                         "spread": [float(min(vals)), float(max(vals))]},
        "e2e": {"value": value, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, args, ws=1):
    if ws > 1 and args.split == "heads":
        par = ("heads split over %d GPUs (%d-%d heads each), no data exchanged"
               % (ws, w.H // ws, -(-w.H // ws)))
    elif ws > 1:
        par = "one independent layer call per GPU on its own batch element (no exchange)"
    else:
        par = "one GPU"
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
            "parallelism": par}


# ---------------------------------------------------------------------------
# DRAM traffic of the attention kernel from a committed ncu capture
# ---------------------------------------------------------------------------
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")
ATTEND_SOURCES = ("attend_sm100.cu", "tc_ptx.cuh", "tc_wait.cuh", "common.cuh", "tma_host.h")


def sources_sha256(names):
    import hashlib
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "clustered_sparse_attention_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attend_traffic(w):
    """DRAM bytes (read + write) of one attention launch of workload w, from
    the capture record of the same kernel source (sha256 of its files) on the
    same shape, scaled by the launch's heads (every head has the same routing
    statistics).  None when no record matches: the kernel changed since its
    capture, or the shape was never captured."""
    if not os.path.exists(TRAFFIC_RECORD):
        return None
    with open(TRAFFIC_RECORD) as f:
        records = json.load(f).get("records", [])
    sha = sources_sha256(ATTEND_SOURCES)
    for r in records:
        if (r.get("kernel") == "attend_sm100_kernel" and r.get("sources_sha256") == sha
                and r.get("N") == w.N and r.get("Cq") == w.Cq and r.get("Ck") == w.Ck
                and r.get("d") == w.d and abs(r.get("density", -1) - w.density) < 1e-9):
            return r["dram_bytes_per_launch"] * (w.B * w.H) / r["heads"]
    return None


def main():
    args = parse()
    w = synth.WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name="%s_h%d" % (w.name, args.heads))
    if args.density:
        import dataclasses
        w = dataclasses.replace(w, density=args.density)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch

    import clustered_sparse_attention_b200 as csa
    from clustered_sparse_attention_b200 import ranks as ranks_mod
    ws, rank, local = dist_setup(args)
    iters = args.iters or w.iters
    density = w.density
    dev = torch.device("cuda", torch.cuda.current_device())
    threads = min(16, os.cpu_count() or 1)

    # this rank's share: a head range of batch element 0 (head split) or its
    # own batch element (batch split); the inputs are resident in HBM
    split = args.split if ws > 1 else "heads"
    heads = list(range(w.H))
    batch_offset = 0
    if split == "heads":
        lo, hi = ranks_mod.head_range(w.H, ws, rank)
        heads = list(range(lo, hi))
    else:
        batch_offset = ranks_mod.batch_offset(rank)
    Hl = len(heads)

    def host_tensor(name):
        if w.dtype == "f32":
            return torch.from_numpy(synth.layer_tensor(w, name, heads=heads, threads=threads))
        bits = synth.layer_tensor_bits(w, name, heads=heads, threads=threads,
                                       batch_offset=batch_offset)
        return torch.from_numpy(bits).view(torch.bfloat16)

    host = {n: host_tensor(n).pin_memory() for n in ("q", "k", "v")}
    Q, K, V = (host[n].to(dev) for n in ("q", "k", "v"))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev_names = ("cluster_q", "cluster_k", "values", "route", "attend")
    common = dict(scale=w.scale, seed=rank, topp=args.topp, var_lambda=args.var_lambda)

    # Warm-start workload (centroid cache, SVG2 section 3.4): a cold call
    # (untimed) fills the cache; every later step's inputs drift by
    # drift * N(0, 1) per element (drawn on the device before the timed
    # region) and each call clusters with one round from the previous
    # centroids, updating the cache in place.
    warm = {"q": None, "k": None}
    inputs = None
    if w.warm_steps:
        _, warm["q"], warm["k"] = csa.svgear_layer(Q, K, V, w.Cq, w.Ck, 40, density, **common)
        gen = torch.Generator(device=dev)
        inputs, cur = [], [Q, K, V]
        for t in range(max(3, args.warmup) + args.steps + 1):
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

    def next_inputs():
        if inputs is None:
            return Q, K, V
        t = step_no[0]
        step_no[0] += 1
        return inputs[t]

    O = torch.empty_like(Q)

    def step(Qs, Ks, Vs, events=None):
        csa.svgear_layer(Qs, Ks, Vs, w.Cq, w.Ck, iters, density, O=O, warm_q=warm["q"],
                         warm_k=warm["k"], cent_q=warm["q"], cent_k=warm["k"], stage_events=events,
                         **common)

    # the clock sampler starts (and finishes initialising) before the warm-up
    clocks = ClockSampler(local if ws > 1 else torch.cuda.current_device())
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    for e in (x for row in evs for x in row):
        e.record(stream)          # each CUDA event exists from its first record
    for _ in range(max(3, args.warmup)):
        step(*next_inputs())
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_inputs = [next_inputs() for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize()
    l0 = csa.kernel_launches()
    t_begin = time.time()
    start.record(stream)
    for s in range(args.steps):
        step(*step_inputs[s], evs[s])
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

    # Work and quality (untimed): the same call run stage by stage on the last
    # step's inputs returns its intermediates (the kernels are deterministic,
    # so a cold call repeats the timed one exactly; a warm call is one more
    # step from the cache).
    Qs, Ks, Vs = step_inputs[-1]
    ref = csa.layer(Qs, Ks, Vs, w.Cq, w.Ck, iters, density, w.scale, seed=rank,
                    warm_q=None if warm["q"] is None else warm["q"].clone(),
                    warm_k=None if warm["k"] is None else warm["k"].clone(), topp=args.topp,
                    var_lambda=args.var_lambda)
    cq, ck, po, pk, Vp_last = ref["q"], ref["k"], ref["pair_off"], ref["pair_kc"], ref["Vp"]
    BH = w.B * Hl
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
        import dataclasses
        traffic = attend_traffic(dataclasses.replace(w, H=Hl))
        roofline = {"kernel": "attend_sm100_kernel (svgear_attend, bf16)", "bound": "tensor",
                    "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak,
                    "peak_kind": "bf16 dense, sustained, %s" % (
                        "of measured" if peaks["source"] == "measured" else "of fallback"),
                    "traffic": traffic, "flops_per_launch": f_sel + f_comp}
    else:
        # fp32 SIMT attention: FMA units, 148 SMs x 128 lanes x 2 flops x 1.965 GHz
        alu_peak = 148 * 128 * 2 * 1.965e9 / 1e12
        roofline = {"kernel": "attend_simt_kernel (svgear_attend, fp32)", "bound": "alu",
                    "achieved": achieved, "peak": alu_peak, "unit": "TFLOP/s",
                    "frac": achieved / alu_peak,
                    "peak_kind": "fp32 FMA, from unit counts and the 1965 MHz clock",
                    "traffic": None, "flops_per_launch": f_sel + f_comp}

    # quality of the timed configuration: attention recall and the output
    # error against dense attention on 64 sampled query rows per head
    g = np.random.default_rng(1234)
    R = min(64, w.N)
    rows = np.stack([np.sort(g.choice(w.N, R, replace=False)) for _ in range(BH)])
    rec, e2, r2 = csa.svgear_diagnostics(
        cq.Xp, ck.Xp, Vp_last, cq.offsets, ck.offsets, po, pk, ref["O"], cq.perm, w.scale,
        torch.from_numpy(rows.astype(np.int32)).view(w.B, Hl, R).to(dev))
    rec, e2, r2 = (t.double().cpu().numpy() for t in (rec, e2, r2))
    quality = {"rows_per_head": R, "recall_mean": float(rec.mean()),
               "recall_min": float(rec.min()),
               "relative_mse": float(e2.sum() / max(r2.sum(), 1e-300))}
    del ref, cq, ck, po, pk, Vp_last

    # end to end through the C ABI's host-buffer call: every step copies this
    # rank's pinned host inputs to the device inside the call (overlapped with
    # the stages that do not read them yet) and O back into pinned host memory
    e2e = None
    if not args.no_e2e:
        Od_host = torch.empty(tuple(host["q"].shape), dtype=Q.dtype).pin_memory()

        def e2e_step():
            csa.layer_host(host["q"], host["k"], host["v"], w.Cq, w.Ck, iters, density,
                           out=Od_host, warm_q=warm["q"], warm_k=warm["k"], cent_q=warm["q"],
                           cent_k=warm["k"], **common)

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
        nbytes = int(host["q"].numel()) * host["q"].element_size()
        e2e = {"value": ranks_mod.job_ms_per_call(e2e_ms, ws, split), "unit": "ms",
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "call": "svgear_layer_host (C ABI, host buffers)"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        import oracle
        sample = OracleSample(w, density=density, iters=iters, topp=args.topp,
                              var_lambda=args.var_lambda)
        sample.run()              # warm-up: caches, page faults, CPU clocks
        runs = [sample.run() for _ in range(max(1, args.cpu_samples))]
        runs.sort(key=lambda r: r[0])
        v, parts = runs[len(runs) // 2]
        cpu = {"value": v, "unit": "ms", "cores": oracle.num_threads(), "kind": "oracle",
               "sample": sample.describe(), "stages_ms": parts,
               "spread": [runs[0][0], runs[-1][0]]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": ranks_mod.job_ms_per_call(ms_step_max, ws, split),
            "unit": "ms", "n_gpus": ws,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step_max,
            "higher_is_better": False, "scaling": "strong" if split == "heads" else "weak",
            "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic: seeded patch-coherent Gaussian mixtures at the %s shape" % w.name,
            "config": {**workload_config(w, args, ws), "density_selected": density_real},
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
