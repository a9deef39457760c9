"""Benchmark of one SVG-EAR attention layer (k-means, permute, probe, route,
block-sparse attention with compensation) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ear|reference]
                    [--workload wan|hunyuan|mid|tiny] [--no-cpu-baseline] [--no-e2e]

A step is the whole hot path over one synthetic layer whose inputs are
already resident in HBM.  The default workload is the Wan2.x-shaped layer
(40 heads, 75,600 tokens, d = 128, bf16, C_q = 100, C_k = 500, 5 k-means
iterations, density 0.10).  Inputs (2.3 GB per step) are larger than the
126 MB L2, so no explicit flush runs between steps.

N > 1 (under torchrun): every rank runs an independent layer (its own seeded
heads); no collective touches the data path.  Timing is bracketed by a
barrier and a device synchronize, and the reported time is the max over
ranks.  `value` = milliseconds per layer for the whole job = max step time /
layers processed by all ranks per step.

--impl reference times the fp64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from clustered_block_sparse_b200 import inputs as gen  # noqa: E402

METRIC = "EAR attention ms/layer & tensor-pipe % of peak, Wan-shape 75.6k tok, density 0.10"
WORKLOADS = {"tiny": gen.TINY, "mid": gen.MID, "wan": gen.WAN, "hunyuan": gen.HUNYUAN}
STAGES = ("kmeans", "permute", "probe", "route", "attention")


# --------------------------------------------------------------------------- helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"ear_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        sm = [r[0] for r in rows]
        loaded = [r[0] for r in rows if r[2] > 300.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


def flops_of(w, exact_pairs_total: int, comp_terms_total: int) -> dict:
    """Algorithmic work: QK^T and PV (2 flops per MAC each) per exact pair and per
    compensated (query, centroid) term; k-means and probe distance GEMMs."""
    d = w.d
    return {
        "attention": 4.0 * d * (exact_pairs_total + comp_terms_total),
        "exact": 4.0 * d * exact_pairs_total,
        "dense_equiv": 4.0 * d * w.n * w.n * w.heads,
        "kmeans": 2.0 * w.n * (w.c_q + w.c_k) * d * w.iters * w.heads,
        "probe": 2.0 * w.c_q * w.n * d * w.heads,
    }


def attention_bytes(w) -> float:
    """Bytes the attention step must move once: Q, K, V in and O out."""
    return 4.0 * w.heads * w.n * w.d * (2 if w.dtype == "bf16" else 4)


def stage_bytes(w, layout="permuted") -> dict:
    """Algorithmic HBM bytes of each stage (what it must move at least once):
    k-means reads Q and K once per iteration (labels are 4 bytes a row), and
    its stage also holds Q's permutation, which runs under K's k-means;
    permute reads and writes K and V (plus labels in, permutation out) --
    gathered, it reads only V (for v̄) besides the labels and permutations;
    the probe reads the keys once and writes E; the route reads E and writes
    the mask and lists; attention reads Q, K, V and writes O."""
    el = 2 if w.dtype == "bf16" else 4
    tok = w.heads * w.n * w.d * el
    rows = w.heads * w.n
    blocks = w.heads * w.c_q * w.c_k
    # Q's permutation is timed in the k-means stage (it runs under K's k-means)
    q_perm = 2 * tok + 2 * 4 * rows if layout == "permuted" else 2 * 4 * rows
    permute = (2.0 * 2 * tok + 2 * 2 * 4 * rows if layout == "permuted"
               else tok + 2 * 4 * rows + 4 * rows)
    return {
        "kmeans": 2.0 * w.iters * (tok + 4 * rows) + q_perm,
        "permute": permute,
        "probe": tok + 4.0 * blocks,
        "route": 4.0 * blocks + 1.0 * blocks + 4.0 * blocks,
        "attention": attention_bytes(w),
    }


# --------------------------------------------------------------------------- oracle arm
def oracle_sample(w, layer, query_fraction=0.05, seed=0):
    """Time the fp64 oracle on head 0: every step in full except attention,
    which runs on a seeded sample of the queries.  Returns (ms per layer
    extrapolated, seconds actually spent, description)."""
    from oracle import ear_oracle as eo

    h = 0
    q, k, v = layer.q[h], layer.k[h], layer.v[h]
    s = 1.0 / math.sqrt(w.d)
    t0 = time.perf_counter()
    qc, ql, qn = eo.kmeans(q, layer.q_init[h], w.iters)
    kc, kl, kn = eo.kmeans(k, layer.k_init[h], w.iters)
    eo.permute(ql, w.c_q)
    eo.permute(kl, w.c_k)
    vm = eo.segment_mean(v, kl, w.c_k)
    e = eo.probe(qc, qn, k, kl, kc, kn, s)
    exact, _ = eo.route(e, qn, kn, w.n, w.n, w.density)
    t1 = time.perf_counter()
    rng = np.random.default_rng(seed)
    nsel = max(1, int(round(query_fraction * w.n)))
    sel = rng.choice(w.n, nsel, replace=False)
    eo.attention(q[sel], k, v, ql[sel], kl, kc, vm, kn, exact, s)
    t2 = time.perf_counter()
    per_head = (t1 - t0) + (t2 - t1) * (w.n / nsel)
    desc = (f"head 0 of {w.heads}: k-means/permute/probe/route in full, attention on "
            f"{nsel} of {w.n} queries; extrapolated x{w.n / nsel:.1f} (attention) and "
            f"x{w.heads} (heads)")
    return per_head * w.heads * 1e3, t2 - t0, desc


def run_reference(args, w):
    from oracle import ear_oracle as eo

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    layer = gen.make_layer(w, heads=[0])
    frac = 0.02 if w.n > 50000 else 1.0
    for _ in range(args.warmup):
        oracle_sample(w, layer, frac)
    vals = []
    spent = 0.0
    desc = ""
    for i in range(args.steps):
        ms, sec, desc = oracle_sample(w, layer, frac, seed=i)
        vals.append(ms)
        spent += sec
    value = statistics.mean(vals)
    cores = eo.max_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "ms/layer",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": value,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args.gpus, args.layout, args.kmeans_streams),
        "cpu_baseline": {"value": value, "unit": "ms/layer", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "ms/layer", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def recorded_traffic(heads: int):
    """Per-launch DRAM bytes of the attention kernel from the committed ncu
    summary, scaled to `heads`, or None when the kernel source has changed
    since the capture (the counters no longer describe it)."""
    import hashlib

    here = os.path.dirname(os.path.abspath(__file__))
    prof = os.path.join(here, "profiles", "attention_tc_wan.txt")
    src = os.path.join(here, "clustered_block_sparse_b200", "csrc", "attention_tc.cu")
    try:
        text = open(prof).read()
        per_head = int(text.split("traffic_bytes_per_head:")[1].split()[0])
        sha = text.split("kernel_source_sha256:")[1].split()[0]
        cur = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except (OSError, IndexError, ValueError):
        return None
    return per_head * heads if sha == cur else None


def config_of(w, n_gpus, layout="permuted", kmeans_streams=2):
    return {"workload": w.name, "heads": w.heads, "n_q": w.n, "n_k": w.n, "d": w.d,
            "c_q": w.c_q, "c_k": w.c_k, "kmeans_iters": w.iters, "density": w.density,
            "ratio_mode": 0, "compensate": True,
            "kmeans_streams": kmeans_streams,
            "layout": ("gathered: Q, K, V stay in token order; probe and attention read rows "
                       "through the permutations (TMA tile::gather4)" if layout == "gathered"
                       else "permuted: cluster-contiguous copies of Q, K, V"),
            "l2": "inputs larger than L2 (Q, K, V per step >> 126 MB); no flush",
            "parallelism": f"{n_gpus} independent replica(s), one layer per rank, no collective"}


# --------------------------------------------------------------------------- GPU arm
def run_ear(args, w):
    import torch
    import torch.distributed as dist

    from clustered_block_sparse_b200 import _native as nat
    from clustered_block_sparse_b200 import ear, replicas

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    distributed = world > 1
    if distributed:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if distributed:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return replicas.max_over_ranks(x, device=torch.device("cuda", local))

    heads = replicas.rank_heads(rank, w.heads)
    layer = gen.make_layer(w, heads=heads)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = torch.device("cuda", local)
    q = torch.from_numpy(layer.q).to(dev, tdt)
    k = torch.from_numpy(layer.k).to(dev, tdt)
    v = torch.from_numpy(layer.v).to(dev, tdt)
    qi = torch.from_numpy(layer.q_init).to(dev)
    ki = torch.from_numpy(layer.k_init).to(dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    gathered = args.layout == "gathered"

    def step(ev=None):
        """One layer; `ev` = 6 events recorded at the stage boundaries."""
        rec = (lambda i: ev[i].record(stream)) if ev is not None else (lambda i: None)
        rec(0)
        # Q's permutation runs right after Q's k-means, under K's (timed in
        # the k-means stage)
        q_perm = lambda qc_, ql_, qn_: ear.ear_permute(ql_, w.c_q, None if gathered else q)
        (qc, ql, qn), (kc, kl, kn), (qp, qo, qx, _) = ear.ear_kmeans_pair(
            q, qi, k, ki, w.iters, streams=args.kmeans_streams, q_after=q_perm)
        rec(1)
        if gathered:
            kp, ko, _, _ = ear.ear_permute(kl, w.c_k)
            _, vm = ear.ear_permute_apply(kp, ko, v, seg_mean=True, write_perm=False)
        else:
            kp, ko, kx, _ = ear.ear_permute(kl, w.c_k, k)
            vx, vm = ear.ear_permute_apply(kp, ko, v, seg_mean=True)
        rec(2)
        e = (ear.ear_probe_gather(qc, qn, kc, k, kp, ko) if gathered
             else ear.ear_probe(qc, qn, kc, kx, ko))
        rec(3)
        exact, bo, bl, pairs = ear.ear_route(e, qn, kn, w.n, w.n, w.density)
        rec(4)
        if gathered:
            ear.ear_attention_gather(q, k, v, qo, ko, qp, kp, kc, vm, exact, bo, bl, out=out)
        else:
            ear.ear_attention(qx, kx, vx, qo, ko, qp, kc, vm, exact, bo, bl, out=out)
        rec(5)
        return exact, qo, kn, pairs

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ear.ear_get_device_status() != 0:
        raise RuntimeError("device status latched an error during warm-up")

    # algorithmic work of this layer (routing is deterministic given the inputs)
    exact, qo, kn, pairs = step()
    torch.cuda.synchronize()
    exact_h = exact.cpu().numpy().astype(np.int64)
    qsz = np.diff(qo.cpu().numpy().astype(np.int64), axis=1)
    k_sizes = kn.cpu().numpy()
    pairs_total = int(pairs.sum().item())

    # timed region: K steps with stage events, clocks sampled meanwhile
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    launches0 = nat.launch_count()
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    launches = nat.launch_count() - launches0
    total_ms = t_start.elapsed_time(t_end)
    stage_ms = {s: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                for j, s in enumerate(STAGES)}
    ms_step = max_over_ranks(total_ms / args.steps)
    if ear.ear_get_device_status() != 0:
        raise RuntimeError("device status latched an error in the timed region")

    # compensated (query, centroid) terms: |a| x (non-empty, non-exact key clusters)
    comp_terms = 0
    for h in range(exact_h.shape[0]):
        nonempty = k_sizes[h] > 0
        comp = ((exact_h[h] == 0) & nonempty[None, :]).sum(axis=1)
        comp_terms += int((qsz[h] * comp).sum())
    fl = flops_of(w, pairs_total, comp_terms)
    peaks = measured_peaks()
    attn_s = stage_ms["attention"] * 1e-3
    achieved = fl["attention"] / attn_s / 1e12
    # the attention kernel runs at full clock inside the step (see "clocks"), so
    # the burst figure is its denominator; the sustained one is reported beside it
    peak = peaks["bf16_tflops"]
    sb = stage_bytes(w, args.layout)
    hbm = {st: {"algorithmic_gb": sb[st] / 1e9,
                "achieved_gbs": sb[st] / (stage_ms[st] * 1e-3) / 1e9,
                "frac_of_measured_hbm": sb[st] / (stage_ms[st] * 1e-3) / 1e9 / peaks["hbm_gbs"]}
           for st in STAGES}

    # end to end through the public API: pinned host inputs in, output back out
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(args, w, layer, ear, dev, tdt, stream)
        e2e["value"] = max_over_ranks(e2e["value"]) / world

    line = {
        "metric": METRIC,
        "value": replicas.job_ms_per_layer(ms_step, world),
        "unit": "ms/layer",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded Gaussian-mixture / smoothed-field tokens; no model weights)",
        "config": config_of(w, world, args.layout, args.kmeans_streams),
        "stages_ms": {s: round(v, 4) for s, v in stage_ms.items()},
        "overhead_frac": (stage_ms["kmeans"] + stage_ms["probe"] + stage_ms["route"]) /
                         sum(stage_ms.values()),
        "tflops": {"attention_algorithmic": achieved,
                   "exact_blocks": fl["exact"] / attn_s / 1e12,
                   "dense_equivalent_layer": fl["dense_equiv"] / (ms_step * 1e-3) / 1e12},
        "tensor_pipe_pct_of_peak": 100.0 * achieved / peak,
        "stage_hbm": hbm,
        "roofline": {"bound": "tensor", "kernel": "ear_attention", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                     "peak_source": f"{peaks['source']} bf16 burst (MEASURED_PEAKS.json)",
                     "traffic": recorded_traffic(w.heads),
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of "
                                       "at_tc at 4 heads (profiles/attention_tc_wan.txt), "
                                       "scaled by heads; null if the kernel changed since",
                     "algorithmic_bytes": attention_bytes(w),
                     "algorithmic_flops": fl["attention"]},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import ear_oracle as eo
        base = gen.make_layer(w, heads=[0]) if w.heads > 1 else layer
        # head 0 in full (about 15-30 s of CPU work at the Wan shape), scaled by the heads
        ms, spent, desc = oracle_sample(w, base, 1.0)
        line["cpu_baseline"] = {"value": ms, "unit": "ms/layer", "cores": eo.max_threads(),
                                "kind": "oracle", "sample": desc, "cpu_seconds": spent}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if distributed:
        dist.destroy_process_group()
    return 0


def time_e2e(args, w, layer, ear, dev, tdt, stream):
    """End to end through the public API: every step copies its inputs from
    pinned host memory to the device and its output back.  Steps run the way a
    serving loop pipelines them: the next step's inputs upload on a copy stream
    and each step's output downloads on another while the compute stream works
    (two device input sets, two pinned output buffers, events between them)."""
    import torch

    host = {n: torch.from_numpy(getattr(layer, n)).to(tdt).pin_memory() for n in ("q", "k", "v")}
    host_init = {n: torch.from_numpy(getattr(layer, n)).pin_memory() for n in ("q_init", "k_init")}
    o_host = [torch.empty(host["q"].shape, dtype=tdt).pin_memory() for _ in range(2)]
    bufs = [{n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in host.items()}
            for _ in range(2)]
    ibufs = [{n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in host_init.items()}
             for _ in range(2)]
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    uploaded = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def upload(i):
        sl = i % 2
        up.wait_event(consumed[sl])  # step i-2 is done with this input set
        with torch.cuda.stream(up):
            for n in host:
                bufs[sl][n].copy_(host[n], non_blocking=True)
            for n in host_init:
                ibufs[sl][n].copy_(host_init[n], non_blocking=True)
        uploaded[sl].record(up)

    def compute(i):
        sl = i % 2
        stream.wait_event(uploaded[sl])
        with torch.cuda.stream(stream):
            res = ear.ear_layer(bufs[sl]["q"], bufs[sl]["k"], bufs[sl]["v"], ibufs[sl]["q_init"],
                                ibufs[sl]["k_init"], w.iters, w.density,
                                gather=args.layout == "gathered")
        consumed[sl].record(stream)
        down.wait_event(consumed[sl])
        with torch.cuda.stream(down):
            o_host[sl].copy_(res.o, non_blocking=True)
        res.o.record_stream(down)

    def run(n):
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)

    run(max(1, args.warmup))
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_event(a)
    run(args.steps)
    stream.wait_stream(up)
    stream.wait_stream(down)
    b.record(stream)
    torch.cuda.synchronize()
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + \
        sum(t.numel() * t.element_size() for t in host_init.values())
    d2h = o_host[0].numel() * o_host[0].element_size()
    return {"value": a.elapsed_time(b) / args.steps, "unit": "ms/layer",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "pipelining": "next step's upload and each step's download overlap compute "
                          "(separate copy streams, two input sets)"}


def run_skew_study(args):
    """Skewed cluster sizes (Zipf 1.2 mixture, Wan shape, heads 0 and 1): the
    relative L2 error against dense attention, on 4096 seeded query rows per
    head, of (i) error-routed attention with compensation (the method), (ii)
    routing by the centroid block mass P_ab = |b| e^(s q̄_a·k̄_b) / sum over b'
    with compensation, (iii) the same routing with the skipped blocks dropped,
    at each density.  All three use the same global prefix budget; the score
    key enters ear_route as E = P_ab |b|, so its E/|b| ratio is P_ab.  The
    dense reference and the score key are plain fp64 torch on the GPU
    (measurement only); every routed output comes from the library."""
    import torch

    from clustered_block_sparse_b200 import ear

    w = gen.SKEW
    heads = [0, 1]
    layer = gen.make_layer(w, heads=heads)
    dev = torch.device("cuda", 0)
    tdt = torch.bfloat16
    q = torch.from_numpy(layer.q).to(dev, tdt)
    k = torch.from_numpy(layer.k).to(dev, tdt)
    v = torch.from_numpy(layer.v).to(dev, tdt)
    qi = torch.from_numpy(layer.q_init).to(dev)
    ki = torch.from_numpy(layer.k_init).to(dev)
    s = 1.0 / math.sqrt(w.d)
    qc, ql, qn = ear.ear_kmeans(q, qi, w.iters)
    kc, kl, kn = ear.ear_kmeans(k, ki, w.iters)
    qp, qo, qx, _ = ear.ear_permute(ql, w.c_q, q)
    kp, ko, kx, _ = ear.ear_permute(kl, w.c_k, k)
    vx, vm = ear.ear_permute_apply(kp, ko, v, seg_mean=True)
    e_err = ear.ear_probe(qc, qn, kc, kx, ko)
    knd = kn.double()
    logw = s * torch.einsum("had,hbd->hab", qc.double(), kc.double()) + torch.log(knd).unsqueeze(1)
    e_score = (torch.softmax(logw, dim=2) * knd.unsqueeze(1)).float().contiguous()

    rng = np.random.default_rng(5005)
    n_rows = 4096
    rows = [torch.from_numpy(np.sort(rng.choice(w.n, n_rows, replace=False))).to(dev)
            for _ in heads]
    dense = []
    for h in range(len(heads)):
        kh, vh = k[h].double(), v[h].double()
        parts = []
        for c0 in range(0, n_rows, 512):
            qs = q[h, rows[h][c0:c0 + 512]].double()
            parts.append(torch.softmax(s * qs @ kh.T, dim=1) @ vh)
        dense.append(torch.cat(parts))
    ref_norm = math.sqrt(sum(float((d_ ** 2).sum()) for d_ in dense))

    variants = (("error_routed_compensated", e_err, True),
                ("score_routed_compensated", e_score, True),
                ("score_routed_dropped", e_score, False))
    table = {}
    for rho in gen.SKEW_DENSITIES:
        row = {}
        for name, e, comp in variants:
            exact, bo, bl, pairs = ear.ear_route(e, qn, kn, w.n, w.n, rho)
            o, _ = ear.ear_attention(qx, kx, vx, qo, ko, qp, kc, vm, exact, bo, bl,
                                     compensate=comp)
            err2 = sum(float(((o[h, rows[h]].double() - dense[h]) ** 2).sum())
                       for h in range(len(heads)))
            row[name] = math.sqrt(err2) / ref_norm
        row["exact_pair_fraction"] = float(pairs.double().sum()) / (len(heads) * w.n * w.n)
        table[f"{rho:.2f}"] = row
    if ear.ear_get_device_status() != 0:
        raise RuntimeError("device status latched an error in the study")
    print(json.dumps({"study": "skew", "workload": w.name, "heads": heads,
                      "sampled_query_rows_per_head": n_rows, "metric": "relative L2 vs dense",
                      "dense_reference": "fp64 softmax(s q K^T) V on the sampled rows",
                      "rel_l2": table}), flush=True)
    return 0


def _study_layer(w, heads, c_q=None):
    """Cluster, permute and probe one synthetic layer on the GPU (the library's
    calls); returns the tensors the quality studies route and attend with."""
    import torch

    from clustered_block_sparse_b200 import ear

    if c_q is not None:
        w = w.with_(c_q=c_q)
    layer = gen.make_layer(w, heads=heads)
    dev = torch.device("cuda", 0)
    t = torch.bfloat16
    d = {n: torch.from_numpy(getattr(layer, n)).to(dev, t) for n in ("q", "k", "v")}
    q_init = torch.from_numpy(layer.q_init).to(dev)  # C_q seeded rows of Q
    k_init = torch.from_numpy(layer.k_init).to(dev)
    L = {"w": w, **d}
    L["qc"], L["ql"], L["qn"] = ear.ear_kmeans(d["q"], q_init, w.iters)
    L["kc"], L["kl"], L["kn"] = ear.ear_kmeans(d["k"], k_init, w.iters)
    L["qp"], L["qo"], L["qx"], _ = ear.ear_permute(L["ql"], w.c_q, d["q"])
    L["kp"], L["ko"], L["kx"], _ = ear.ear_permute(L["kl"], w.c_k, d["k"])
    L["vx"], L["vm"] = ear.ear_permute_apply(L["kp"], L["ko"], d["v"], seg_mean=True)
    L["e"] = ear.ear_probe(L["qc"], L["qn"], L["kc"], L["kx"], L["ko"])
    return L


def _sampled_map_errors(L, rows, exact, lse, compensate):
    """On sampled query rows: the attention-map MSE (1/(N_q N_k)) ||A_sparse -
    A_full||_F^2 estimated over the sampled rows (SVG-EAR §5.3 "Strategy of block
    selection"), with A_sparse(i, j) = e^{z_ij - lse_i} on exact blocks,
    e^{s q_i·k̄_b(j) - lse_i} on compensated ones and 0 on dropped ones (lse from
    ear_attention); plus the dense normalizer for the same rows.  Plain fp64
    torch on the GPU: measurement only."""
    import torch

    w = L["w"]
    s = 1.0 / math.sqrt(w.d)
    err2, n_el = 0.0, 0
    for h, r in enumerate(rows):
        q = L["q"][h, r].double()
        k = L["k"][h].double()
        z = s * q @ k.T                                   # [rows, N_k]
        full = torch.softmax(z, dim=1)
        kl = L["kl"][h].long()
        ql = L["ql"][h, r].long()
        ex = exact[h][ql][:, kl].bool()                    # token-level mask
        zc = s * q @ L["kc"][h].double().T                 # [rows, C_k]
        zs = torch.where(ex, z, zc[:, kl] if compensate else torch.full_like(z, -math.inf))
        sparse = torch.exp(zs - lse[h, r].double()[:, None])
        err2 += float(((sparse - full) ** 2).sum())
        n_el += z.numel()
    return err2 / n_el


def run_fig6a_study(args):
    """Attention-map MSE against density (SVG-EAR §5.3 "Strategy of block
    selection", Fig. 6(a)) for top-p selection, top-p with compensation and
    error-aware routing with compensation, all three under the same SVG2-style
    per-query-cluster budgets (ear_topp_budget at each p).  Wan-shaped layer,
    heads 0 and 1, 1024 seeded query rows per head, at the pages' Fig. 6(a)
    setting Q_C = 300, K_C = 1000 unless --c-q / --c-k say otherwise."""
    import torch

    from clustered_block_sparse_b200 import ear

    w = gen.WAN.with_(c_q=args.c_q or 300, c_k=args.c_k or 1000)
    heads = [0, 1]
    L = _study_layer(w, heads)
    s = 1.0 / math.sqrt(w.d)
    rng = np.random.default_rng(6006)
    dev = L["q"].device
    rows = [torch.from_numpy(np.sort(rng.choice(w.n, 1024, replace=False))).to(dev) for _ in heads]
    knd = L["kn"].double()
    logw = s * torch.einsum("had,hbd->hab", L["qc"].double(), L["kc"].double())
    logw = logw + torch.log(knd).unsqueeze(1)
    mass = torch.softmax(logw, dim=2) * knd.unsqueeze(1)  # E whose E/|b| is the block mass
    e_score = mass.float().contiguous()
    # the exp-space and value-aware probes (weight-space errors) beside the logit probe
    e_w = ear.ear_probe(L["qc"], L["qn"], L["kc"], L["kx"], L["ko"], mode=1)
    e_v = ear.ear_probe(L["qc"], L["qn"], L["kc"], L["kx"], L["ko"], mode=2, v_perm=L["vx"],
                        v_centroids=L["vm"])
    table = {}
    for p in (0.5, 0.7, 0.85, 0.9, 0.95):
        budget = ear.ear_topp_budget(L["qc"], L["qn"], L["kc"], L["kn"], p)
        row = {}
        for name, e, comp in (("topp_dropped", e_score, False), ("topp_compensated", e_score, True),
                              ("error_routed_compensated", L["e"], True),
                              ("weight_error_routed_compensated", e_w, True),
                              ("value_error_routed_compensated", e_v, True)):
            exact, bo, bl, pairs = ear.ear_route_rows(e, L["qn"], L["kn"], budget)
            _, lse = ear.ear_attention(L["qx"], L["kx"], L["vx"], L["qo"], L["ko"], L["qp"],
                                       L["kc"], L["vm"], exact, bo, bl, compensate=comp,
                                       want_lse=True)
            row[name] = _sampled_map_errors(L, rows, exact, lse, comp)
        row["density"] = float(pairs.double().sum()) / (len(heads) * w.n * w.n)
        table[f"p={p}"] = row
    if ear.ear_get_device_status() != 0:
        raise RuntimeError("device status latched an error in the study")
    print(json.dumps({"study": "fig6a", "workload": w.name, "heads": heads,
                      "c_q": w.c_q, "c_k": w.c_k, "sampled_query_rows_per_head": 1024,
                      "metric": "attention-map MSE (1/(N_q N_k)) ||A_sparse - A_full||_F^2",
                      "budgets": "SVG2-style top-p per query cluster (ear_topp_budget)",
                      "mse": table}), flush=True)
    return 0


def run_clustering_study(args):
    """Clustering error and attention error against the number of query
    centroids (SVG-EAR §5.3 "Effect of clustering", Fig. 6(b)): per C_q, the
    query clustering error δ_q^2 (ear_cluster_stats), the bound's residual
    8 δ_q^2 K_max^2 / (N_k d), the attention-map MSE on 1024 sampled rows per
    head and the average normalizer change against dense attention (§5.1), at
    top-p budgets with p = 0.85 (the pages' setting, whose density moves with
    C_q) and at a fixed density 0.10.  Wan-shaped layer, heads 0 and 1, at the
    pages' Fig. 6(b) setting K_C = 1000 unless --c-k says otherwise."""
    import torch

    from clustered_block_sparse_b200 import ear

    w = gen.WAN.with_(c_k=args.c_k or 1000)
    heads = [0, 1]
    table = {}
    rng = np.random.default_rng(6007)
    rows = None
    for c_q in (25, 50, 100, 200, 300):
        L = _study_layer(w, heads, c_q=c_q)
        ww = L["w"]
        dev = L["q"].device
        if rows is None:
            rows = [torch.from_numpy(np.sort(rng.choice(w.n, 1024, replace=False))).to(dev)
                    for _ in heads]
        dq, _ = ear.ear_cluster_stats(L["q"], L["ql"], L["qc"])
        _, kmax = ear.ear_cluster_stats(L["k"], L["kl"], L["kc"])
        full = torch.ones((len(heads), ww.c_q, ww.c_k), dtype=torch.uint8, device=dev)
        fo = torch.arange(0, (ww.c_q + 1) * ww.c_k, ww.c_k, device=dev, dtype=torch.int32)
        fo = fo.unsqueeze(0).expand(len(heads), -1).contiguous()
        fl = torch.arange(ww.c_k, device=dev, dtype=torch.int32).repeat(ww.c_q)
        fl = fl.unsqueeze(0).expand(len(heads), -1).contiguous()
        _, lse_dense = ear.ear_attention(L["qx"], L["kx"], L["vx"], L["qo"], L["ko"], L["qp"],
                                         L["kc"], L["vm"], full, fo, fl, want_lse=True)
        entry = {"delta_q_sq": [float(x) for x in dq.cpu()],
                 "bound_residual": [float(x) for x in
                                    ear.bound_residual(dq, kmax, w.n, w.d).cpu()]}
        e_v = ear.ear_probe(L["qc"], L["qn"], L["kc"], L["kx"], L["ko"], mode=2, v_perm=L["vx"],
                            v_centroids=L["vm"])
        topp = ear.ear_topp_budget(L["qc"], L["qn"], L["kc"], L["kn"], 0.85)
        dens = ear.ear_uniform_budget(L["qn"], w.n, 0.10)
        arms = (("topp_0.85", L["e"], topp), ("density_0.10", L["e"], dens),
                ("value_topp_0.85", e_v, topp), ("value_density_0.10", e_v, dens))
        for name, e, budget in arms:
            exact, bo, bl, pairs = ear.ear_route_rows(e, L["qn"], L["kn"], budget)
            _, lse = ear.ear_attention(L["qx"], L["kx"], L["vx"], L["qo"], L["ko"], L["qp"],
                                       L["kc"], L["vm"], exact, bo, bl, want_lse=True)
            change = ear.ear_normalizer_change(lse, lse_dense)
            entry[name] = {"attention_map_mse": _sampled_map_errors(L, rows, exact, lse, True),
                           "normalizer_change": [float(x) for x in change.cpu()],
                           "density": float(pairs.double().sum()) / (len(heads) * w.n * w.n)}
        table[f"C_q={c_q}"] = entry
    if ear.ear_get_device_status() != 0:
        raise RuntimeError("device status latched an error in the study")
    print(json.dumps({"study": "clustering", "workload": w.name, "heads": heads, "c_k": w.c_k,
                      "budgets": "per query cluster: top-p with p = 0.85, and the share of "
                                 "density 0.10; routed on the logit probe, and (value_*) on the "
                                 "value-aware probe", "by_c_q": table}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ear", "reference"), default="ear")
    ap.add_argument("--workload", choices=tuple(WORKLOADS), default="wan")
    ap.add_argument("--heads", type=int, default=None,
                    help="override the head count (smaller profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--study", choices=("skew", "fig6a", "clustering"), default=None,
                    help="run a quality study instead of the timing line")
    ap.add_argument("--c-q", type=int, default=None, help="query clusters of a study")
    ap.add_argument("--c-k", type=int, default=None, help="key clusters of a study")
    ap.add_argument("--kmeans-streams", type=int, choices=(1, 2), default=2,
                    help="Q's and K's k-means one after the other (1) or side by side (2)")
    ap.add_argument("--layout", choices=("permuted", "gathered"), default="permuted",
                    help="permuted copies of Q, K, V, or reads through the permutations")
    args = ap.parse_args(argv)
    if args.study == "skew":
        return run_skew_study(args)
    if args.study == "fig6a":
        return run_fig6a_study(args)
    if args.study == "clustering":
        return run_clustering_study(args)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.heads is not None and args.heads != w.heads:
        w = w.with_(heads=args.heads, name=f"{w.name.split('-')[0]}-shape-{args.heads}head-"
                    f"N{w.n}-d{w.d}-{w.dtype}")
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ear(args, w)


if __name__ == "__main__":
    sys.exit(main())
