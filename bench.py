"""Benchmark: one sparse 3D-attention call per step on the HunyuanVideo-shaped
workload (B=1, H=24, N=33 latent frames x F=3600 tokens, L=118800, d=128,
bf16, a1=3 / a2=281 for ~15% mask density, S=128 sampled profiling rows).

A step is the whole hot path through the C ABI: online profiling ->
token-major permutation of temporal heads -> block-sparse attention ->
inverse permutation.  Inputs are synthetic (seeded generator with the
workload's shape and head structure) and resident in HBM; they are larger
than L2 (3 x 730 MB), so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  value = ms per call for the whole job
(max-over-ranks step time divided by the calls all ranks made; each rank runs
its own independent call, so scaling is weak).  N > 1 runs under torchrun.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_video_profile_b200 import metrics, synth  # noqa: E402

METRIC = "ms per sparse 3D-attention call; effective TFLOPS vs bf16 peak; speedup vs dense"

# DRAM bytes (read + write) per full-size launch of the attention kernel, from
# an ncu capture of a 4-head case of the same shape scaled by heads (the
# "-blhd" entry: of the full launch itself), keyed by
# the sha256 prefix of the kernel sources it was taken on and by the layout
# (fused or separate, "-blhd" appended for [B, L, H, d] tensors).  Any other
# revision or layout reports traffic as null until it is captured again.
NCU_TRAFFIC = {("645b18066bbc1e1a", "d2f4abb45748fc0c", "fused"): 2.8525e9,
               ("20c87c577a0d9af9", "5edc1f6588b2c178", "fused"): 2.8583e9,
               ("239a7b5e36619c63", "3c4a90062d61487f", "fused"): 2.8442e9,
               ("239a7b5e36619c63", "3c4a90062d61487f", "separate-blhd"): 2.9109e9}


# The same for the profiling stage-1 kernel (full HunyuanVideo launch), keyed by
# the sha256 prefix of its source.
PROF_NCU_TRAFFIC = {"5732be8477404d60": 1.488e9, "a5d1bd300122e4a1": 1.4840e9, "cabba81d0b39bcb9": 1.4901e9,
                    "cfcfb262609a7c06": 1.4874e9}


def prof_source_key():
    import hashlib
    path = os.path.join(ROOT, "sparse_attention_video_profile_b200", "csrc", "profile_sm100.cu")
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def attn_source_key():
    import hashlib
    csrc = os.path.join(ROOT, "sparse_attention_video_profile_b200", "csrc")
    return tuple(hashlib.sha256(open(os.path.join(csrc, f), "rb").read()).hexdigest()[:16]
                 for f in ("attn_sm100.cu", "sm100.cuh"))
# kernels one bf16 profiling call launches: tcgen05 stage 1, row combine, per-head finalize
PROFILE_LAUNCHES = 3
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# dense tf32 / bf16 tensor throughput, nominal (1.1 / 2.25 PFLOP/s per B200)
TF32_PER_BF16 = 1.1 / 2.25
TF32_PEAK_NOTE = " x 1.1/2.25 (nominal tf32 / bf16 ratio)"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- distributed plumbing

def dist_setup(n_gpus):
    if n_gpus <= 1 and "WORLD_SIZE" not in os.environ:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (device timings are combined this way:
    the job is as slow as its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_call(step_ms_per_rank: float, world: int) -> float:
    """Whole-job ms per call: every rank runs one independent call per step, so
    the job completes `world` calls in the slowest rank's step time."""
    return max_over_ranks(step_ms_per_rank, world) / world


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of this GPU's SM clock and throttle reasons while
    the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            ident = str(device_index)
        self.cmd = ["nvidia-smi", "-i", ident, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "200"]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unsampled"], "samples": 0}
        # median over the samples taken under load (the top half of clocks
        # excludes idle gaps at the edges of the window)
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU baseline (oracle)

def head_f64(wl, q, k, v, h=0):
    """fp64 host copies of one head's q, k, v ([1, 1, L, d]) for the oracle."""
    return tuple(t[:, h:h + 1].to("cpu", torch.float64).numpy() for t in (q, k, v))


def oracle_sample(wl, qkv64, rows_np, labels, n_prof_rows=16, n_attn_rows=16, seed=0):
    """Times the fp64 oracle, as it stands, on a bounded sample of one call
    and scales the time linearly to the whole call: profiling of
    n_prof_rows sampled rows of one head (the call profiles S rows of every
    head) and masked attention of n_attn_rows query rows of one head (the
    call computes all L rows of every head).
    Returns (ms_per_call_estimate, description, seconds_spent)."""
    import oracle  # test infrastructure: only this baseline leg runs it
    rng = np.random.default_rng(seed)
    qn, kn, vn = qkv64
    prof_rows = np.sort(rng.choice(rows_np, n_prof_rows, replace=False))
    t0 = time.perf_counter()
    oracle.profile_heads(qn, kn, vn, wl.N, wl.F, wl.a1, wl.a2, prof_rows)
    t_prof = time.perf_counter() - t0
    sample = np.sort(rng.choice(wl.L, n_attn_rows, replace=False))
    t0 = time.perf_counter()
    oracle.sparse_attention(qn, kn, vn, labels[:, :1], wl.N, wl.F, wl.a1, wl.a2, rows=sample)
    t_attn = time.perf_counter() - t0
    heads = wl.B * wl.H
    per_call_s = t_prof * (wl.S / n_prof_rows) * heads + t_attn * (wl.L / n_attn_rows) * heads
    desc = (f"fp64 oracle: profiling of {n_prof_rows} of the {wl.S} sampled rows and masked attention of "
            f"{n_attn_rows} of the {wl.L} query rows, both on 1 of the {heads} heads, scaled linearly to the call")
    return per_call_s * 1e3, desc, t_prof + t_attn


def oracle_sample_svg2(wl, qkv64, n_attn_rows=16, seed=0):
    """The fp64 oracle on a bounded sample of one SVG2-style call, scaled
    linearly: one Lloyd round of k-means of one head's Q and of its K (the
    call runs `iters` rounds of both on every head), the centroid top-p of
    that head, and the masked attention of n_attn_rows of its query rows.
    Returns (ms_per_call_estimate, description, seconds_spent)."""
    import oracle  # test infrastructure: only this baseline leg runs it
    prm = synth.SVG2_PARAMS
    qn, kn, vn = (x[0, 0] for x in qkv64)
    t0 = time.perf_counter()
    aq, mu_q, _ = oracle.kmeans(qn, prm["Cq"], 1)
    ak, mu_k, n_k = oracle.kmeans(kn, prm["Ck"], 1)
    t_km = time.perf_counter() - t0
    t0 = time.perf_counter()
    sel = oracle.centroid_topp(mu_q, mu_k, n_k, prm["p"])
    t_sel = time.perf_counter() - t0
    rows = np.sort(np.random.default_rng(seed).choice(wl.L, n_attn_rows, replace=False))
    t0 = time.perf_counter()
    oracle.svg2_attention_given(qn, kn, vn, aq, ak, sel, rows=rows)
    t_attn = time.perf_counter() - t0
    heads = wl.B * wl.H
    per_call_s = (t_km * prm["iters"] + t_sel) * heads + t_attn * (wl.L / n_attn_rows) * heads
    desc = (f"fp64 oracle: one k-means round of Q ({prm['Cq']}) and K ({prm['Ck']}) clusters, the top-p selection, "
            f"and the attention of {n_attn_rows} of the {wl.L} query rows, all on 1 of the {heads} heads, scaled "
            f"linearly to the call ({prm['iters']} rounds, all rows and heads)")
    return per_call_s * 1e3, desc, t_km + t_sel + t_attn


def step_spread(step_events, names):
    """p10 / median / p90 of the per-call device time (first kernel's start
    to the last kernel's end of each timed call)."""
    t = np.array([e[names[0]][0].elapsed_time(e[names[-1]][1]) for e in step_events])
    return {"p10": float(np.percentile(t, 10)), "p50": float(np.median(t)), "p90": float(np.percentile(t, 90))}


def cpu_cores():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------- arms

def run_reference(args, wl, rank, world):
    """The oracle on the host cores, on a bounded sample of the workload per
    step (rank 0 only)."""
    if rank != 0:
        return
    q, k, v = synth.make_qkv(wl, seed=0, device="cpu")
    rows_np = synth.sample_rows(wl.L, wl.S, 0)
    labels = synth.head_kinds(wl, 0)
    qkv64 = head_f64(wl, q, k, v)
    del q, k, v
    svg2 = wl.name == "svg2"
    for w in range(args.warmup):
        if svg2:
            oracle_sample_svg2(wl, qkv64, n_attn_rows=4, seed=1000 + w)
        else:
            oracle_sample(wl, qkv64, rows_np, labels, n_prof_rows=4, n_attn_rows=4, seed=1000 + w)
    ests, secs = [], 0.0
    desc = ""
    for s in range(args.steps):
        if svg2:
            ms, desc, sec = oracle_sample_svg2(wl, qkv64, n_attn_rows=32, seed=s)
        else:
            ms, desc, sec = oracle_sample(wl, qkv64, rows_np, labels, n_prof_rows=32, n_attn_rows=64, seed=s)
        ests.append(ms)
        secs += sec
    value = float(np.mean(ests))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "ms/call", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": value, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(wl, world, args.shard),
        "cpu_baseline": {"value": value, "unit": "ms/call", "cores": cpu_cores(), "kind": "oracle",
                         "sample": desc + " (per step)"},
        "e2e": {"value": value, "unit": "ms/call", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(wl, world, shard="replicas"):
    shape_name = "mixed sparse-pattern" if wl.name.startswith("mixed") else "HunyuanVideo-shaped"
    return {"workload": f"{shape_name} {wl.name}: B={wl.B} H={wl.H} N={wl.N} F={wl.F} L={wl.L} d={wl.d}",
            "B": wl.B, "H": wl.H, "N": wl.N, "F": wl.F, "L": wl.L, "d": wl.d, "a1": wl.a1, "a2": wl.a2, "S": wl.S,
            "global_batch": wl.B * (world if shard == "replicas" else 1), "seq_len": wl.L,
            "parallelism": f"{shard}{world}" if world > 1 else "single",
            "l2": f"inputs larger than L2 (Q,K,V 3 x {wl.B * wl.H * wl.L * wl.d * 2 / 1e6:.0f} MB); no flush"}


def s2_computed_pairs(cid_sorted, keep, nk, rows_per_cta=256, bk=128):
    """(query, key) pairs the cluster-pair attention kernel computes for one
    head: each CTA of 256 cluster-sorted query rows walks the union of the key
    clusters its query clusters keep, as runs of consecutive kept clusters in
    the cluster-sorted key order (empty clusters do not break a run), in
    128-key tiles; every tile is computed for all 256 rows."""
    ne = nk > 0
    sizes = nk[ne]
    csum = np.concatenate(([0], np.cumsum(sizes)))
    total = 0
    L = cid_sorted.shape[0]
    for q0 in range(0, L, rows_per_cta):
        c0, c1 = cid_sorted[q0], cid_sorted[min(q0 + rows_per_cta, L) - 1]
        u = keep[c0:c1 + 1].any(axis=0)[ne].astype(np.int8)
        edges = np.diff(np.concatenate(([0], u, [0])))
        starts, ends = np.flatnonzero(edges == 1), np.flatnonzero(edges == -1)
        lens = csum[ends] - csum[starts]
        total += int(((lens + bk - 1) // bk).sum()) * bk * rows_per_cta
    return total


def run_svg2(args, wl, rank, world, local):
    """One SVG2-style call per step on the HunyuanVideo shape: k-means of Q
    and of K, then the semantic-aware attention (sort, gathers, centroids,
    top-p, attention)."""
    from sparse_attention_video_profile_b200 import svg
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    prm = synth.SVG2_PARAMS
    Cq, Ck, iters, p = prm["Cq"], prm["Ck"], prm["iters"], prm["p"]
    q, k, v = synth.make_qkv(wl, seed=rank, device=dev)
    N, F, L = wl.N, wl.F, wl.L
    shape = svg.make_shape(q, N, F)
    o = torch.empty_like(q)
    aq = torch.empty(wl.B, wl.H, L, dtype=torch.int32, device=dev)
    ak = torch.empty_like(aq)
    cq = torch.empty(wl.B, wl.H, Cq, wl.d, dtype=torch.float32, device=dev)
    ck = torch.empty(wl.B, wl.H, Ck, wl.d, dtype=torch.float32, device=dev)
    sel = torch.empty(wl.B, wl.H, Cq, (Ck + 31) // 32, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    km_ws = svg.alloc_workspace(max(svg.lib.svg_kmeans_workspace_size(svg.ctypes.byref(shape), Cq),
                                    svg.lib.svg_kmeans_workspace_size(svg.ctypes.byref(shape), Ck)), dev)
    at_ws = svg.alloc_workspace(svg.lib.svg_semantic_attn_workspace_size(svg.ctypes.byref(shape), Cq, Ck), dev)
    names = ("kmeans_q", "kmeans_k", "attn")

    def step(e=None):
        def mark(n, i):
            if e:
                e[n][i].record(stream)
        mark("kmeans_q", 0)
        svg.svg_kmeans(q, N, F, Cq, iters, assign=aq, centroids=cq, workspace=km_ws, status=status)
        mark("kmeans_q", 1)
        mark("kmeans_k", 0)
        svg.svg_kmeans(k, N, F, Ck, iters, assign=ak, centroids=ck, workspace=km_ws, status=status)
        mark("kmeans_k", 1)
        mark("attn", 0)
        svg.svg_semantic_attn(q, k, v, N, F, aq, ak, Cq, Ck, p, o=o, selected=sel, workspace=at_ws, status=status)
        mark("attn", 1)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # unmasked pairs: sum over query clusters of |c_q| x |kept keys|
    bits = svg.selected_bits(sel, Ck)
    aq_np, ak_np = aq.cpu().numpy(), ak.cpu().numpy()
    pairs = 0
    computed = 0
    for b in range(wl.B):
        for h in range(wl.H):
            nq = np.bincount(aq_np[b, h], minlength=Cq)
            nk = np.bincount(ak_np[b, h], minlength=Ck)
            pairs += int((nq * (bits[b, h] @ nk)).sum())
            computed += s2_computed_pairs(np.sort(aq_np[b, h]), bits[b, h].astype(bool), nk)
    density = pairs / (wl.B * wl.H * float(L) * L)
    flops = metrics.attention_flops(pairs, wl.d)
    step_events = [{n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in names}
                   for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t_start.record(stream)
        for e in step_events:
            step(e)
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status word {int(status.item())} after the timed region")
    kern_ms = {n: sum(e[n][0].elapsed_time(e[n][1]) for e in step_events) / args.steps for n in names}
    spread = step_spread(step_events, names)
    step_ms = max_over_ranks(t_start.elapsed_time(t_end) / args.steps, world)
    value = step_ms / world
    dense_ms = None
    if not args.no_dense:
        od = torch.empty_like(q)
        svg.svg_dense_attn(q, k, v, N, F, o=od)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(2):
            svg.svg_dense_attn(q, k, v, N, F, o=od)
        b.record(stream)
        torch.cuda.synchronize()
        dense_ms = a.elapsed_time(b) / 2
        del od
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ms, desc, _ = oracle_sample_svg2(wl, head_f64(wl, q, k, v), n_attn_rows=32)
        cpu = {"value": ms, "unit": "ms/call", "cores": cpu_cores(), "kind": "oracle", "sample": desc}
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    attn_tflops = flops / (kern_ms["attn"] * 1e-3) / 1e12
    km_flops = 2.0 * wl.B * wl.H * L * wl.d * (Cq + Ck) * iters  # distance products of all rounds
    km_tflops = km_flops / ((kern_ms["kmeans_q"] + kern_ms["kmeans_k"]) * 1e-3) / 1e12
    line = {
        "metric": "ms per SVG2-style sparse attention call (k-means of Q and K, top-p, attention)",
        "value": value, "unit": "ms/call", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dict(config_dict(wl, world), Cq=Cq, Ck=Ck, iters=iters, p=p),
        "kernel_ms": kern_ms, "call_ms_spread": spread, "density": density,
        "computed_pairs": computed, "tile_efficiency": pairs / computed if computed else None,
        "effective_tflops_attn_stage": attn_tflops,
        "kmeans_tflops": km_tflops,
        "speedup_vs_dense": (dense_ms / step_ms) if dense_ms else None, "dense_ms": dense_ms,
        "roofline": {"bound": "tensor", "kernel": "attn_sm100_kernel<128, cluster-pair> stage (with sort, gathers, "
                     "centroids, top-p)", "achieved": attn_tflops, "peak": peak,
                     "peak_kind": f"{peak_kind} bf16_tflops (burst)", "unit": "TFLOP/s", "frac": attn_tflops / peak,
                     "peak_sustained": peak_sus, "frac_sustained": attn_tflops / peak_sus,
                     "traffic": None, "algorithmic_work": f"{flops:.4e} flops = 4*d*kept pairs"},
        "clocks": clocks.summary(),
        "e2e": None,
        "gpu_launches": (2 * (1 + 5 * iters) + 13) * args.steps,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def time_calls(fn, reps, stream, warm=2):
    """Mean device time (ms) of `reps` back-to-back calls of fn on `stream`,
    after `warm` untimed calls (CUDA events on the launching stream)."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def measure_config(wl, dev, stream, peak, seed=0, steps=5, warm=2, layout="bhld"):
    """One workload timed outside the headline's timed region: the whole call
    step by step (profile -> attention with the layout the call picks, or
    permute -> attention -> unpermute), CUDA events around each stage, on
    [B, H, L, d] tensors or (layout "blhd") [B, L, H, d] ones.  Returns ms per
    call, attention-kernel ms, effective TFLOPS and the fraction of the bf16
    peak."""
    from sparse_attention_video_profile_b200 import svg
    q, k, v = synth.make_qkv(wl, seed=seed, device=dev)
    if layout == "blhd":
        q, k, v = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    rows = torch.from_numpy(synth.sample_rows(wl.L, wl.S, seed)).to(dev)
    N, F = wl.N, wl.F
    shape = svg.make_shape(q, N, F, layout=layout)
    lk = {"layout": layout}  # every call of this config
    o = torch.empty_like(q)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    mixed = wl.name.startswith("mixed")
    prm = synth.MIXED_PARAMS
    band = prm["md_half"] + 1 if mixed else wl.a2
    fused = svg.svg_sparse_3d_attn_plan(shape, band)[2]
    if mixed:
        modes_np = synth.head_modes(wl.B, wl.H, seed)
        mode = torch.from_numpy(modes_np).to(dev)
        md_label = torch.from_numpy((modes_np == 3).astype(np.int8)).to(dev)
    else:
        mse = torch.empty(wl.B, wl.H, 2, dtype=torch.float32, device=dev)
        label = torch.empty(wl.B, wl.H, dtype=torch.int8, device=dev)
        prof_ws = svg.alloc_workspace(svg.svg_profile_workspace_size(shape, wl.S), dev)
    if not fused:
        qp, kp, vp, op = (torch.empty_like(q) for _ in range(4))

    def step(ev):
        ev[0].record(stream)
        if not mixed:
            svg.svg_profile_heads(q, k, v, N, F, wl.a1, wl.a2, rows, mse=mse, label=label, workspace=prof_ws, **lk)
        lab = md_label if mixed else label
        if not fused:
            svg.svg_permute_qkv(q, k, v, N, F, lab, out=(qp, kp, vp), **lk)
        ev[1].record(stream)
        if mixed and fused:
            svg.svg_mixed_attn_fused(q, k, v, mode, N, F, prm["window"], prm["md_half"], prm["stripe"], o=o,
                                     status=status, **lk)
        elif mixed:
            svg.svg_mixed_attn(q, k, v, qp, kp, vp, mode, N, F, prm["window"], prm["md_half"], prm["stripe"], o=o,
                               op=op, status=status, **lk)
        elif fused:
            svg.svg_block_sparse_attn_fused(q, k, v, label, N, F, wl.a1, wl.a2, o=o, status=status, **lk)
        else:
            svg.svg_block_sparse_attn(q, k, v, qp, kp, vp, label, N, F, wl.a1, wl.a2, o=o, op=op, status=status, **lk)
        ev[2].record(stream)
        if not fused:
            svg.svg_unpermute(op, N, F, lab, out=o, **lk)
        ev[3].record(stream)

    def events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    for _ in range(warm):
        step(events())
    torch.cuda.synchronize()
    evs = [events() for _ in range(steps)]
    for ev in evs:
        step(ev)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status word {int(status.item())} in the {wl.name} config")
    call_ms = float(np.mean([ev[0].elapsed_time(ev[3]) for ev in evs]))
    attn_ms = float(np.mean([ev[1].elapsed_time(ev[2]) for ev in evs]))
    if mixed:
        pairs = metrics.mixed_pairs(N, F, modes_np, prm["window"], prm["md_half"], prm["stripe"])
    else:
        pairs = metrics.effective_pairs(N, F, wl.a1, wl.a2, label.cpu().numpy())
    tflops = metrics.attention_flops(pairs, wl.d) / (attn_ms * 1e-3) / 1e12
    tag = "" if layout == "bhld" else " [B, L, H, d]"
    return {"workload": f"{wl.name}{tag}: B={wl.B} H={wl.H} N={N} F={F} L={wl.L} d={wl.d} a1={wl.a1} a2={wl.a2}",
            "ms": call_ms, "attn_ms": attn_ms, "effective_tflops": tflops, "frac_bf16_peak": tflops / peak,
            "density": pairs / (wl.B * wl.H * float(wl.L) * wl.L),
            "layout": "fused" if fused else "separate", "steps": steps}


def run_ours(args, wl, rank, world, local):
    from sparse_attention_video_profile_b200 import svg
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    # N > 1: every rank takes its block of the heads of ONE call (the head
    # partition of svg_head_shard, as svg_sparse_3d_attn_shard runs it: views
    # of the block, no copies), or with --shard replicas runs its own call
    shard_heads = world > 1 and args.shard == "heads"
    tl = args.tensor_layout
    if shard_heads and tl != "bhld":
        raise SystemExit("--tensor-layout blhd runs one call per rank: use --shard replicas for N > 1")
    lk = {"layout": tl}  # every call of the step on the same tensor layout
    tf32 = args.precision == "tf32"
    ak = dict(lk, tf32=True) if tf32 else lk  # attention calls: fp32 tensors through the tf32 tensor cores
    if tf32 and (shard_heads or wl.name.startswith("mixed")):
        raise SystemExit("--precision tf32 runs the spatial / temporal call on one GPU (or replicas)")
    job_wl = wl
    if shard_heads:
        import dataclasses
        n_heads = wl.B * wl.H
        first, count = svg.svg_head_shard(n_heads, rank, world)
        if count == 0:
            raise SystemExit(f"--shard heads needs at least one head per rank ({n_heads} heads, {world} ranks)")
        q, k, v = (t.view(n_heads, wl.L, wl.d)[first:first + count].view(1, count, wl.L, wl.d)
                   for t in synth.make_qkv(wl, seed=0, device=dev))
        wl = dataclasses.replace(wl, B=1, H=count)
        rows_np = synth.sample_rows(wl.L, wl.S, 0)
    else:
        q, k, v = synth.make_qkv(wl, seed=rank, device=dev)
        rows_np = synth.sample_rows(wl.L, wl.S, rank)
    if tl == "blhd":  # [B, L, H, d]: the same values, heads inside the token axis
        q, k, v = (t.transpose(1, 2).contiguous() for t in (q, k, v))
    if tf32:  # the same values as fp32 tensors
        q, k, v = (t.float().contiguous() for t in (q, k, v))
    es = q.element_size()
    rows = torch.from_numpy(rows_np).to(dev)
    N, F = wl.N, wl.F
    o = torch.empty_like(q)
    # token-major copies: only the separate layout path needs them
    qp = kp = vp = op = None
    mse = torch.empty(wl.B, wl.H, 2, dtype=torch.float32, device=dev)
    label = torch.empty(wl.B, wl.H, dtype=torch.int8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    shape = svg.make_shape(q, N, F, layout=tl, tf32=tf32)
    prof_ws = svg.alloc_workspace(svg.svg_profile_workspace_size(shape, wl.S), dev)

    mixed = wl.name.startswith("mixed")
    if mixed:
        prm = synth.MIXED_PARAMS
        modes_np = synth.head_modes(wl.B, wl.H, rank)
        mode = torch.from_numpy(modes_np).to(dev)
    # layout of token-major heads; auto = the whole call's own choice
    band = prm["md_half"] + 1 if mixed else wl.a2
    plan_sep, plan_fused, plan_choice = svg.svg_sparse_3d_attn_plan(shape, band)
    fused = plan_choice if args.layout == "auto" else args.layout == "fused"
    if not fused:
        qp, kp, vp, op = (torch.empty_like(q) for _ in range(4))
    if mixed:
        names = ("attn",) if fused else ("permute", "attn", "unpermute")
    else:
        names = ("profile", "attn") if fused else ("profile", "permute", "attn", "unpermute")

    def new_events():
        return {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in names}

    def step_mixed(e=None):
        if fused:
            if e:
                e["attn"][0].record(stream)
            svg.svg_mixed_attn_fused(q, k, v, mode, N, F, prm["window"], prm["md_half"], prm["stripe"], o=o,
                                     status=status, **lk)
            if e:
                e["attn"][1].record(stream)
            return
        if e:
            e["permute"][0].record(stream)
        svg.svg_permute_qkv(q, k, v, N, F, md_label, out=(qp, kp, vp), **lk)
        if e:
            e["permute"][1].record(stream)
            e["attn"][0].record(stream)
        svg.svg_mixed_attn(q, k, v, qp, kp, vp, mode, N, F, prm["window"], prm["md_half"], prm["stripe"], o=o,
                           op=op, status=status, **lk)
        if e:
            e["attn"][1].record(stream)
            e["unpermute"][0].record(stream)
        svg.svg_unpermute(op, N, F, md_label, out=o, **lk)
        if e:
            e["unpermute"][1].record(stream)

    def step(e=None):
        if mixed:
            return step_mixed(e)
        if e:
            e["profile"][0].record(stream)
        svg.svg_profile_heads(q, k, v, N, F, wl.a1, wl.a2, rows, mse=mse, label=label, workspace=prof_ws, **lk)
        if fused:
            if e:
                e["profile"][1].record(stream)
                e["attn"][0].record(stream)
            svg.svg_block_sparse_attn_fused(q, k, v, label, N, F, wl.a1, wl.a2, o=o, status=status, **ak)
            if e:
                e["attn"][1].record(stream)
            return
        if e:
            e["profile"][1].record(stream)
            e["permute"][0].record(stream)
        svg.svg_permute_qkv(q, k, v, N, F, label, out=(qp, kp, vp), **lk)
        if e:
            e["permute"][1].record(stream)
            e["attn"][0].record(stream)
        svg.svg_block_sparse_attn(q, k, v, qp, kp, vp, label, N, F, wl.a1, wl.a2, o=o, op=op, status=status, **ak)
        if e:
            e["attn"][1].record(stream)
            e["unpermute"][0].record(stream)
        svg.svg_unpermute(op, N, F, label, out=o, **lk)
        if e:
            e["unpermute"][1].record(stream)

    if mixed:
        # heads that run on token-major copies (label 1 for the permute calls)
        md_label = torch.from_numpy((modes_np == 3).astype(np.int8)).to(dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if mixed:
        labels_np = (modes_np == 3).astype(np.int8)
        pairs = metrics.mixed_pairs(N, F, modes_np, prm["window"], prm["md_half"], prm["stripe"])
    else:
        labels_np = label.cpu().numpy()
        pairs = metrics.effective_pairs(N, F, wl.a1, wl.a2, labels_np)
    n_temporal = int(labels_np.sum())
    flops = metrics.attention_flops(pairs, wl.d)

    step_events = [new_events() for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        t_start.record(stream)
        for e in step_events:
            step(e)
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    acc = {n: sum(e[n][0].elapsed_time(e[n][1]) for e in step_events) for n in names}
    spread = step_spread(step_events, names)
    step_ms_local = t_start.elapsed_time(t_end) / args.steps
    if int(status.item()) != 0:
        raise RuntimeError(f"device status word {int(status.item())} after the timed region")
    step_ms = max_over_ranks(step_ms_local, world)
    kern_ms = {n: acc[n] / args.steps for n in acc}
    # ms per call, whole job: head shards finish one call per step (the
    # slowest rank's step); replicas finish `world` calls per step
    value = step_ms if shard_heads else step_ms / world

    # dense reference on the same inputs (speedup vs dense), outside the timed region
    dense_ms = None
    if not args.no_dense:
        od = torch.empty_like(q)
        svg.svg_dense_attn(q, k, v, N, F, o=od, **ak)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 2
        a.record(stream)
        for _ in range(reps):
            svg.svg_dense_attn(q, k, v, N, F, o=od, **ak)
        b.record(stream)
        torch.cuda.synchronize()
        dense_ms = a.elapsed_time(b) / reps
        del od

    # offline mode search of the mixed patterns on the same inputs (run once per
    # model, not part of the call), outside the timed region
    mode_search = None
    if mixed:
        ms_ws = svg.alloc_workspace(int(svg.lib.svg_mode_search_workspace_size(svg.ctypes.byref(shape), wl.S)), dev)
        ms_loss = torch.empty(wl.B, wl.H, 4, dtype=torch.float32, device=dev)
        ms_mode = torch.empty(wl.B, wl.H, dtype=torch.int8, device=dev)

        def search():
            svg.svg_mode_search(q, k, v, N, F, rows, prm["window"], prm["md_half"], prm["stripe"], loss=ms_loss,
                                mode=ms_mode, workspace=ms_ws, **lk)

        search()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        a.record(stream)
        for _ in range(reps):
            search()
        b.record(stream)
        torch.cuda.synchronize()
        t_ms = a.elapsed_time(b) / reps
        kv_bytes = 2 * 2 * wl.B * wl.H * wl.L * wl.d * 2  # K and V read by each of the two passes
        counts = np.bincount(ms_mode.cpu().numpy().reshape(-1).astype(np.int64) + 1, minlength=6)
        mode_search = {"ms": t_ms, "kv_gbs": kv_bytes / (t_ms * 1e-3) / 1e9, "lambda": 0.5, "epsilon": 1.0,
                       "modes_chosen": {nm: int(c) for nm, c in zip(
                           ("failed", "full", "skip", "diagonal", "multidiag", "stripe"), counts)}}
        del ms_ws

    # end to end through the public call with host buffers
    e2e = None
    if not args.no_e2e and not mixed and tl == "bhld":  # the host-buffer call takes [B, H, L, d]
        # host tensors (page-locked); the call pipelines its own copies
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        mseh = torch.empty(mse.shape, dtype=mse.dtype, pin_memory=True)
        labh = torch.empty(label.shape, dtype=label.dtype, pin_memory=True)
        rowsh = torch.from_numpy(rows_np).pin_memory()
        need = int(svg.lib.svg_sparse_3d_attn_host_workspace_size(svg.ctypes.byref(shape), wl.a2, wl.S, args.e2e_chunk))
        ws_host_call = svg.alloc_workspace(need, dev)

        def e2e_step():
            svg.svg_sparse_3d_attn_host(qh, kh, vh, N, F, wl.a1, wl.a2, rowsh, o=oh, mse=mseh, label=labh,
                                        heads_per_chunk=args.e2e_chunk, workspace=ws_host_call, status=status,
                                        tf32=tf32)

        e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(1, min(args.steps, 5))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b) / n_e2e, world) / (1 if shard_heads else world)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, rowsh))
        d2h = sum(t.numel() * t.element_size() for t in (oh, mseh, labh))
        e2e = {"value": e2e_ms, "unit": "ms/call", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "call": f"svg_sparse_3d_attn_host (host buffers, {args.e2e_chunk} heads per chunk, copies overlapped)"}
        del qh, kh, vh, oh, ws_host_call

    peaks, peak_kind = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    attn_tflops = flops / (kern_ms["attn"] * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    if tf32:  # dense tf32 runs at the nominal tf32 / bf16 ratio of the bf16 rate
        peak *= TF32_PER_BF16
    perm_bytes = 2 * 3 * n_temporal * wl.B * wl.L * wl.d * es
    unperm_bytes = 2 * n_temporal * wl.B * wl.L * wl.d * es

    # the layout-transformation kernels on this call's labels, timed on their
    # own after the timed region (when the call fuses the layout they are not
    # part of it); each moves more than L2 holds, so no flush is needed
    layout_kernels = None
    if not mixed and n_temporal and not args.no_configs:
        if fused:
            qp, kp, vp, op = (torch.empty_like(q) for _ in range(4))
        t_perm = time_calls(lambda: svg.svg_permute_qkv(q, k, v, N, F, label, out=(qp, kp, vp), **lk), 5, stream)
        t_unperm = time_calls(lambda: svg.svg_unpermute(op, N, F, label, out=o, **lk), 5, stream)
        layout_kernels = {
            "permute_ms": t_perm, "permute_gbs": perm_bytes / (t_perm * 1e-3) / 1e9,
            "permute_frac_hbm": perm_bytes / (t_perm * 1e-3) / 1e9 / hbm,
            "unpermute_ms": t_unperm, "unpermute_gbs": unperm_bytes / (t_unperm * 1e-3) / 1e9,
            "unpermute_frac_hbm": unperm_bytes / (t_unperm * 1e-3) / 1e9 / hbm,
            "bytes": {"permute": perm_bytes, "unpermute": unperm_bytes},
            "note": "svg_permute_qkv / svg_unpermute on this call's temporal heads, 2 warm + 5 timed calls each"}
        if fused:
            qp = kp = vp = op = None
    prof_bytes = 2 * wl.B * wl.H * wl.L * wl.d * es  # K and V read once
    roofline_profile = None
    if not mixed:
        prof_gbs = prof_bytes / (kern_ms["profile"] * 1e-3) / 1e9
        roofline_profile = {"bound": "hbm", "kernel": "svg_profile_heads: profile_sm100_kernel + "
                            "profile_combine_rows_kernel + profile_finalize_kernel (whole call timed)",
                            "achieved": prof_gbs, "peak": hbm, "peak_kind": f"{peak_kind} hbm_gbs",
                            "unit": "GB/s", "frac": prof_gbs / hbm,
                            "traffic": PROF_NCU_TRAFFIC.get(prof_source_key()) if wl.name == "hunyuan" else None,
                            "algorithmic_work": f"{prof_bytes:.4e} bytes/launch = K and V of every head once"}
    configs = None
    if not args.no_configs and rank == 0 and world == 1 and wl.name == "hunyuan" and tl == "bhld" and not tf32:
        configs = []
        qp = kp = vp = op = None
        torch.cuda.empty_cache()
        for cw in (synth.WORKLOADS["cogvideox"], wl.with_bands(*synth.HUNYUAN_SWEEP[0.05], name="hunyuan-5%"),
                   wl.with_bands(*synth.HUNYUAN_SWEEP[0.5], name="hunyuan-50%"), synth.WORKLOADS["mixed"]):
            configs.append(measure_config(cw, dev, stream, peak))
            torch.cuda.empty_cache()
        # the headline workload again on [B, L, H, d] tensors
        configs.append(measure_config(wl, dev, stream, peak, layout="blhd"))
        torch.cuda.empty_cache()
    # the seconds-long power-capped figure, shown beside the burst one
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    if tf32:
        peak_sus *= TF32_PER_BF16

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not mixed:
        qkv64 = head_f64(wl, *((t.transpose(1, 2) for t in (q, k, v)) if tl == "blhd" else (q, k, v)))
        ms, desc, _ = oracle_sample(wl, qkv64, rows_np, labels_np, n_prof_rows=wl.S, n_attn_rows=1024)
        cpu = {"value": ms, "unit": "ms/call", "cores": cpu_cores(), "kind": "oracle", "sample": desc}

    line = {
        "metric": METRIC, "value": value, "unit": "ms/call", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": False,
        "scaling": "strong" if shard_heads else "weak",
        "vs_baseline": None, "dtype": "tf32" if tf32 else "bf16", "data": "synthetic",
        "config": dict(config_dict(job_wl, world, "heads" if shard_heads else "replicas"),
                       tensor_layout="[B, L, H, d]" if tl == "blhd" else "[B, H, L, d]"),
        "effective_tflops": attn_tflops, "effective_tflops_call": flops / (step_ms * 1e-3) / 1e12,
        "frac_bf16_peak": attn_tflops / peak,
        "speedup_vs_dense": (dense_ms / step_ms) if dense_ms else None,
        "dense_ms": dense_ms,
        "kernel_ms": kern_ms,
        "call_ms_spread": spread,
        "layout": ("fused: token-major heads loaded by frame-group boxes in the attention kernel, no permuted copies"
                   if fused else "separate: permute -> attention -> unpermute"),
        "layout_plan": {"separate_tiles_per_head": plan_sep, "fused_tiles_per_head": plan_fused,
                        "choice": "fused" if plan_choice else "separate", "requested": args.layout},
        "permute_gbs": (perm_bytes / (kern_ms["permute"] * 1e-3) / 1e9 if n_temporal and not fused else
                        layout_kernels["permute_gbs"] if layout_kernels else None),
        "unpermute_gbs": (unperm_bytes / (kern_ms["unpermute"] * 1e-3) / 1e9 if n_temporal and not fused else
                          layout_kernels["unpermute_gbs"] if layout_kernels else None),
        "layout_kernels": layout_kernels,
        "temporal_heads": n_temporal,
        "density": pairs / (wl.B * wl.H * float(wl.L) * wl.L),
        "roofline": {"bound": "tensor", "kernel": f"{'attn_tf32_kernel' if tf32 else 'attn_sm100_kernel'}<{wl.d}>",
                     "achieved": attn_tflops, "peak": peak,
                     "peak_kind": f"{peak_kind} bf16_tflops (burst)" + (TF32_PEAK_NOTE if tf32 else ""),
                     "unit": "TFLOP/s", "frac": attn_tflops / peak,
                     "peak_sustained": peak_sus, "frac_sustained": attn_tflops / peak_sus,
                     "traffic": args.traffic if args.traffic is not None else (
                         NCU_TRAFFIC.get(attn_source_key() + (("fused" if fused else "separate")
                                                               + ("" if tl == "bhld" else "-blhd")
                                                               + ("-tf32" if tf32 else ""),))
                         if wl.name == "hunyuan" else None),
                     "algorithmic_work": f"{flops:.4e} flops/launch = 4*d*unmasked pairs"},
        "roofline_profile": roofline_profile,
        "hbm_peak_gbs": hbm,
        "configs": configs,
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": len(names) * args.steps + (0 if mixed else (PROFILE_LAUNCHES - 1) * args.steps),
        "cpu_baseline": cpu,
    }
    if mode_search is not None:
        line["mode_search"] = mode_search
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="hunyuan")
    ap.add_argument("--density", type=float, default=None, help="HunyuanVideo sweep density (0.05..0.5)")
    ap.add_argument("--heads", type=int, default=None, help="override the head count (small profiling cases)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--shard", choices=["heads", "replicas"], default="heads",
                    help="N > 1: split the heads of one call over the ranks (strong scaling), or run one "
                         "independent call per rank (weak scaling)")
    ap.add_argument("--layout", choices=["auto", "fused", "separate"], default="auto",
                    help="temporal heads' layout transformation fused into attention, or as separate kernels; "
                         "auto = the whole call's own choice")
    ap.add_argument("--tensor-layout", choices=["bhld", "blhd"], default="bhld",
                    help="q, k, v, o as [B, H, L, d] or [B, L, H, d] (the whole call then takes the separate plan; "
                         "no host-buffer e2e, which takes [B, H, L, d])")
    ap.add_argument("--precision", choices=["bf16", "tf32"], default="bf16",
                    help="tf32: the same inputs as fp32 tensors, attention on the tensor cores in tf32 (SVG_TF32; "
                         "profiling in fp32 on the CUDA cores)")
    ap.add_argument("--e2e-chunk", type=int, default=2, help="heads per chunk of the host-buffer call")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-config lines (CogVideoX, the 5 %% / 50 %% sweep ends, mixed) and the "
                         "stand-alone permute / unpermute timing that follow the timed region")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per attention launch from an ncu capture of this kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    if args.density is not None:
        a1, a2 = synth.HUNYUAN_SWEEP[args.density]
        wl = wl.with_bands(a1, a2)
    if args.heads is not None:
        import dataclasses
        wl = dataclasses.replace(wl, H=args.heads, name=f"{wl.name}-{args.heads}heads")
    if args.impl == "reference":
        # the oracle runs on host cores; no process group is needed: rank 0
        # works, the other ranks exit at once
        run_reference(args, wl, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
        return
    if not torch.cuda.is_available():
        raise SystemExit("no CUDA device: the benchmark measures the CUDA path only")
    rank, world, local = dist_setup(args.gpus)
    try:
        if wl.name == "svg2":
            run_svg2(args, wl, rank, world, local)
        else:
            run_ours(args, wl, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    main()
