"""Benchmark of the h3attn hot path on B200: one step = the Q/K RMSNorm + RoPE
prologue followed by dense non-causal attention, on the 2K-refine workload
(one clip of a 32 x 48 x 84 latent grid = 129,024 tokens, 24 heads of 128).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl h3attn|reference]

Prints one JSON line (rank 0).  Metric: attention forward TFLOP/s counted as
4 * N^2 * d * H per clip, whole job, max time over ranks.  With N GPUs every
rank runs its own clip (weak scaling, no collective on the data path).

--impl reference times the fp64 CPU oracle (the correctness reference of this
project) on the host cores, on a bounded sample of the same workload.

Besides the step, the line carries rooflines of the kernels timed on their own
after it (not part of the step): the LSE merge on the clip's output shape, the
fused Q/K/V projection at model width against cuBLAS + the prologue, and
block-sparse attention on the clip's sequence with a seeded 25% tile pattern.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (4·N²·d·H) and % of B200 dense BF16 peak at N=129k"
WORKLOAD = "2k"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def workload_config(w, n_gpus):
    return {
        "workload": "2K refine clip: latent grid 32x48x84 = 129024 tokens, 24 heads x 128, "
                    "Q/K RMSNorm (eps 1e-6) + 3D RoPE 32/48/48 (theta 1e4) + non-causal attention",
        "global_batch": n_gpus,
        "seq_len": int(w.total),
        "heads": int(w.n_heads),
        "head_dim": int(w.head_dim),
        "parallelism": "replicas" if n_gpus == 1 else "dp%d" % n_gpus,
        "l2": "inputs larger than L2 (Q, K, V 2.4 GB per clip)",
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# -----------------------------------------------------------------------------------------
# clocks during the timed region
# -----------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.samples = []
        if self.proc is None:
            return False
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)
        return False

    def summary(self):
        if not getattr(self, "samples", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        pw = [float(s[3]) for s in self.samples if s[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for s in self.samples for n, v in zip(names, s[5:9]) if v.lower() == "active"})
        loaded = [c for c, p in zip(sm, pw) if p > 0.5 * max(pw)] if pw else sm
        return {"sm_mhz": statistics.median(loaded or sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples), "power_w_max": max(pw) if pw else None}


# -----------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)
# -----------------------------------------------------------------------------------------
def _cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_sample_setup(w, orc):
    """K' of the whole clip (every query attends to all of it) -- done once."""
    t0 = time.perf_counter()
    _, k16 = orc.rmsnorm_rope(w.k, w.gamma_k, w.eps, w.pos, w.kind, w.sections, w.theta, want_f64=False)
    return k16, time.perf_counter() - t0


def oracle_sample_step(w, orc, k16, rows):
    """Oracle prologue of the sampled query rows + attention of those rows over all keys."""
    _, q16 = orc.rmsnorm_rope(w.q[rows], w.gamma_q, w.eps, w.pos[rows], w.kind[rows], w.sections,
                              w.theta, want_f64=False)
    # the oracle reads query rows by index: scatter the sampled rows into a full-size
    # buffer (np.empty maps pages lazily, so only the sampled rows are touched)
    qbuf = np.empty_like(w.q)
    qbuf[rows] = q16
    orc.attention(qbuf, k16, w.v, w.cu_seqlens, rows=rows)


def cpu_baseline(w, rows_target_s=15.0):
    import oracle
    orc = oracle.get()
    k16, t_k = oracle_sample_setup(w, orc)
    rows = np.arange(4, dtype=np.int64) * 7919 % w.total
    t0 = time.perf_counter()
    oracle_sample_step(w, orc, k16, rows)
    t_probe = time.perf_counter() - t0
    n = int(max(4, min(w.total, len(rows) * rows_target_s / max(t_probe, 1e-3))))
    rows = np.unique(np.linspace(0, w.total - 1, n).astype(np.int64))
    t0 = time.perf_counter()
    oracle_sample_step(w, orc, k16, rows)
    t_rows = time.perf_counter() - t0
    flops_rows = 4.0 * len(rows) * w.total * w.head_dim * w.n_heads
    # whole-clip time: prologue of all Q and K rows (2x the K pass) + attention of every row
    t_full = 2.0 * t_k + t_rows * w.total / len(rows)
    return {
        "value": w.attention_flops() / t_full / 1e12,
        "unit": "TFLOP/s",
        "cores": _cores_used(),
        "kind": "oracle",
        "sample": "%d of %d query rows x %d heads (full keys) + the K prologue of the whole clip; "
                  "extrapolated linearly to the whole clip (rows are independent and equal cost)"
                  % (len(rows), w.total, w.n_heads),
        "sample_tflops": flops_rows / t_rows / 1e12,
        "seconds": t_k + t_rows,
    }


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from video_diffusion_transformer_h3attn_b200 import inputs
    w = inputs.workload(WORKLOAD)
    orc = oracle.get()
    k16, _ = oracle_sample_setup(w, orc)
    rng = np.random.default_rng(0)
    n_rows = 8
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(w.total, n_rows, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle_sample_step(w, orc, k16, rows)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    step = statistics.mean(times)
    flops = 4.0 * n_rows * w.total * w.head_dim * w.n_heads
    value = flops / step / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cores_used(), "kind": "oracle",
                         "sample": "%d random query rows x %d heads per step (full keys; K prologue "
                                   "done once before timing)" % (n_rows, w.n_heads)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# -----------------------------------------------------------------------------------------
# GPU arm
# -----------------------------------------------------------------------------------------
ATTENTION_SOURCES = ("attention.cuh", "sm100_ptx.cuh", "common.cuh")


def source_hash():
    """Hash of the attention kernel's sources with comments and blank space
    removed (a stored ncu figure is only used while the code is unchanged)."""
    import re
    h = hashlib.sha256()
    for f in ATTENTION_SOURCES:
        with open(os.path.join(ROOT, "video_diffusion_transformer_h3attn_b200", "csrc", f)) as fh:
            text = re.sub(r"//[^\n]*", "", fh.read())
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "attention_2k_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("source_hash") != source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


def reduce_max(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (the job is as slow as its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import video_diffusion_transformer_h3attn_b200 as h3
    from video_diffusion_transformer_h3attn_b200 import inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        args.gpus = world
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    w = inputs.workload(WORKLOAD)
    dev = torch.device("cuda", local)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

    host = {
        "q": bf16(w.q).pin_memory(), "k": bf16(w.k).pin_memory(), "v": bf16(w.v).pin_memory(),
        "gq": bf16(w.gamma_q).pin_memory(), "gk": bf16(w.gamma_k).pin_memory(),
        "pos": torch.from_numpy(w.pos).pin_memory(), "kind": torch.from_numpy(w.kind).pin_memory(),
    }
    d = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    qp = torch.empty_like(d["q"])
    kp = torch.empty_like(d["k"])
    o = torch.empty_like(d["q"])
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    ev = {"pro": [], "att": []}

    def step(record=False):
        if record:
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
        h3.prologue(d["q"], d["k"], qp, kp, d["gq"], d["gk"], w.eps, d["pos"], d["kind"], w.sections, w.theta)
        if record:
            e[1].record(stream)
        h3.attention(qp, kp, d["v"], o)
        if record:
            e[2].record(stream)
            ev["pro"].append((e[0], e[1]))
            ev["att"].append((e[1], e[2]))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    # ---- device-resident timing ----
    for _ in range(args.warmup):
        step()
    h3.device_status()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for _ in range(args.steps):
            step(record=True)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    h3.device_status()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps)
    att_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["att"])
    pro_ms = statistics.mean(a.elapsed_time(b) for a, b in ev["pro"])

    # ---- end to end through the public API: host buffers in, result back to host ----
    # Every step copies its inputs from pinned host memory and its output back.  Two
    # buffer sets and two copy streams let step i+1's upload and step i-1's download
    # run under step i's kernels (the copies use the PCIe engines, the kernels the SMs).
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o.numel() * o.element_size()
    sets = [dict(d=d, qp=qp, kp=kp, o=o, oh=o_host)]
    sets.append(dict(d={k: torch.empty_like(v) for k, v in d.items()}, qp=torch.empty_like(qp),
                     kp=torch.empty_like(kp), o=torch.empty_like(o),
                     oh=torch.empty(o.shape, dtype=o.dtype).pin_memory()))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("up", "run", "down")}

    def e2e_run(n_steps, t_start=None, t_end=None):
        for i in range(n_steps):
            b = sets[i % 2]
            e_up, e_run, e_down = ev["up"][i % 2], ev["run"][i % 2], ev["down"][i % 2]
            s_in.wait_event(e_run)          # set b's previous kernels finished reading it
            if i == 0 and t_start is not None:
                t_start.record(s_in)
            with torch.cuda.stream(s_in):
                for k, v in host.items():
                    b["d"][k].copy_(v, non_blocking=True)
            e_up.record(s_in)
            stream.wait_event(e_up)
            stream.wait_event(e_down)       # set b's previous output is already on the host
            h3.prologue(b["d"]["q"], b["d"]["k"], b["qp"], b["kp"], b["d"]["gq"], b["d"]["gk"], w.eps,
                        b["d"]["pos"], b["d"]["kind"], w.sections, w.theta)
            h3.attention(b["qp"], b["kp"], b["d"]["v"], b["o"])
            e_run.record(stream)
            s_out.wait_event(e_run)
            with torch.cuda.stream(s_out):
                b["oh"].copy_(b["o"], non_blocking=True)
            e_down.record(s_out)
        if t_end is not None:
            s_out.wait_event(ev["down"][(n_steps - 1) % 2])
            t_end.record(s_out)

    e2e_run(max(1, args.warmup))
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, e0, e1)
    torch.cuda.synchronize()
    barrier()
    h3.device_status()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)

    flops = w.attention_flops()
    value = world * flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    merge_line = measure_merge(h3, w, dev, stream, max(3, args.steps), peaks, peak_src)
    qkv_line = measure_qkv(h3, w, dev, stream, max(3, args.steps), peaks, peak_src)
    sparse_line = measure_sparse(h3, w, dev, stream, max(3, args.steps), peaks, peak_src, att_ms)
    att_tflops = flops / (att_ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    pro_bytes = 4.0 * w.total * w.n_heads * w.head_dim * 2 + 12.0 * w.total + w.total + 4 * w.head_dim
    pro_gbs = pro_bytes / (pro_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(w, world),
        "pct_of_datasheet_2250": 100.0 * value / world / DATASHEET_BF16_TFLOPS,
        "pct_of_measured_burst": 100.0 * value / world / peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
        "kernels_ms": {"prologue": pro_ms, "attention": att_ms},
        "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": att_tflops / peak, "traffic": profiled_traffic(),
                     "kernel": "attn_fwd_kernel<128,false>",
                     "peak_source": "%s bf16_tflops_sustained (kernel timed inside a long step)" % peak_src},
        "roofline_prologue": {"bound": "hbm", "achieved": pro_gbs, "peak": peaks.get("hbm_gbs"),
                              "unit": "GB/s", "frac": pro_gbs / peaks.get("hbm_gbs", 6650.0),
                              "peak_source": peak_src},
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "overlap": "uploads and downloads on two copy streams under the previous/next step's kernels"},
        "roofline_merge": merge_line,
        "roofline_qkv": qkv_line,
        "roofline_sparse": sparse_line,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = cpu_baseline(w)
        except Exception as exc:  # the baseline is reported, never required
            line["cpu_baseline"] = {"value": None, "unit": "TFLOP/s", "cores": _cores_used(),
                                    "kind": "oracle", "sample": "failed: %s" % exc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def measure_merge(h3, w, dev, stream, steps, peaks, peak_src):
    """The log-sum-exp merge of two partial results (a key-split schedule's
    combine step) on the workload's full output shape, timed on its own after
    the step measurements: HBM-bound, 3 rows of d bf16 + 3 fp32 per (token, head)."""
    import torch
    g = torch.Generator(device=dev).manual_seed(5)
    shape = (1, w.total, w.n_heads, w.head_dim)
    oa = torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    ob = torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    la = torch.randn((1, w.n_heads, w.total), generator=g, device=dev) * 4
    lb = torch.randn((1, w.n_heads, w.total), generator=g, device=dev) * 4
    o = torch.empty_like(oa)
    lse = torch.empty_like(la)
    for _ in range(3):
        h3.merge(oa, la, ob, lb, o=o, lse=lse)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        h3.merge(oa, la, ob, lb, o=o, lse=lse)
    e1.record(stream)
    torch.cuda.synchronize()
    h3.device_status()
    ms = e0.elapsed_time(e1) / steps
    nbytes = 3.0 * w.total * w.n_heads * (w.head_dim * 2 + 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    del oa, ob, la, lb, o, lse
    return {"bound": "hbm", "achieved": gbs, "peak": peaks.get("hbm_gbs"), "unit": "GB/s",
            "frac": gbs / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), "ms": ms,
            "bytes_per_launch": nbytes, "kernel": "merge_kernel<128>", "peak_source": peak_src,
            "note": "not part of the step: the combine of two partial results over split keys, "
                    "on this workload's output shape"}


SPARSE_KEEP = 0.25  # share of the off-diagonal key tiles each query-tile pair keeps


def _sparse_lists(w):
    """The block-sparse pattern measured on a single-sequence workload (its diagonal
    key tiles plus a seeded quarter of the others per (head, 256-row query block))
    and the FLOPs it leaves: 4 d x (query rows) x (listed keys) per list."""
    from video_diffusion_transformer_h3attn_b200 import inputs
    N, H, d = w.total, w.n_heads, w.head_dim
    off, idx = inputs.block_lists(1, H, N, N, SPARSE_KEEP, seed=w.seed + 77)
    n_qp, n_kt = -(-N // 256), -(-N // 128)
    keys = np.full(n_kt, 128, dtype=np.int64)
    keys[-1] = N - 128 * (n_kt - 1)
    rows = np.full(n_qp, 256, dtype=np.int64)
    rows[-1] = N - 256 * (n_qp - 1)
    cs = np.concatenate([[0], np.cumsum(keys[idx])])
    keys_per_list = cs[off[1:]] - cs[off[:-1]]
    flops = 4.0 * d * float(np.sum(np.tile(rows, H) * keys_per_list))
    return off, idx, flops


def measure_sparse(h3, w, dev, stream, steps, peaks, peak_src, dense_ms):
    """Block-sparse attention on the workload's sequence with the pattern above,
    timed on its own after the step measurements (not part of the step);
    tensor-bound on the FLOPs of the listed tiles."""
    import torch
    if len(w.seqlens) != 1:
        return None
    off, idx, flops = _sparse_lists(w)
    N, H, d = w.total, w.n_heads, w.head_dim

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = (bf16(a).view(1, N, H, d) for a in (w.q, w.k, w.v))
    offt = torch.from_numpy(off).to(dev)
    idxt = torch.from_numpy(idx).to(dev)
    o = torch.empty_like(q)
    for _ in range(3):
        h3.attention_block_sparse(q, k, v, offt, idxt, o=o)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        h3.attention_block_sparse(q, k, v, offt, idxt, o=o)
    e1.record(stream)
    torch.cuda.synchronize()
    h3.device_status()
    ms = e0.elapsed_time(e1) / steps
    tflops = flops / (ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    del q, k, v, o
    return {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
            "ms": ms, "flops_per_launch": flops, "density": flops / w.attention_flops(),
            "speedup_vs_dense": dense_ms / ms, "kernel": "attn_fwd_kernel<128,false> with key lists",
            "peak_source": "%s bf16_tflops_sustained" % peak_src,
            "note": "not part of the step: block-sparse attention over this workload's sequence, "
                    "diagonal key tiles plus a seeded %.0f%% of the others per 256-row query block"
                    % (100 * SPARSE_KEEP)}


def _qkv_inputs(w, dev):
    """Token activations and a projection weight of the workload's model width
    (dim_in = H*d, 3*H*d features), seeded; positions and gammas from the workload."""
    import torch
    g = torch.Generator(device=dev).manual_seed(7)
    hd = w.n_heads * w.head_dim
    x = torch.randn((w.total, hd), generator=g, device=dev).to(torch.bfloat16)
    wt = (torch.randn((3 * hd, hd), generator=g, device=dev) / hd ** 0.5).to(torch.bfloat16)
    bias = (torch.randn(3 * hd, generator=g, device=dev) * 0.1).to(torch.bfloat16)
    return x, wt, bias


def measure_qkv(h3, w, dev, stream, steps, peaks, peak_src):
    """The Q/K/V projection with the prologue fused into its epilogue, on the
    workload's token count at model width, against the unfused path (cuBLAS
    projection, then the prologue kernel) timed the same way.  Not part of the step."""
    import torch

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    x, wt, bias = _qkv_inputs(w, dev)
    gq, gk = bf16(w.gamma_q), bf16(w.gamma_k)
    pos, kind = torch.from_numpy(w.pos).to(dev), torch.from_numpy(w.kind).to(dev)
    H, d = w.n_heads, w.head_dim
    out = torch.empty((w.total, 3, H, d), dtype=torch.bfloat16, device=dev)
    q, k, v = out[:, 0], out[:, 1], out[:, 2]

    def fused():
        h3.qkv_fused(x, wt, H, bias=bias, q_out=q, k_out=k, v_out=v, gamma_q=gq, gamma_k=gk, eps=w.eps,
                     pos=pos, kind=kind, sections=w.sections, theta=w.theta)

    proj = torch.empty((w.total, 3 * H * d), dtype=torch.bfloat16, device=dev)
    qp = torch.empty((w.total, H, d), dtype=torch.bfloat16, device=dev)
    kp = torch.empty_like(qp)

    def unfused():
        torch.addmm(bias, x, wt.T, out=proj)
        pv = proj.view(w.total, 3, H, d)
        h3.prologue(pv[:, 0], pv[:, 1], qp, kp, gq, gk, w.eps, pos, kind, w.sections, w.theta)

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms = timed(fused)
    h3.device_status()
    ms_unfused = timed(unfused)
    flops = 2.0 * w.total * (H * d) * (3 * H * d)
    tf = flops / (ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    del x, wt, bias, out, proj, qp, kp
    return {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak, "ms": ms,
            "unfused_ms": ms_unfused, "speedup_vs_unfused": ms_unfused / ms, "flops_per_launch": flops,
            "kernel": "qkv_fused_pair_kernel<%d>" % d, "peak_source": "%s bf16_tflops (kernel timed alone)" % peak_src,
            "note": "not part of the step: projection dim_in = H*d to 3*H*d features with RMSNorm + RoPE in the "
                    "epilogue, on this workload's tokens; unfused = cuBLAS addmm then the prologue kernel"}


def run_kernel_only(args):
    """W + K launches of one kernel on one workload and nothing else (for ncu captures)."""
    import torch

    import video_diffusion_transformer_h3attn_b200 as h3
    from video_diffusion_transformer_h3attn_b200 import inputs

    w = inputs.workload(args.workload)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

    q, k, v = bf16(w.q), bf16(w.k), bf16(w.v)
    out = torch.empty_like(q)
    if args.kernel_only == "qkv":
        x, wt, bias = _qkv_inputs(w, "cuda")
        gq, gk = bf16(w.gamma_q), bf16(w.gamma_k)
        pos, kind = torch.from_numpy(w.pos).cuda(), torch.from_numpy(w.kind).cuda()
        run = lambda: h3.qkv_fused(x, wt, w.n_heads, bias=bias, gamma_q=gq, gamma_k=gk, eps=w.eps, pos=pos,
                                   kind=kind, sections=w.sections, theta=w.theta)
        unit = 2.0 * w.total * (w.n_heads * w.head_dim) * (3 * w.n_heads * w.head_dim) / 1e12
    elif args.kernel_only == "merge":
        g = torch.Generator(device="cuda").manual_seed(5)
        shape = (1, w.total, w.n_heads, w.head_dim)
        oa = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
        ob = torch.randn(shape, generator=g, device="cuda").to(torch.bfloat16)
        la = torch.randn((1, w.n_heads, w.total), generator=g, device="cuda")
        lb = torch.randn((1, w.n_heads, w.total), generator=g, device="cuda")
        lo = torch.empty_like(la)
        run = lambda: h3.merge(oa, la, ob, lb, o=out.view(shape), lse=lo)
        unit = 3.0 * w.total * w.n_heads * (w.head_dim * 2 + 4) / 1e9
    elif args.kernel_only == "sparse":
        off, idx, flops = _sparse_lists(w)
        shape = (1, w.total, w.n_heads, w.head_dim)
        offt, idxt = torch.from_numpy(off).cuda(), torch.from_numpy(idx).cuda()
        run = lambda: h3.attention_block_sparse(q.view(shape), k.view(shape), v.view(shape), offt, idxt,
                                                o=out.view(shape))
        unit = flops / 1e12
    elif args.kernel_only == "prologue":
        g = (bf16(w.gamma_q), bf16(w.gamma_k)) if w.gamma_q is not None else (None, None)
        pos = torch.from_numpy(w.pos).cuda() if w.pos is not None else None
        kind = torch.from_numpy(w.kind).cuda() if w.kind is not None else None
        kout = torch.empty_like(k)
        run = lambda: h3.prologue(q, k, out, kout, g[0], g[1], w.eps, pos, kind, w.sections, w.theta)
        unit = 4.0 * w.total * w.n_heads * w.head_dim * 2 / 1e9  # GB per launch
    elif len(w.seqlens) > 1:
        cu = torch.from_numpy(w.cu_seqlens).cuda()
        run = lambda: h3.attention_varlen(q, k, v, cu, max(w.seqlens), out)
        unit = w.attention_flops() / 1e12
    else:
        run = lambda: h3.attention(q, k, v, out)
        unit = w.attention_flops() / 1e12
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        run()
    e1.record()
    torch.cuda.synchronize()
    h3.device_status()
    ms = e0.elapsed_time(e1) / args.steps
    print(json.dumps({"kernel": args.kernel_only, "workload": args.workload, "ms": ms,
                      "rate": unit / (ms * 1e-3),
                      "rate_unit": "TFLOP/s" if args.kernel_only in ("attention", "qkv", "sparse") else "GB/s"}),
          flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["h3attn", "reference"], default="h3attn")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="workload for --kernel-only runs (tiny, small, joint, 2k, ragged)")
    ap.add_argument("--kernel-only", choices=["attention", "prologue", "merge", "qkv", "sparse"],
                    help="launch only this kernel W + K times (profiling runs)")
    args = ap.parse_args()
    if args.kernel_only:
        return run_kernel_only(args)
    if args.warmup < 3 and args.impl == "h3attn":
        print("note: raising --warmup to 3", file=sys.stderr)
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
