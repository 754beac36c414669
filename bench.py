"""Benchmark of the h3attn hot path on B200: one step = the Q/K RMSNorm + RoPE
prologue followed by non-causal attention on one clip; by default the 2K-refine
workload (a 32 x 48 x 84 latent grid = 129,024 tokens, 24 heads of 128).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl h3attn|reference]
                    [--workload tiny|small|joint|2k|ragged] [--parallel replicas|ulysses]
    python bench.py --table [names]      one line per workload, with the oracle beside it

Prints one JSON line (rank 0).  Metric: attention forward TFLOP/s counted as
4 * N^2 * d * H per clip (summed over the sequences of a ragged batch), whole
job, max time over ranks.  --parallel replicas (default): every rank runs its
own clip (weak scaling, no collective on the data path).  --parallel ulysses:
the ranks share one clip, split by tokens, with NCCL all-to-alls to head shards
around attention (strong scaling).

--impl reference times the fp64 CPU oracle (the correctness reference of this
project) on the host cores, on a bounded sample of the same workload.

Besides the step, the default line carries rooflines of the kernels timed on
their own after it (not part of the step): the LSE merge on the clip's output
shape, the fused Q/K/V projection at model width against cuBLAS + the prologue,
and block-sparse attention on the clip's sequence with a seeded 25% tile pattern.
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


WORKLOAD_TEXT = {
    "tiny": "tiny clip: 4x8x8 grid = 256 tokens, 2 heads x 64, attention only",
    "small": "small DiT block: 8x16x24 grid = 3072 tokens, 24 heads x 128, Q/K RMSNorm (eps 1e-6) + 3D RoPE "
             "32/48/48 (theta 1e4) + non-causal attention",
    "joint": "joint video+audio clip: 16x30x54 grid = 25920 video + 256 audio = 26176 tokens, 24 heads x 128, "
             "Q/K RMSNorm + 3D RoPE (video) / 1D RoPE (audio) + non-causal attention",
    "2k": "2K refine clip: latent grid 32x48x84 = 129024 tokens, 24 heads x 128, Q/K RMSNorm (eps 1e-6) + "
          "3D RoPE 32/48/48 (theta 1e4) + non-causal attention",
    "ragged": "ragged packed batch: 4 sequences of 4096/9000/17001/31234 = 61331 tokens, 16 heads x 128, "
              "1D RoPE (theta 1e4), Q x4, no norm, attention per sequence via cu_seqlens",
}


def workload_config(w, n_gpus, parallel="replicas"):
    cfg = {
        "workload": WORKLOAD_TEXT.get(w.name, w.name),
        "global_batch": n_gpus if parallel == "replicas" else 1,
        "seq_len": int(w.total),
        "heads": int(w.n_heads),
        "head_dim": int(w.head_dim),
        "parallelism": ("replicas" if n_gpus == 1 else "dp%d" % n_gpus) if parallel == "replicas"
        else "ulysses%d" % n_gpus,
    }
    qkv_bytes = 3 * w.total * w.n_heads * w.head_dim * 2
    cfg["l2"] = ("inputs larger than L2 (Q, K, V %.1f GB per clip)" % (qkv_bytes / 1e9) if qkv_bytes > 126e6
                 else "inputs smaller than L2 (%.1f MB): L2 is not flushed between steps" % (qkv_bytes / 1e6))
    return cfg


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


CPU_SAMPLE_PAIRS = 2048   # (query row, head) pairs timed for cpu_baseline
REFERENCE_STEP_PAIRS = 1024  # (query row, head) pairs per step of --impl reference


def oracle_k_prologue(w, orc):
    """K' of the whole clip (every sampled query attends to all of it): done once, timed."""
    t0 = time.perf_counter()
    if w.has_prologue:
        _, k16 = orc.rmsnorm_rope(w.k, w.gamma_k, w.eps, w.pos, w.kind, w.sections, w.theta, want_f64=False)
    else:
        k16 = w.k
    return k16, time.perf_counter() - t0


def sample_pairs(w, n_pairs, seed):
    """n_pairs (query row, head) pairs: rows that visit every 128-row query tile
    (inputs.sample_rows_every_tile), heads assigned in turn."""
    from video_diffusion_transformer_h3attn_b200 import inputs
    rows = inputs.sample_rows_every_tile(w.cu_seqlens, n_pairs, seed=seed)
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    rows = np.sort(rng.choice(rows, size=min(n_pairs, len(rows)), replace=False))
    heads = np.arange(len(rows)) % w.n_heads
    return rows, heads


def oracle_pairs(w, orc, k16, rows, heads):
    """The oracle on the given (row, head) pairs: the prologue of those query rows,
    then each row's attention over all keys of its sequence, one head per row.
    Returns the FLOPs of the attention part (4 d per key per pair)."""
    if w.has_prologue:
        _, q16 = orc.rmsnorm_rope(w.q[rows], w.gamma_q, w.eps, w.pos[rows], w.kind[rows], w.sections,
                                  w.theta, want_f64=False)
    else:
        q16 = w.q[rows]
    # the oracle reads query rows by index: scatter the sampled rows into a full-size
    # buffer (np.empty maps pages lazily, so only the sampled rows are touched)
    flops = 0.0
    seq_of = np.searchsorted(w.cu_seqlens, rows, side="right") - 1
    lens = np.diff(w.cu_seqlens)
    for h in range(w.n_heads):
        sel = heads == h
        if not np.any(sel):
            continue
        qb = np.empty((w.total, 1, w.head_dim), dtype=np.uint16)
        qb[rows[sel], 0] = q16[sel, h]
        orc.attention(qb, np.ascontiguousarray(k16[:, h:h + 1]), np.ascontiguousarray(w.v[:, h:h + 1]),
                      w.cu_seqlens, rows=rows[sel])
        flops += 4.0 * w.head_dim * float(np.sum(lens[seq_of[sel]]))
    return flops


def cpu_baseline(w):
    """The oracle timed on this host: the K prologue of the whole clip, then 2,048
    (query row, head) pairs over every query tile; extrapolated to the whole clip."""
    import oracle
    orc = oracle.get()
    k16, t_k = oracle_k_prologue(w, orc)
    rows, heads = sample_pairs(w, CPU_SAMPLE_PAIRS, seed=w.seed + 2000)
    t0 = time.perf_counter()
    flops = oracle_pairs(w, orc, k16, rows, heads)
    t_pairs = time.perf_counter() - t0
    # whole clip: the prologue of every Q and K row (twice the K pass) and the
    # attention of every (row, head) pair at the sampled rate
    t_full = (2.0 * t_k if w.has_prologue else 0.0) + t_pairs * w.attention_flops() / flops
    return {
        "value": w.attention_flops() / t_full / 1e12,
        "unit": "TFLOP/s",
        "cores": _cores_used(),
        "kind": "oracle",
        "sample": "%d (query row, head) pairs, rows visiting all %d query tiles of 128, heads in turn, "
                  "each over every key of its sequence (%s), + the K prologue of the whole clip (%.1f s); "
                  "extrapolated linearly to the whole clip (pairs are independent, cost proportional to keys)"
                  % (len(rows), sum(-(-n // 128) for n in w.seqlens),
                     "%d keys" % w.total if len(w.seqlens) == 1 else "%d sequences" % len(w.seqlens), t_k),
        "sample_tflops": flops / t_pairs / 1e12,
        "seconds": t_k + t_pairs,
    }


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from video_diffusion_transformer_h3attn_b200 import inputs
    w = inputs.workload(args.workload)
    orc = oracle.get()
    k16, _ = oracle_k_prologue(w, orc)
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        rows, heads = sample_pairs(w, REFERENCE_STEP_PAIRS, seed=w.seed + 3000 + i)
        t0 = time.perf_counter()
        f = oracle_pairs(w, orc, k16, rows, heads)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            flops.append(f)
    step = statistics.mean(times)
    value = sum(flops) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cores_used(), "kind": "oracle",
                         "sample": "%d (query row, head) pairs per step, rows visiting every query tile, "
                                   "each over all keys (the K prologue is done once before timing)"
                                   % REFERENCE_STEP_PAIRS},
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


def _bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def host_inputs(w, rows=None):
    """The workload's inputs (or the token rows `rows` of them) in pinned host memory."""
    import torch
    sel = slice(None) if rows is None else rows
    host = {"q": _bf16(w.q[sel]).pin_memory(), "k": _bf16(w.k[sel]).pin_memory(),
            "v": _bf16(w.v[sel]).pin_memory()}
    if w.gamma_q is not None:
        host["gq"] = _bf16(w.gamma_q).pin_memory()
        host["gk"] = _bf16(w.gamma_k).pin_memory()
    if w.pos is not None:
        host["pos"] = torch.from_numpy(np.ascontiguousarray(w.pos[sel])).pin_memory()
        host["kind"] = torch.from_numpy(np.ascontiguousarray(w.kind[sel])).pin_memory()
    if rows is None and len(w.seqlens) > 1:
        host["cu"] = torch.from_numpy(np.ascontiguousarray(w.cu_seqlens, dtype=np.int32)).pin_memory()
    return host


def step_buffers(w, d):
    """Q', K' (when the workload has a prologue) and O for one clip on the device."""
    import torch
    b = {"o": torch.empty_like(d["q"])}
    if w.has_prologue:
        b["qp"] = torch.empty_like(d["q"])
        b["kp"] = torch.empty_like(d["k"])
    return b


def run_step(h3, w, d, b, ev=None, stream=None):
    """One pass of the hot path on one clip: the prologue into Q', K' (when the
    workload has one), then attention (ragged when it packs several sequences).
    ev = three CUDA events recorded before, between and after the two kernels."""
    if ev is not None:
        ev[0].record(stream)
    if w.has_prologue:
        h3.prologue(d["q"], d["k"], b["qp"], b["kp"], d.get("gq"), d.get("gk"), w.eps, d.get("pos"),
                    d.get("kind"), w.sections, w.theta)
        q, k = b["qp"], b["kp"]
    else:
        q, k = d["q"], d["k"]
    if ev is not None:
        ev[1].record(stream)
    if "cu" in d:
        h3.attention_varlen(q, k, d["v"], d["cu"], w.max_seqlen, b["o"])
    else:
        h3.attention(q, k, d["v"], b["o"])
    if ev is not None:
        ev[2].record(stream)


def prologue_bytes(w):
    """Algorithmic bytes of one prologue launch: Q and K read and written once, plus
    positions (12 B) and kind (1 B) per token when RoPE runs, plus both gammas."""
    b = 4.0 * w.total * w.n_heads * w.head_dim * 2
    if w.pos is not None:
        b += 13.0 * w.total
    if w.gamma_q is not None:
        b += 4.0 * w.head_dim
    return b


def timed_steps(h3, w, d, b, stream, warmup, steps):
    """W untimed then K timed steps; returns (ms per step, prologue ms, attention ms)."""
    import torch
    for _ in range(warmup):
        run_step(h3, w, d, b)
    h3.device_status()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        run_step(h3, w, d, b, evs[i], stream)
    t1.record(stream)
    torch.cuda.synchronize()
    h3.device_status()
    pro = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    return t0.elapsed_time(t1) / steps, pro, att


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

    w = inputs.workload(args.workload)
    dev = torch.device("cuda", local)
    host = host_inputs(w)
    d = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    b = step_buffers(w, d)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    # ---- device-resident timing ----
    for _ in range(args.warmup):
        run_step(h3, w, d, b)
    h3.device_status()
    barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for i in range(args.steps):
            run_step(h3, w, d, b, evs[i], stream)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    h3.device_status()
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps)
    pro_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)

    # ---- end to end through the public API: host buffers in, result back to host ----
    # Every step copies its inputs from pinned host memory and its output back.  Two
    # buffer sets and two copy streams let step i+1's upload and step i-1's download
    # run under step i's kernels (the copies use the PCIe engines, the kernels the SMs).
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = b["o"].numel() * b["o"].element_size()
    sets = [dict(d=d, b=b, oh=torch.empty(b["o"].shape, dtype=b["o"].dtype).pin_memory())]
    d2 = {k: torch.empty_like(v) for k, v in d.items()}
    sets.append(dict(d=d2, b=step_buffers(w, d2), oh=torch.empty(b["o"].shape, dtype=b["o"].dtype).pin_memory()))
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("up", "run", "down")}

    def e2e_run(n_steps, t_start=None, t_end=None):
        for i in range(n_steps):
            st = sets[i % 2]
            e_up, e_run, e_down = ev["up"][i % 2], ev["run"][i % 2], ev["down"][i % 2]
            s_in.wait_event(e_run)          # set i%2's previous kernels finished reading it
            if i == 0 and t_start is not None:
                t_start.record(s_in)
            with torch.cuda.stream(s_in):
                for k, v in host.items():
                    st["d"][k].copy_(v, non_blocking=True)
            e_up.record(s_in)
            stream.wait_event(e_up)
            stream.wait_event(e_down)       # set i%2's previous output is already on the host
            run_step(h3, w, st["d"], st["b"])
            e_run.record(stream)
            s_out.wait_event(e_run)
            with torch.cuda.stream(s_out):
                st["oh"].copy_(st["b"]["o"], non_blocking=True)
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
    del sets, d2

    flops = w.attention_flops()
    value = world * flops / (ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    side = {}
    if not args.no_side and len(w.seqlens) == 1 and w.has_prologue:
        side["roofline_merge"] = measure_merge(h3, w, dev, stream, max(3, args.steps), peaks, peak_src)
        side["roofline_qkv"] = measure_qkv(h3, w, dev, stream, max(3, args.steps), peaks, peak_src)
        side["roofline_sparse"] = measure_sparse(h3, w, dev, stream, max(3, args.steps), peaks, peak_src,
                                                 att_ms)
    att_tflops = flops / (att_ms * 1e-3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
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
        "kernels_ms": {"prologue": pro_ms if w.has_prologue else 0.0, "attention": att_ms},
        "roofline": {"bound": "tensor", "achieved": att_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": att_tflops / peak,
                     "traffic": profiled_traffic() if args.workload == WORKLOAD else None,
                     "kernel": "attn_fwd_kernel<%d,%s>" % (w.head_dim, "true" if "cu" in d else "false"),
                     "peak_source": "%s bf16_tflops_sustained (kernel timed inside a long step)" % peak_src},
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "overlap": "uploads and downloads on two copy streams under the previous/next step's kernels"},
        "gpu_launches": (2 if w.has_prologue else 1) * args.steps,
        "clocks": clocks.summary(),
    }
    if w.has_prologue:
        pro_gbs = prologue_bytes(w) / (pro_ms * 1e-3) / 1e9
        line["roofline_prologue"] = {"bound": "hbm", "achieved": pro_gbs, "peak": peaks.get("hbm_gbs"),
                                     "unit": "GB/s", "frac": pro_gbs / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
                                     "bytes_per_launch": prologue_bytes(w), "peak_source": peak_src}
    line.update(side)
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


def run_ulysses(args):
    """Ulysses sequence parallelism over the ranks of this job: every rank holds a
    contiguous token shard of ONE clip (the first N mod P ranks one token more);
    per step, the prologue of the shard into per-head-group send blocks, an
    all-to-all to head shards, attention over all N tokens of H/P heads, and an
    all-to-all back.  Strong scaling: the clip's FLOPs are shared by all ranks."""
    import torch
    import torch.distributed as dist

    import video_diffusion_transformer_h3attn_b200 as h3
    from video_diffusion_transformer_h3attn_b200 import inputs, ulysses

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    args.gpus = world
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    w = inputs.workload(args.workload)
    dev = torch.device("cuda", local)
    N, H, dd = w.total, w.n_heads, w.head_dim
    sizes = [N // world + (1 if r < N % world else 0) for r in range(world)]
    lo = sum(sizes[:rank])
    host = host_inputs(w, rows=slice(lo, lo + sizes[rank]))
    d = {k: v.to(dev) for k, v in host.items()}
    cu = None
    if len(w.seqlens) > 1:
        cu = torch.from_numpy(np.ascontiguousarray(w.cu_seqlens, dtype=np.int32)).to(dev)
    stream = torch.cuda.current_stream()

    def step():
        return ulysses.ulysses_attention(d["q"], d["k"], d["v"], sizes, gamma_q=d.get("gq"), gamma_k=d.get("gk"),
                                         eps=w.eps, pos=d.get("pos"), kind=d.get("kind"), sections=w.sections,
                                         theta=w.theta, cu_seqlens=cu, max_seqlen=w.max_seqlen)

    for _ in range(args.warmup):
        step()
    h3.device_status()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    h3.device_status()
    ms = reduce_max(t0.elapsed_time(t1) / args.steps, world, dev)
    flops = w.attention_flops()
    row_bytes = H * dd * 2
    n_r = sizes[rank]
    line = {
        "metric": METRIC, "value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, world, parallel="ulysses"),
        "all_to_all_bytes_per_rank": {
            "before_attention": 3 * n_r * row_bytes * (world - 1) // world,
            "after_attention": n_r * row_bytes * (world - 1) // world,
            "note": "rank 0's shard; Q', K', V sent to the other ranks' head groups, O returned"},
        "e2e": None,
        "gpu_launches": None,
        "clocks": clocks.summary(),
        "note": "one clip split over the ranks by tokens; the exchange goes through NCCL all-to-all "
                "(a copy on one rank)",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


TABLE_WORKLOADS = ("tiny", "small", "joint", "2k", "ragged")
TABLE_SAMPLED_ROWS = {"2k": 2048}  # the full fp64 oracle of the 2k clip takes hours on a host


def run_table(args):
    """One JSON line per workload: the step's TFLOP/s against the datasheet and the
    measured peaks, the prologue's GB/s, the error against the fp64 oracle and the
    oracle's own time on this host's cores (full for every workload but the 2k
    clip, which is compared and timed on 2,048 query rows x all heads that visit
    every query tile, then extrapolated)."""
    import torch

    import oracle
    import video_diffusion_transformer_h3attn_b200 as h3
    from video_diffusion_transformer_h3attn_b200 import inputs

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()
    orc = oracle.get()
    names = TABLE_WORKLOADS if args.table == "all" else tuple(args.table.split(","))
    for name in names:
        w = inputs.workload(name)
        host = host_inputs(w)
        d = {k: v.to(dev) for k, v in host.items()}
        b = step_buffers(w, d)
        ms, pro_ms, att_ms = timed_steps(h3, w, d, b, stream, args.warmup, args.steps)
        run_step(h3, w, d, b)
        h3.device_status()
        gpu_o = b["o"].view(torch.int16).cpu().numpy().view(np.uint16)
        gpu_qp = b["qp"].view(torch.int16).cpu().numpy().view(np.uint16) if w.has_prologue else None
        gpu_kp = b["kp"].view(torch.int16).cpu().numpy().view(np.uint16) if w.has_prologue else None
        del d, b
        torch.cuda.empty_cache()

        t0 = time.perf_counter()
        (_, q16), (_, k16) = orc.prologue_workload(w)
        t_pro = time.perf_counter() - t0
        max_ulp = None
        if w.has_prologue:
            def ordered(x):
                x = x.astype(np.int32)
                return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
            max_ulp = int(max(np.abs(ordered(gpu_qp) - ordered(q16)).max(),
                              np.abs(ordered(gpu_kp) - ordered(k16)).max()))
        # the attention kernel alone on the oracle's own Q', K' (the same inputs on both sides)
        dq = {"q": _bf16(q16).to(dev), "k": _bf16(k16).to(dev), "v": _bf16(w.v).to(dev)}
        if len(w.seqlens) > 1:
            o_same = h3.attention_varlen(dq["q"], dq["k"], dq["v"], torch.from_numpy(
                np.ascontiguousarray(w.cu_seqlens, dtype=np.int32)).to(dev), w.max_seqlen)
        else:
            o_same = h3.attention(dq["q"], dq["k"], dq["v"])
        h3.device_status()
        gpu_o_same = o_same.view(torch.int16).cpu().numpy().view(np.uint16)
        del dq, o_same
        torch.cuda.empty_cache()
        n_rows = TABLE_SAMPLED_ROWS.get(name)
        rows = None if n_rows is None else inputs.sample_rows_every_tile(w.cu_seqlens, n_rows, seed=w.seed + 1000)
        t0 = time.perf_counter()
        ro, _ = orc.attention(q16, k16, w.v, w.cu_seqlens, rows=rows)
        t_att = time.perf_counter() - t0
        # the error beyond half a bf16 ulp of the exact value (what storing even the
        # correctly rounded result in bf16 costs)
        _, ex = np.frexp(np.maximum(np.abs(ro), 2.0 ** -126))
        half_ulp = np.ldexp(1.0, ex - 9)

        def errors(bits):
            got = (bits if rows is None else bits[rows]).astype(np.uint32) << 16
            e = np.abs(got.view(np.float32).astype(np.float64) - ro)
            return e, np.maximum(e - half_ulp, 0.0)

        err, excess = errors(gpu_o)
        err_same, excess_same = errors(gpu_o_same)
        frac = 1.0 if rows is None else len(rows) / w.total
        oracle_s = t_pro + t_att / frac
        tf = w.attention_flops() / (ms * 1e-3) / 1e12
        line = {
            "table": name, "config": workload_config(w, 1), "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "tflops": tf,
            "pct_of_datasheet_2250": 100.0 * tf / DATASHEET_BF16_TFLOPS,
            "pct_of_measured_burst": 100.0 * tf / peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
            "pct_of_measured_sustained": 100.0 * tf / peaks.get("bf16_tflops_sustained",
                                                                 FALLBACK_PEAKS["bf16_tflops_sustained"]),
            "attention_ms": att_ms, "attention_tflops": w.attention_flops() / (att_ms * 1e-3) / 1e12,
            "prologue_ms": pro_ms if w.has_prologue else None,
            "prologue_gbs": prologue_bytes(w) / (pro_ms * 1e-3) / 1e9 if w.has_prologue else None,
            "prologue_max_ulp": max_ulp,
            "max_abs": float(err.max()), "mean_abs": float(err.mean()),
            "max_abs_beyond_half_ulp": float(excess.max()),
            "n_over_1e-2": int(np.sum(err > 1e-2)), "n_over_1e-2_beyond_half_ulp": int(np.sum(excess > 1e-2)),
            "n_compared": int(err.size),
            "errors_above": "the step end to end: GPU prologue + attention against the oracle's prologue + attention",
            "attention_same_inputs": {
                "max_abs": float(err_same.max()), "mean_abs": float(err_same.mean()),
                "max_abs_beyond_half_ulp": float(excess_same.max()),
                "n_over_1e-2": int(np.sum(err_same > 1e-2)),
                "n_over_1e-2_beyond_half_ulp": int(np.sum(excess_same > 1e-2)),
                "note": "the attention kernel on the oracle's own Q', K' (identical inputs on both sides)"},
            "compared": "every output" if rows is None else
                        "%d query rows x %d heads visiting every query tile" % (len(rows), w.n_heads),
            "oracle_s": oracle_s,
            "oracle_kind": "full" if rows is None else
                           "prologue of the whole clip + attention of the sampled rows, extrapolated",
            "oracle_tflops": w.attention_flops() / oracle_s / 1e12,
            "cores": _cores_used(), "peak_source": peak_src,
        }
        print(json.dumps(line), flush=True)
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
    ap.add_argument("--no-side", action="store_true",
                    help="skip the side measurements (merge, fused projection, block-sparse)")
    ap.add_argument("--workload", default=WORKLOAD, choices=TABLE_WORKLOADS,
                    help="workload of the step (default: the 2K refine clip)")
    ap.add_argument("--parallel", choices=["replicas", "ulysses"], default="replicas",
                    help="replicas: every rank its own clip (weak scaling); ulysses: one clip split "
                         "over the ranks by tokens, all-to-all to head shards (strong scaling)")
    ap.add_argument("--table", nargs="?", const="all", default=None,
                    help="one line per workload (comma-separated names, default all) with the error "
                         "against the oracle and the oracle's time")
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
    if args.table:
        return run_table(args)
    if args.parallel == "ulysses":
        return run_ulysses(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
