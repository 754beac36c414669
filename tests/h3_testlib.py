"""Helpers shared by the GPU parity tests: moving bf16 bit patterns to CUDA,
comparing against the fp64 oracle, and the tolerances.

Tolerances (written here once, used by every parity test):
  prologue   every output within 1 bf16 ulp of the correctly rounded oracle value
             (|ordered(bits_gpu) - ordered(bf16(oracle))| <= 1);
  attention  the error beyond the half-ulp that storing the exact value as bf16
             costs by itself, e = max(0, |o_gpu - o_ref| - ulp_bf16(o_ref)/2), has
             max <= 1e-2 and mean <= 1e-3 (for |o| >= 4 that half ulp alone exceeds
             1e-2; for rows over a few keys |o| ~ 1 and it averages ~2e-3, above the
             mean bound, even for the exactly rounded output);
             strict=True also requires the plain mean |o_gpu - o_ref| <= 1e-3
             and (unless plain_max=False) the plain max <= 1e-2: used for the five
             named workloads, the one-rank Ulysses path and every sequence of 64
             keys or more, where |o| is small enough that the plain bounds are
             attainable.  The ragged workload (Q x 4: peaked rows that reproduce one
             value row, |o| up to ~4) keeps the plain mean but not the plain max:
             there the correctly rounded exact output alone is 0.0078 from the
             fp64 value, leaving no room for the rounding of the weights;
  lse        |lse_gpu - lse_ref| <= 1e-3 (fp32 output).
"""
from __future__ import annotations

import numpy as np

PROLOGUE_MAX_ULP = 1
ATTN_MAX_ABS = 1e-2
ATTN_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_cuda_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_cuda_bf16(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def ordered(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns mapped to integers that order like the values (+0 == -0)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    return np.abs(ordered(a_bits) - ordered(b_bits))


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(np.maximum(ax, 2.0 ** -126))  # ax in [2^(e-1), 2^e)
    return np.ldexp(1.0, e - 1 - 7) / 2.0


def check_prologue(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str) -> dict:
    d = ulp_distance(gpu_bits, ref_bits)
    stats = {"n": int(d.size), "exact": int(np.sum(d == 0)), "max_ulp": int(d.max()) if d.size else 0}
    assert stats["max_ulp"] <= PROLOGUE_MAX_ULP, "%s: %s (worst at %s)" % (
        what, stats, np.unravel_index(int(np.argmax(d)), d.shape))
    return stats


def check_attention(o_gpu: np.ndarray, o_ref: np.ndarray, what: str, lse_gpu=None, lse_ref=None,
                    strict: bool = False, plain_max=None) -> dict:
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    err = np.abs(o_gpu - o_ref)
    excess = np.maximum(err - bf16_half_ulp(o_ref), 0.0)
    stats = {"max_abs": float(err.max()), "mean_abs": float(err.mean()),
             "max_excess": float(excess.max()), "mean_excess": float(excess.mean())}
    assert np.all(np.isfinite(o_gpu)), "%s: non-finite output" % what
    assert stats["max_excess"] <= ATTN_MAX_ABS, "%s: %s at %s" % (
        what, stats, np.unravel_index(int(np.argmax(excess)), excess.shape))
    assert stats["mean_excess"] <= ATTN_MEAN_ABS, "%s: %s" % (what, stats)
    if strict:
        assert stats["mean_abs"] <= ATTN_MEAN_ABS, "%s (strict): %s" % (what, stats)
    if strict if plain_max is None else plain_max:
        assert stats["max_abs"] <= ATTN_MAX_ABS, "%s (strict): %s" % (what, stats)
    if lse_gpu is not None:
        le = np.abs(np.asarray(lse_gpu, dtype=np.float64) - lse_ref)
        stats["lse_max_abs"] = float(le.max())
        assert stats["lse_max_abs"] <= LSE_MAX_ABS, "%s lse: %s" % (what, stats)
    return stats
