"""Host-side pieces of bench.py (no GPU): the oracle sample behind cpu_baseline and
the reference arm, the prologue's algorithmic bytes, and the workload lines."""
import numpy as np
import pytest

import bench
from video_diffusion_transformer_h3attn_b200 import inputs


@pytest.mark.parametrize("lens,H", [([1000], 4), ([130, 1, 500, 257], 3)])
def test_sample_pairs_visit_every_tile_with_heads_in_turn(lens, H):
    w = inputs.make_workload("bench_host", lens, H, 64, seed=4, norm=False)
    rows, heads = bench.sample_pairs(w, 64, seed=9)
    assert len(rows) == len(heads) >= min(64, w.total)
    assert np.all(np.diff(rows) > 0)
    assert np.array_equal(heads, np.arange(len(rows)) % H)
    for s in range(len(lens)):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        for t0 in range(a, b, 128):
            assert np.any((rows >= t0) & (rows < min(t0 + 128, b)))


def test_oracle_pairs_count_the_keys_of_each_pairs_sequence():
    """A sampled (row, head) pair costs 4 d FLOP per key of its own sequence."""
    import oracle
    orc = oracle.get()
    lens = [100, 37, 200]
    w = inputs.make_workload("bench_host2", lens, 2, 64, seed=5, norm=False)
    rows, heads = bench.sample_pairs(w, 24, seed=1)
    flops = bench.oracle_pairs(w, orc, w.k, rows, heads)
    seq = np.searchsorted(w.cu_seqlens, rows, side="right") - 1
    assert flops == 4.0 * w.head_dim * float(np.sum(np.asarray(lens)[seq]))


def test_prologue_bytes_and_workload_lines():
    w = inputs.workload("small")
    assert bench.prologue_bytes(w) == 4.0 * 3072 * 24 * 128 * 2 + 13 * 3072 + 4 * 128
    for name in bench.TABLE_WORKLOADS:
        cfg = bench.workload_config(inputs.workload(name) if name in ("tiny", "small") else
                                    type("W", (), {"name": name, "total": 1, "n_heads": 1, "head_dim": 64})(), 1)
        assert cfg["workload"] == bench.WORKLOAD_TEXT[name] and cfg["parallelism"] == "replicas"
    ul = bench.workload_config(w, 4, parallel="ulysses")
    assert ul["parallelism"] == "ulysses4" and ul["global_batch"] == 1
