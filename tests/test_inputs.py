"""The seeded input generator: determinism, shapes and layout of the workloads."""
import numpy as np
import pytest

from video_diffusion_transformer_h3attn_b200 import inputs


def test_bf16_conversion_round_trip_and_ties():
    x = np.array([1.0, -2.5, 1.00390625, 1.005859375, 3.0e38, 0.0], dtype=np.float32)
    b = inputs.f32_to_bf16_bits(x)
    # 1.00390625 is the midpoint of 1 and 1+2^-7: ties go to the even pattern (1.0)
    assert list(b[:3]) == [0x3F80, 0xC020, 0x3F80]
    # 1.005859375 = 1 + 3*2^-9 is above the midpoint -> rounds up to 1 + 2^-7
    assert b[3] == 0x3F81
    assert np.array_equal(inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(np.float32([0.75]))),
                          np.float32([0.75]))


def test_workloads_are_deterministic_and_shaped():
    a = inputs.workload("tiny")
    b = inputs.workload("tiny")
    assert np.array_equal(a.q, b.q) and np.array_equal(a.v, b.v)
    assert a.q.shape == (256, 2, 64) and a.pos is None and a.gamma_q is None
    s = inputs.workload("small")
    assert s.q.shape == (3072, 24, 128) and s.gamma_q.shape == (128,)
    assert s.pos.shape == (3072, 3) and np.all(s.kind == inputs.KIND_3D)
    # row-major (t, h, w): token 24*16 + 24 + 5 is (1, 1, 5)
    assert tuple(s.pos[24 * 16 + 24 + 5]) == (1, 1, 5)
    g = inputs.bf16_bits_to_f32(s.gamma_q)
    assert g.min() >= 0.5 and g.max() <= 1.5


def test_joint_and_ragged_layouts():
    pos, kind = inputs.video_layout(16, 30, 54, 256)
    assert len(pos) == 26176 and np.all(kind[:25920] == 1) and np.all(kind[25920:] == 2)
    assert np.array_equal(pos[25920:, 0], np.arange(256))
    pos, kind = inputs.ragged_layout([4096, 9000, 17001, 31234])
    assert len(pos) == 61331 and pos[4096, 0] == 0 and pos[4095, 0] == 4095 and pos[-1, 0] == 31233


def test_sample_rows_cover_boundaries():
    cu = np.array([0, 300, 700])
    rows = inputs.sample_rows(cu, 64, seed=1)
    for r in (0, 299, 300, 699, 127, 128, 427, 428):
        assert r in rows
    assert rows.min() >= 0 and rows.max() < 700


def _lists(off, idx):
    return [idx[off[c]:off[c + 1]] for c in range(len(off) - 1)]


def test_block_lists_are_valid_and_seeded():
    B, H, nq, nk = 2, 3, 700, 900
    off, idx = inputs.block_lists(B, H, nq, nk, 0.3, seed=5, empty_every=4)
    n_qb, n_kb = -(-nq // 256), -(-nk // 128)
    assert off.dtype == np.int32 and idx.dtype == np.int32
    assert off.shape == (B * H * n_qb + 1,) and off[0] == 0 and off[-1] == idx.size
    for c, lst in enumerate(_lists(off, idx)):
        assert np.all(np.diff(lst) > 0) and (lst.size == 0 or (lst[0] >= 0 and lst[-1] < n_kb))
        qb = c % n_qb
        if c % 4 == 0:
            assert lst.size == 0
        else:  # the key tiles overlapping the query block's own rows are always listed
            lo, hi = qb * 256 // 128, min(n_kb, -(-min((qb + 1) * 256, nq) // 128))
            assert set(range(lo, hi)) <= set(lst.tolist())
    off2, idx2 = inputs.block_lists(B, H, nq, nk, 0.3, seed=5, empty_every=4)
    assert np.array_equal(off, off2) and np.array_equal(idx, idx2)


def test_block_lists_density_follows_keep():
    off, idx = inputs.block_lists(1, 8, 4096, 65536, 0.25, seed=9, diagonal=False)
    n_kb = 65536 // 128
    share = idx.size / ((len(off) - 1) * n_kb)
    assert abs(share - 0.25) < 0.01
    off1, idx1 = inputs.block_lists(1, 2, 300, 300, 1.0, seed=1)
    assert all(len(lst) == 3 for lst in _lists(off1, idx1))  # every tile of 300 keys


def test_bench_sparse_flops_match_a_mask_count():
    """The benchmark's FLOP count of a block-sparse launch equals 4 d x the number
    of visible (query, key) pairs counted on the dense mask."""
    import bench
    w = inputs.make_workload("sp", [1000], 2, 64, seed=3, norm=False)
    w.seed = 11
    off, idx, flops = bench._sparse_lists(w)
    N, H, d = w.total, w.n_heads, w.head_dim
    n_qp = -(-N // 256)
    mask = np.zeros((H, N, N), dtype=bool)
    for h in range(H):
        for qp in range(n_qp):
            c = h * n_qp + qp
            for t in idx[off[c]:off[c + 1]]:
                mask[h, 256 * qp:256 * (qp + 1), 128 * int(t):128 * (int(t) + 1)] = True
    assert flops == 4.0 * d * int(mask.sum())


@pytest.mark.parametrize("lens", [[129024], [4096, 9000, 17001, 31234], [1, 130, 0, 255, 4, 513, 128], [300]])
def test_sample_rows_every_tile_visits_every_query_tile(lens):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    rows = inputs.sample_rows_every_tile(cu, 64, seed=3)
    assert np.all(np.diff(rows) > 0) and rows[0] >= 0 and rows[-1] < cu[-1]
    for s in range(len(lens)):
        a, b = int(cu[s]), int(cu[s + 1])
        mine = rows[(rows >= a) & (rows < b)]
        for t0 in range(a, b, 128):
            assert np.any((mine >= t0) & (mine < min(t0 + 128, b))), "tile at %d of sequence %d not sampled" % (t0, s)
        if b > a:
            assert a in mine and b - 1 in mine
    assert len(rows) >= min(64, int(cu[-1]))
    assert np.array_equal(rows, inputs.sample_rows_every_tile(cu, 64, seed=3))
