"""Property-based checks (hypothesis) of the host-side logic: the Ulysses shard
plan, the block-sparse list generator and the input generator's bf16 rounding."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from video_diffusion_transformer_h3attn_b200 import inputs, ulysses


@given(st.integers(0, 10 ** 6), st.integers(1, 64))
def test_shards_cover_the_sequence_contiguously(n, world):
    sizes = ulysses.shard_sizes(n, world)
    off = ulysses.shard_offsets(sizes)
    assert len(sizes) == world and sum(sizes) == n
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    assert off[0] == 0 and off[-1] == n and all(off[i + 1] - off[i] == sizes[i] for i in range(world))


@settings(max_examples=40, deadline=None)
@given(st.integers(1, 2), st.integers(1, 3), st.integers(1, 900), st.integers(1, 900),
       st.floats(0.0, 1.0), st.booleans(), st.integers(0, 5), st.integers(0, 2 ** 31 - 1))
def test_block_lists_hold_their_invariants(B, H, nq, nk, keep, diagonal, empty_every, seed):
    off, idx = inputs.block_lists(B, H, nq, nk, keep, seed, diagonal=diagonal, empty_every=empty_every)
    n_qb, n_kb = -(-nq // 256), -(-nk // 128)
    assert off.shape == (B * H * n_qb + 1,) and off[0] == 0 and np.all(np.diff(off) >= 0)
    assert off[-1] == idx.size
    for c in range(B * H * n_qb):
        lst = idx[off[c]:off[c + 1]]
        assert np.all(np.diff(lst) > 0) and (lst.size == 0 or (lst[0] >= 0 and lst[-1] < n_kb))
        if empty_every and c % empty_every == 0:
            assert lst.size == 0
        elif keep >= 1.0:
            assert lst.size == n_kb


@given(st.floats(-2.0 ** 127, 2.0 ** 127, allow_nan=False, width=32))
def test_bf16_rounding_is_nearest(x):
    b = int(inputs.f32_to_bf16_bits(np.array([x], dtype=np.float32))[0])
    got = float(inputs.bf16_bits_to_f32(np.array([b], dtype=np.uint16))[0])
    # the neighbours of the chosen pattern are no closer to x (ties to the even pattern)
    for nb in (b - 1, b + 1):
        if 0 <= nb <= 0xFFFF and (nb & 0x7F80) != 0x7F80:
            other = float(inputs.bf16_bits_to_f32(np.array([nb], dtype=np.uint16))[0])
            if np.sign(other) == np.sign(got) or other == 0.0:
                assert abs(got - x) <= abs(other - x)
