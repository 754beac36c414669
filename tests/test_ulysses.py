"""Ulysses sequence parallelism on CPU ranks (gloo): the exchange, packing and
unpacking of video_diffusion_transformer_h3attn_b200.ulysses, with the oracle
standing in for the prologue and attention kernels.

Every rank's output shard must equal the matching rows of a one-rank run bit for
bit, for ragged shard sizes (the token count does not divide by the number of
ranks), 2 and 3 ranks, and one or several packed sequences."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from video_diffusion_transformer_h3attn_b200 import inputs, ulysses


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _oracle_prologue(q_in, k_in, q_out, k_out, gamma_q, gamma_k, eps, pos, kind, sections, theta):
    import oracle
    orc = oracle.get()
    g = lambda t: None if t is None else _bits(t)
    p = None if pos is None else pos.numpy()
    kd = None if kind is None else kind.numpy()
    _, yq = orc.rmsnorm_rope(_bits(q_in), g(gamma_q), eps, p, kd, sections, theta, want_f64=False)
    _, yk = orc.rmsnorm_rope(_bits(k_in), g(gamma_k), eps, p, kd, sections, theta, want_f64=False)
    q_out.copy_(_tensor(yq))
    k_out.copy_(_tensor(yk))


def _oracle_attention(q, k, v, cu_seqlens, max_seqlen, softmax_scale):
    import oracle
    orc = oracle.get()
    cu = [0, q.shape[0]] if cu_seqlens is None else cu_seqlens.numpy()
    o, _ = orc.attention(_bits(q), _bits(k), _bits(v), cu, softmax_scale)
    return _tensor(orc.bf16_round(o))


def _case(seqlens, H, d, seed):
    w = inputs.make_workload("ulysses%d" % seed, list(seqlens), H, d, seed, norm=True)
    pos = np.zeros((w.total, 3), dtype=np.int32)
    pos[:, 0] = np.arange(w.total) % 7
    pos[:, 1] = (np.arange(w.total) // 7) % 5
    pos[:, 2] = np.arange(w.total) // 35
    kind = (np.arange(w.total) % 3).astype(np.uint8)  # none, 3D and 1D tokens mixed
    return w, pos, kind


def _worker(rank, world, port, seqlens, H, d, seed, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, pos, kind = _case(seqlens, H, d, seed)
        sizes = ulysses.shard_sizes(w.total, world)
        off = ulysses.shard_offsets(sizes)
        sl = slice(off[rank], off[rank + 1])
        sections = (d // 4, 3 * d // 8, 3 * d // 8)
        cu = torch.from_numpy(np.asarray(w.cu_seqlens, dtype=np.int32)) if len(seqlens) > 1 else None
        o = ulysses.ulysses_attention(
            _tensor(w.q[sl]), _tensor(w.k[sl]), _tensor(w.v[sl]), sizes,
            gamma_q=_tensor(w.gamma_q), gamma_k=_tensor(w.gamma_k), eps=1e-6,
            pos=torch.from_numpy(pos[sl]), kind=torch.from_numpy(kind[sl]), sections=sections,
            cu_seqlens=cu, max_seqlen=max(seqlens), prologue_fn=_oracle_prologue,
            attention_fn=_oracle_attention)
        out[rank] = _bits(o).copy()
    finally:
        dist.destroy_process_group()


def _one_rank(seqlens, H, d, seed):
    w, pos, kind = _case(seqlens, H, d, seed)
    sections = (d // 4, 3 * d // 8, 3 * d // 8)
    q, k = torch.empty(w.q.shape, dtype=torch.bfloat16), torch.empty(w.k.shape, dtype=torch.bfloat16)
    _oracle_prologue(_tensor(w.q), _tensor(w.k), q, k, _tensor(w.gamma_q), _tensor(w.gamma_k), 1e-6,
                     torch.from_numpy(pos), torch.from_numpy(kind), sections, 10000.0)
    cu = torch.from_numpy(np.asarray(w.cu_seqlens, dtype=np.int32)) if len(seqlens) > 1 else None
    return _bits(_oracle_attention(q, k, _tensor(w.v), cu, max(seqlens), None))


@pytest.mark.parametrize("world,seqlens", [(2, [37]), (3, [37]), (2, [20, 1, 30]), (3, [64])])
def test_ulysses_matches_one_rank_bit_for_bit(world, seqlens):
    H, d, seed = 6, 16, 11
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), seqlens, H, d, seed, out), nprocs=world, join=True)
    ref = _one_rank(seqlens, H, d, seed)
    off = ulysses.shard_offsets(ulysses.shard_sizes(sum(seqlens), world))
    for r in range(world):
        got = out[r]
        assert got.shape == ref[off[r]:off[r + 1]].shape
        assert np.array_equal(got, ref[off[r]:off[r + 1]]), "rank %d differs from the one-rank run" % r


def test_shard_sizes_are_ragged_and_contiguous():
    assert ulysses.shard_sizes(10, 4) == [3, 3, 2, 2]
    assert ulysses.shard_sizes(8, 4) == [2, 2, 2, 2]
    assert ulysses.shard_sizes(3, 4) == [1, 1, 1, 0]
    assert ulysses.shard_offsets([3, 3, 2, 2]) == [0, 3, 6, 8, 10]
    with pytest.raises(ValueError):
        ulysses.shard_sizes(5, 0)
