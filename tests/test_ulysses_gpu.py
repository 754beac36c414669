"""The GPU side of Ulysses sequence parallelism on one GPU.

The multi-rank exchange itself is covered on CPU ranks (tests/test_ulysses.py).
Here the CUDA kernels are checked for the two properties that make the P-rank
output equal the one-rank output bit for bit:
  * the prologue applied to one head group of a shard (a strided view) and
    written into that group's send block gives the same bits as the prologue of
    the whole tensor, sliced;
  * attention over a subset of the heads gives the same bits as those heads of
    the attention over all heads;
and the one-rank path of ulysses_attention matches the fp64 oracle (and equals
the direct calls bit for bit)."""
import numpy as np
import pytest

from h3_testlib import to_cuda_bf16
from video_diffusion_transformer_h3attn_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import video_diffusion_transformer_h3attn_b200 as mod
    return mod


def _joint_like(n_video_grid=(4, 12, 16), n_audio=40, H=24, d=128, seed=41):
    pos, kind = inputs.video_layout(*n_video_grid, n_audio=n_audio)
    return inputs.make_workload("ulysses_gpu", [len(kind)], H, d, seed, pos=pos, kind=kind)


@pytest.mark.parametrize("world", [2, 3, 4, 8])
def test_prologue_into_head_group_blocks(h3, world):
    import torch
    w = _joint_like()
    q, k = to_cuda_bf16(w.q), to_cuda_bf16(w.k)
    g = (to_cuda_bf16(w.gamma_q), to_cuda_bf16(w.gamma_k))
    pos, kind = torch.from_numpy(w.pos).cuda(), torch.from_numpy(w.kind).cuda()
    full_q, full_k = h3.prologue(q, k, gamma_q=g[0], gamma_k=g[1], pos=pos, kind=kind)
    n, H, d = q.shape
    Hp = H // world
    send_q = torch.empty((world, n, Hp, d), dtype=q.dtype, device=q.device)
    send_k = torch.empty_like(send_q)
    for p in range(world):
        hs = slice(p * Hp, (p + 1) * Hp)
        h3.prologue(q[:, hs], k[:, hs], send_q[p], send_k[p], g[0], g[1], pos=pos, kind=kind)
    h3.device_status()
    for p in range(world):
        hs = slice(p * Hp, (p + 1) * Hp)
        assert torch.equal(send_q[p], full_q[:, hs]) and torch.equal(send_k[p], full_k[:, hs])


@pytest.mark.parametrize("world", [2, 3, 8])
def test_head_subset_attention_is_bitwise_identical(h3, world):
    import torch
    w = inputs.random_case([3000], 24, 128, seed=43)
    q, k, v = to_cuda_bf16(w.q), to_cuda_bf16(w.k), to_cuda_bf16(w.v)
    full = h3.attention(q, k, v)
    Hp = 24 // world
    for p in range(world):
        hs = slice(p * Hp, (p + 1) * Hp)
        part = h3.attention(q[:, hs].contiguous(), k[:, hs].contiguous(), v[:, hs].contiguous())
        assert torch.equal(part, full[:, hs]), "head group %d differs" % p
    h3.device_status()


@pytest.mark.parametrize("seqlens", [None, [300, 1, 507]])
def test_ulysses_one_rank_matches_the_oracle(h3, seqlens):
    """The whole one-rank Ulysses step (prologue into the send blocks, the
    exchange, attention, the return exchange) against the oracle's prologue and
    attention of the same inputs, under the benchmark spec's tolerances; and bit for bit
    the same as the direct calls."""
    import torch
    import oracle
    from h3_testlib import bf16_bits_to_f64, check_attention, from_cuda_bf16
    from video_diffusion_transformer_h3attn_b200 import ulysses
    w = _joint_like()
    n = w.q.shape[0]
    lens = [n] if seqlens is None else seqlens
    assert sum(lens) == n
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v = to_cuda_bf16(w.q), to_cuda_bf16(w.k), to_cuda_bf16(w.v)
    g = (to_cuda_bf16(w.gamma_q), to_cuda_bf16(w.gamma_k))
    pos, kind = torch.from_numpy(w.pos).cuda(), torch.from_numpy(w.kind).cuda()
    cu_t = None if seqlens is None else torch.from_numpy(cu).cuda()
    o = ulysses.ulysses_attention(q, k, v, [n], gamma_q=g[0], gamma_k=g[1], pos=pos, kind=kind,
                                  cu_seqlens=cu_t, max_seqlen=max(lens))
    h3.device_status()
    orc = oracle.get()
    (_, rq), (_, rk) = orc.prologue_workload(w)
    ro, _ = orc.attention(rq, rk, w.v, cu)
    check_attention(bf16_bits_to_f64(from_cuda_bf16(o)), ro, "ulysses one rank", strict=True)
    qp, kp = h3.prologue(q, k, gamma_q=g[0], gamma_k=g[1], pos=pos, kind=kind)
    if seqlens is None:
        ref = h3.attention(qp, kp, v)
    else:
        ref = h3.attention_varlen(qp, kp, v, cu_t, max(lens))
    h3.device_status()
    assert torch.equal(o, ref)


def _staged_exchange(dst, src, out_splits, in_splits, group=None):
    """all_to_all_single for a gloo group: device tensors go through host memory."""
    import torch
    import torch.distributed as dist
    host_dst = torch.empty(dst.shape, dtype=dst.dtype)
    dist.all_to_all_single(host_dst, src.cpu(), out_splits, in_splits, group=group)
    dst.copy_(host_dst)


def _gpu_rank(rank, world, port, seqlens, out):
    """One rank on cuda:0: its token shard through the library's kernels, the two
    exchanges through gloo (host staging); no kernel waits on another rank."""
    import os
    from datetime import timedelta
    import torch
    import torch.distributed as dist
    import video_diffusion_transformer_h3attn_b200 as h3
    from video_diffusion_transformer_h3attn_b200 import ulysses
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w = _joint_like()
        sizes = ulysses.shard_sizes(w.q.shape[0], world)
        off = ulysses.shard_offsets(sizes)
        sl = slice(off[rank], off[rank + 1])
        cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
        o = ulysses.ulysses_attention(
            to_cuda_bf16(w.q[sl]), to_cuda_bf16(w.k[sl]), to_cuda_bf16(w.v[sl]), sizes,
            gamma_q=to_cuda_bf16(w.gamma_q), gamma_k=to_cuda_bf16(w.gamma_k),
            pos=torch.from_numpy(np.ascontiguousarray(w.pos[sl])).cuda(),
            kind=torch.from_numpy(np.ascontiguousarray(w.kind[sl])).cuda(),
            cu_seqlens=torch.from_numpy(cu).cuda() if len(seqlens) > 1 else None, max_seqlen=max(seqlens),
            exchange_fn=_staged_exchange)
        h3.device_status()
        out[rank] = o.view(torch.int16).cpu().numpy().copy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,seqlens", [(2, [808]), (3, [808]), (2, [300, 1, 507])])
def test_ulysses_ranks_on_one_gpu_match_one_rank_and_the_oracle(h3, world, seqlens):
    """Output parity above one rank for the CUDA path: P processes on cuda:0, each
    with a ragged token shard, run the library's prologue and attention kernels; the
    exchanges go through gloo with host staging (one GPU has no second NCCL peer).
    Every shard equals the matching rows of the one-rank kernel output bit for bit
    and matches the fp64 oracle under the benchmark spec's bounds."""
    import socket
    import torch
    import torch.multiprocessing as mp
    import oracle
    from h3_testlib import bf16_bits_to_f64, check_attention
    from video_diffusion_transformer_h3attn_b200 import ulysses
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_gpu_rank, args=(world, port, seqlens, out), nprocs=world, join=True)
    w = _joint_like()
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    q, k, v = to_cuda_bf16(w.q), to_cuda_bf16(w.k), to_cuda_bf16(w.v)
    g = (to_cuda_bf16(w.gamma_q), to_cuda_bf16(w.gamma_k))
    pos, kind = torch.from_numpy(w.pos).cuda(), torch.from_numpy(w.kind).cuda()
    qp, kp = h3.prologue(q, k, gamma_q=g[0], gamma_k=g[1], pos=pos, kind=kind)
    ref = h3.attention(qp, kp, v) if len(seqlens) == 1 else \
        h3.attention_varlen(qp, kp, v, torch.from_numpy(cu).cuda(), max(seqlens))
    h3.device_status()
    ref_bits = ref.view(torch.int16).cpu().numpy()
    off = ulysses.shard_offsets(ulysses.shard_sizes(w.q.shape[0], world))
    got = np.concatenate([out[r] for r in range(world)], axis=0)
    for r in range(world):
        assert np.array_equal(out[r], ref_bits[off[r]:off[r + 1]]), "rank %d differs from the one-rank run" % r
    orc = oracle.get()
    (_, rq), (_, rk) = orc.prologue_workload(w)
    ro, _ = orc.attention(rq, rk, w.v, cu)
    check_attention(bf16_bits_to_f64(got.view(np.uint16)), ro, "ulysses %d ranks" % world, strict=True)
