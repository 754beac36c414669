"""Ulysses sequence parallelism for the attention step of the block.

"H3 Runtime Current State" (Implemented And Validated) runs the denoiser with
ragged Ulysses sequence parallelism (2/4/6/8-rank transport tests; the two-GPU
speedup grows with sequence size).  Each of P ranks holds a contiguous shard of
the packed token sequence for all H heads; the shards may differ in length
(ragged: the sequence length need not divide by P).  An all-to-all turns token
shards into head shards -- rank p receives every token of heads
[p*H/P, (p+1)*H/P) -- attention runs over the whole sequence for those heads,
and a second all-to-all returns to every rank its own tokens for all heads.

Per rank and step (the GPU work is this library's kernels; torch.distributed
carries the two exchanges, NCCL on GPUs):
  1. the Q/K RMSNorm + RoPE prologue on the local shard (per-token work), one
     launch per head group writing straight into that group's send block, so
     normalising, rotating and packing are one pass; V is packed by a copy;
  2. all-to-all of Q', K', V (send blocks [P][n_r][H/P][d], receive
     [N][H/P][d] in global token order: the blocks of ranks 0..P-1 are the
     sequence's consecutive token ranges);
  3. attention on [N, H/P, d] (dense, or ragged over cu_seqlens);
  4. all-to-all of O back (token ranges out, head groups in) and unpacking
     into the shard's [n_r, H, d].
Attention of head h reads exactly the bytes a one-rank run reads for head h,
and the kernels compute each (query tile, head) independently, so the P-rank
output equals the one-rank output bit for bit.

Exchanges move 3 * N * H * d * 2 * (P-1)/P^2 bytes out of each rank before
attention and N * H * d * 2 * (P-1)/P^2 after it.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import video_diffusion_transformer_h3attn_b200 as _h3


def shard_sizes(n_tokens: int, world: int) -> List[int]:
    """Contiguous ragged split of n_tokens over `world` ranks: the first
    n_tokens % world ranks hold one token more."""
    if world <= 0 or n_tokens < 0:
        raise ValueError("need world >= 1 and n_tokens >= 0")
    base, extra = divmod(n_tokens, world)
    return [base + (1 if r < extra else 0) for r in range(world)]


def shard_offsets(sizes: Sequence[int]) -> List[int]:
    out, acc = [], 0
    for s in sizes:
        out.append(acc)
        acc += s
    return out + [acc]


def _default_prologue(q_in, k_in, q_out, k_out, gamma_q, gamma_k, eps, pos, kind, sections, theta):
    _h3.prologue(q_in, k_in, q_out, k_out, gamma_q, gamma_k, eps, pos, kind, sections, theta)


def _default_attention(q, k, v, cu_seqlens, max_seqlen, softmax_scale):
    if cu_seqlens is None:
        return _h3.attention(q, k, v, softmax_scale=softmax_scale)
    return _h3.attention_varlen(q, k, v, cu_seqlens, max_seqlen, softmax_scale=softmax_scale)


def ulysses_attention(q, k, v, sizes: Sequence[int], group=None, *, gamma_q=None, gamma_k=None,
                      eps: float = 1e-6, pos=None, kind=None, sections=(32, 48, 48),
                      theta: float = 10000.0, cu_seqlens=None, max_seqlen: Optional[int] = None,
                      softmax_scale: Optional[float] = None,
                      prologue_fn: Optional[Callable] = None, attention_fn: Optional[Callable] = None,
                      exchange_fn: Optional[Callable] = None):
    """Sequence-parallel prologue + attention over P ranks of `group`.

    q, k, v: this rank's token shard [n_r, H, d] (bf16; q and k with equal
    strides).  sizes: every rank's shard length, identical on all ranks
    (sum = N).  gamma_*/pos/kind: the prologue's arguments for the local shard
    (pos/kind index the shard's own tokens).  cu_seqlens (device int32, global
    token offsets, identical on all ranks) selects ragged attention over several
    sequences packed in the N tokens.  Returns this shard's O [n_r, H, d].

    prologue_fn / attention_fn replace the CUDA kernels (tests run the exchange
    on CPU ranks with reference implementations); by default the library's
    kernels run.  exchange_fn(dst, src, out_splits, in_splits, group) replaces
    torch.distributed.all_to_all_single (flat tensors, split sizes in elements),
    e.g. a transport that stages device tensors through host memory for a
    process group whose backend only moves host tensors.
    """
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    sizes = [int(s) for s in sizes]
    if len(sizes) != world:
        raise ValueError("sizes must list one shard length per rank")
    n_r, H, d = q.shape
    if n_r != sizes[rank] or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must be this rank's [sizes[rank], H, d] shard")
    if H % world:
        raise ValueError("the number of heads must divide by the number of ranks")
    Hp = H // world
    N = sum(sizes)
    prologue_fn = prologue_fn or _default_prologue
    attention_fn = attention_fn or _default_attention
    exchange_fn = exchange_fn or dist.all_to_all_single
    dev, dt = q.device, q.dtype

    # 1. prologue fused with the pack: send blocks [P][n_r][Hp][d]
    send_q = torch.empty((world, n_r, Hp, d), dtype=dt, device=dev)
    send_k = torch.empty_like(send_q)
    for p in range(world):
        heads = slice(p * Hp, (p + 1) * Hp)
        if n_r:
            prologue_fn(q[:, heads], k[:, heads], send_q[p], send_k[p], gamma_q, gamma_k, eps, pos,
                        kind, sections, theta)
    if world == 1:
        # one rank: the shard is the whole sequence and every head is local, so
        # nothing moves; attention reads the prologue's output and V in place
        return attention_fn(send_q[0], send_k[0], v, cu_seqlens, max_seqlen, softmax_scale)
    send_v = torch.empty_like(send_q)
    for p in range(world):
        send_v[p].copy_(v[:, p * Hp:(p + 1) * Hp])

    # 2. token shards -> head shards: receive [N][Hp][d] in global token order
    recv = [torch.empty((N, Hp, d), dtype=dt, device=dev) for _ in range(3)]
    out_splits = [s * Hp * d for s in sizes]
    in_splits = [n_r * Hp * d] * world
    for src, dst in zip((send_q, send_k, send_v), recv):
        exchange_fn(dst.view(-1), src.view(-1), out_splits, in_splits, group=group)

    # 3. attention over the whole sequence for this rank's heads
    o_heads = attention_fn(recv[0], recv[1], recv[2], cu_seqlens, max_seqlen, softmax_scale)

    # 4. head shards -> token shards, then unpack to [n_r][H][d]
    back = torch.empty((world, n_r, Hp, d), dtype=dt, device=dev)
    exchange_fn(back.view(-1), o_heads.contiguous().view(-1), in_splits, out_splits, group=group)
    o = torch.empty((n_r, H, d), dtype=dt, device=dev)
    for p in range(world):
        o[:, p * Hp:(p + 1) * Hp].copy_(back[p])
    return o
