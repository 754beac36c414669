"""Parity of block-sparse attention with the fp64 oracle.

Each group of 256 query rows sees only its listed tiles of 128 keys (CSR lists
from the shared seeded generator).  The kernel is compared with the oracle's
block-sparse attention on the same bf16 inputs and lists, with the attention
tolerances; every tile listed must reproduce the dense kernel bit for bit (the
same arithmetic in the same order); empty lists give the empty sum; lists that
break the rules are reported by the device status and leave the context usable."""
import numpy as np
import pytest

import oracle
from h3_testlib import bf16_bits_to_f64, check_attention, from_cuda_bf16, to_cuda_bf16
from video_diffusion_transformer_h3attn_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import video_diffusion_transformer_h3attn_b200 as mod
    return mod


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


def _case(B, nq, nk, H, d, seed):
    """q [B, nq, H, d] and k, v [B, nk, H, d] bf16 bits from the shared generator."""
    n = max(nq, nk, 1)
    w = inputs.random_case([n] * B, H, d, seed)
    shape = (B, n, H, d)
    return (w.q.reshape(shape)[:, :nq].copy(), w.k.reshape(shape)[:, :nk].copy(),
            w.v.reshape(shape)[:, :nk].copy())


def _cuda_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _run(h3, q, k, v, off, idx):
    o, l = h3.attention_block_sparse(to_cuda_bf16(q), to_cuda_bf16(k), to_cuda_bf16(v), _cuda_i32(off),
                                     _cuda_i32(idx), return_lse=True)
    h3.device_status()
    return from_cuda_bf16(o), l.cpu().numpy()


def _compare(o, lse, ro, rl, what):
    """o [B, nq, H, d] bits, lse [B, H, nq] vs the oracle's [B*nq, H, d], [B*nq, H]."""
    B, nq, H, d = o.shape
    og = bf16_bits_to_f64(o).reshape(B * nq, H, d)
    lg = lse.transpose(0, 2, 1).reshape(B * nq, H).astype(np.float64)
    empty = np.isneginf(rl)
    assert np.array_equal(np.isneginf(lg), empty), "%s: rows without keys differ" % what
    assert np.all(og[empty] == 0.0), "%s: rows without keys must be 0" % what
    check_attention(og[~empty], ro[~empty], what, lg[~empty], rl[~empty], strict=True)


@pytest.mark.parametrize("B,nq,nk,H,d,keep,seed", [
    (1, 700, 900, 2, 128, 0.4, 1),     # ragged query pairs and key tiles
    (2, 513, 385, 2, 64, 0.5, 2),      # head_dim 64, batch 2, 4 key tiles (last holds 1 key)
    (1, 1024, 2000, 2, 128, 0.2, 3),   # 16 key tiles, sparse
    (1, 300, 129, 3, 128, 0.5, 4),     # last key tile of one key
    (1, 256, 128, 2, 128, 1.0, 5),     # exact tiles, everything listed
])
def test_block_sparse_vs_oracle(h3, orc, B, nq, nk, H, d, keep, seed):
    q, k, v = _case(B, nq, nk, H, d, seed=900 + seed)
    off, idx = inputs.block_lists(B, H, nq, nk, keep, seed=seed, diagonal=(seed % 2 == 1),
                                  empty_every=5 if keep < 1.0 else 0)
    o, lse = _run(h3, q, k, v, off, idx)
    ro, rl = orc.attention_block_sparse(q, k, v, off, idx, 256, 128)
    _compare(o, lse, ro, rl, "block-sparse B%d %dx%d d%d keep %.1f" % (B, nq, nk, d, keep))


@pytest.mark.parametrize("nq,nk,d", [(700, 900, 128), (513, 385, 64)])
def test_every_tile_listed_is_dense_bitwise(h3, nq, nk, d):
    """With every key tile listed the kernel runs the dense schedule: identical bits."""
    q, k, v = _case(1, nq, nk, 2, d, seed=950 + nq)
    n_qp, n_kt = -(-nq // 256), -(-nk // 128)
    off = np.arange(0, 2 * n_qp * n_kt + 1, n_kt, dtype=np.int32)
    idx = np.tile(np.arange(n_kt, dtype=np.int32), 2 * n_qp)
    o, lse = _run(h3, q, k, v, off, idx)
    od, ld = h3.attention_kv(to_cuda_bf16(q), to_cuda_bf16(k), to_cuda_bf16(v), return_lse=True)
    h3.device_status()
    assert np.array_equal(o, from_cuda_bf16(od)), "every tile listed: O differs from the dense kernel"
    assert np.array_equal(lse, ld.cpu().numpy()), "every tile listed: LSE differs from the dense kernel"


def test_empty_lists_give_empty_sum(h3):
    import torch
    q, k, v = _case(1, 600, 500, 2, 128, seed=977)
    n_lists = 2 * 3
    off = np.zeros(n_lists + 1, dtype=np.int32)
    o0 = torch.full((1, 600, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    o, l = h3.attention_block_sparse(to_cuda_bf16(q), to_cuda_bf16(k), to_cuda_bf16(v), _cuda_i32(off),
                                     _cuda_i32(np.zeros(0, np.int32)), o=o0, return_lse=True)
    h3.device_status()
    assert torch.all(o == 0), "empty lists: O must be the empty sum (0)"
    assert torch.all(torch.isneginf(l)), "empty lists: LSE must be -inf"


@pytest.mark.parametrize("bad", ["descending", "repeat", "past_end", "negative"])
def test_bad_list_is_reported(h3, orc, bad):
    """A list that is not strictly ascending inside [0, KT) fails the launch on
    the device; the next status call reports it and clears it, and the context
    stays usable."""
    q, k, v = _case(1, 300, 700, 2, 128, seed=990)
    n_kt = 6
    lists = [[0, 2, 5], [1, 3], [0], [4, 5]]
    lists[1] = {"descending": [3, 1], "repeat": [1, 1], "past_end": [1, n_kt], "negative": [-1, 3]}[bad]
    off = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int32)
    idx = np.array([e for x in lists for e in x], dtype=np.int32)
    o, l = h3.attention_block_sparse(to_cuda_bf16(q), to_cuda_bf16(k), to_cuda_bf16(v), _cuda_i32(off),
                                     _cuda_i32(idx), return_lse=True)
    with pytest.raises(h3.H3AttnError, match="block-sparse"):
        h3.device_status()
    h3.device_status()  # cleared
    # the context still works: a valid call afterwards matches the oracle
    good = [[0, 2, 5], [1, 3], [0], [4, 5]]
    off = np.concatenate([[0], np.cumsum([len(x) for x in good])]).astype(np.int32)
    idx = np.array([e for x in good for e in x], dtype=np.int32)
    o, lse = _run(h3, q, k, v, off, idx)
    ro, rl = orc.attention_block_sparse(q, k, v, off, idx, 256, 128)
    _compare(o, lse, ro, rl, "after a bad list")


def test_block_sparse_2k_sampled(h3, orc):
    """The 2K-refine sequence (129,024 tokens, 24 heads of 128) with the
    benchmark's lists (diagonal tiles plus a quarter of the rest), on sampled rows."""
    w = inputs.workload("2k")
    N, H, d = w.total, w.n_heads, w.head_dim
    off, idx = inputs.block_lists(1, H, N, N, 0.25, seed=w.seed + 77)
    q, k, v = (a.reshape(1, N, H, d) for a in (w.q, w.k, w.v))
    o, lse = _run(h3, q, k, v, off, idx)
    rows = inputs.sample_rows(N, 48, seed=w.seed + 1001, tile=256)
    ro, rl = orc.attention_block_sparse(q, k, v, off, idx, 256, 128, rows=rows)
    og = bf16_bits_to_f64(o[0, rows])
    check_attention(og, ro, "block-sparse 2k", lse[0].T[rows], rl, strict=True)
