"""Parity of the CUDA attention kernels (dense and ragged) with the fp64 oracle.

Both sides read the same bf16 Q', K' (the oracle's prologue output, rounded
once) and V.  Small workloads are compared on every output; the large ones,
launched at full size exactly as the benchmark launches them, on sampled query
rows that visit every 128-row query tile (an edge row and a random row of each
tile, every sequence's first and last rows, random rows) with all heads, for
which the oracle's result is exact: 2,048 rows of the 2k clip, 512 of the joint
clip, 1,024 of the ragged mix."""
import numpy as np
import pytest

import oracle
from h3_testlib import check_attention, from_cuda_bf16, to_cuda_bf16, bf16_bits_to_f64
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


_QK_CACHE = {}


def _qk(orc, w):
    """Q', K' (bf16 bits) of a workload from the oracle's prologue."""
    if w.name not in _QK_CACHE:
        (_, q16), (_, k16) = orc.prologue_workload(w)
        _QK_CACHE[w.name] = (q16, k16)
    return _QK_CACHE[w.name]


def _gpu_dense(h3, q, k, v, lse=True):
    import torch
    qt, kt, vt = to_cuda_bf16(q), to_cuda_bf16(k), to_cuda_bf16(v)
    o, l = h3.attention(qt, kt, vt, return_lse=True)
    h3.device_status()
    return from_cuda_bf16(o), l.cpu().numpy()


def _gpu_varlen(h3, q, k, v, cu):
    import torch
    qt, kt, vt = to_cuda_bf16(q), to_cuda_bf16(k), to_cuda_bf16(v)
    cut = torch.from_numpy(np.asarray(cu, dtype=np.int32)).cuda()
    maxlen = int(np.max(np.diff(cu))) if len(cu) > 1 else 1
    o, l = h3.attention_varlen(qt, kt, vt, cut, max(1, maxlen), return_lse=True)
    h3.device_status()
    return from_cuda_bf16(o), l.cpu().numpy()


def test_tiny_full(h3, orc):
    w = inputs.workload("tiny")
    o, lse = _gpu_dense(h3, w.q, w.k, w.v)
    ro, rl = orc.attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(o), ro, "tiny", lse.T, rl, strict=True)


def test_small_full(h3, orc):
    w = inputs.workload("small")
    q, k = _qk(orc, w)
    o, lse = _gpu_dense(h3, q, k, w.v)
    ro, rl = orc.attention(q, k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(o), ro, "small", lse.T, rl, strict=True)


@pytest.mark.parametrize("name,n_rows", [("joint", 512), ("2k", 2048)])
def test_large_sampled(h3, orc, name, n_rows):
    w = inputs.workload(name)
    q, k = _qk(orc, w)
    o, lse = _gpu_dense(h3, q, k, w.v)
    rows = inputs.sample_rows_every_tile(w.cu_seqlens, n_rows, seed=w.seed + 1000)
    assert len(np.unique(rows // 128)) == -(-w.total // 128), "every query tile is sampled"
    ro, rl = orc.attention(q, k, w.v, w.cu_seqlens, rows=rows)
    check_attention(bf16_bits_to_f64(o[rows]), ro, name, lse.T[rows], rl, strict=True)


def test_ragged_sampled(h3, orc):
    w = inputs.workload("ragged")
    q, k = _qk(orc, w)
    o, lse = _gpu_varlen(h3, q, k, w.v, w.cu_seqlens)
    rows = inputs.sample_rows_every_tile(w.cu_seqlens, 1024, seed=w.seed + 1000)
    ro, rl = orc.attention(q, k, w.v, w.cu_seqlens, rows=rows)
    # Q x 4 makes rows peaked (|o| up to ~4): the plain mean bound holds, the max
    # bound is taken beyond the half-ulp cost of storing the output in bf16
    check_attention(bf16_bits_to_f64(o[rows]), ro, "ragged", lse.T[rows], rl, strict=True, plain_max=False)


@pytest.mark.parametrize("n", [1, 2, 3, 7, 63, 64, 127, 128, 129, 255, 256, 257, 383, 640])
@pytest.mark.parametrize("d", [64, 128])
def test_edge_lengths(h3, orc, n, d):
    """Every output of sequences of 1 to 640 keys.  From 64 keys on, the plain
    spec bounds hold as well (strict); below that, an output row is the mean
    of a few N(0, 1) value rows, |o| ~ 1, and storing even the exact value in bf16
    costs about a quarter ulp (~2e-3) on average, so the mean bound applies to the
    error beyond that half-ulp storage cost (the h3_testlib reading)."""
    w = inputs.random_case([n], 3, d, seed=500 + n + d)
    o, lse = _gpu_dense(h3, w.q, w.k, w.v)
    ro, rl = orc.attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(o), ro, "n=%d d=%d" % (n, d), lse.T, rl, strict=n >= 64)


@pytest.mark.parametrize("d", [64, 128])
def test_ragged_edges(h3, orc, d):
    lens = [1, 130, 0, 255, 4, 513, 128]
    w = inputs.random_case(lens, 2, d, seed=900 + d, q_scale=3.0)
    o, lse = _gpu_varlen(h3, w.q, w.k, w.v, w.cu_seqlens)
    ro, rl = orc.attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(o), ro, "ragged edges d=%d" % d, lse.T, rl)


def test_batched_strided_views(h3, orc):
    """B = 2 sequences read through strided views of one fused [B, N, 3, H, d] QKV buffer."""
    import torch
    B, N, H, d = 2, 300, 4, 128
    w = inputs.random_case([N] * B, H, d, seed=31)
    buf = torch.zeros((B, N, 3, H, d), dtype=torch.bfloat16, device="cuda")
    for i, a in enumerate((w.q, w.k, w.v)):
        buf[:, :, i] = to_cuda_bf16(a).view(B, N, H, d)
    o = h3.attention(buf[:, :, 0], buf[:, :, 1], buf[:, :, 2])
    h3.device_status()
    got = bf16_bits_to_f64(from_cuda_bf16(o)).reshape(B * N, H, d)
    ro, _ = orc.attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(got, ro, "batched strided")


def test_special_cases(h3, orc):
    """Q = 0 gives the mean of V; constant V rows give that row (to rounding)."""
    w = inputs.random_case([700], 2, 128, seed=41)
    zero = np.zeros_like(w.q)
    o, _ = _gpu_dense(h3, zero, w.k, w.v)
    mean = bf16_bits_to_f64(w.v).mean(axis=0)
    check_attention(bf16_bits_to_f64(o), np.broadcast_to(mean, o.shape), "Q=0")
    vc = np.broadcast_to(w.v[5], w.v.shape).copy()
    o, _ = _gpu_dense(h3, w.q, w.k, vc)
    check_attention(bf16_bits_to_f64(o), bf16_bits_to_f64(vc), "constant V")
    assert np.mean(o == vc) > 0.99, "constant V rows should come back (almost always) exactly"


@pytest.mark.parametrize("d", [64, 128])
def test_ragged_many_sequences(h3, orc, d):
    """More sequences than the in-kernel longest-first ranking takes (256): the
    launch falls back to the given order, with empty and one-token sequences."""
    rng = np.random.default_rng(77 + d)
    lens = rng.integers(0, 200, size=300)
    lens[::37] = 0
    lens[5] = 1
    w = inputs.random_case(list(int(x) for x in lens), 2, d, seed=960 + d)
    o, lse = _gpu_varlen(h3, w.q, w.k, w.v, w.cu_seqlens)
    ro, rl = orc.attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(o), ro, "300 sequences d=%d" % d, lse.T, rl)


def test_ragged_schedule_does_not_change_results(h3):
    """The same sequences give the same bits whether the kernel ranks them
    longest first (<= 256 sequences) or takes them in the given order (more
    sequences: 50 empty ones appended), and in a dense launch of one of them."""
    import torch
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(1, 400, size=200)]
    w = inputs.random_case(lens, 2, 128, seed=970)
    o_sorted, l_sorted = _gpu_varlen(h3, w.q, w.k, w.v, w.cu_seqlens)
    cu_more = np.concatenate([w.cu_seqlens, np.full(50, w.cu_seqlens[-1], dtype=np.int32)])
    o_given, l_given = _gpu_varlen(h3, w.q, w.k, w.v, cu_more)
    assert np.array_equal(o_sorted, o_given), "ranked and given orders must give identical outputs"
    assert np.array_equal(l_sorted, l_given)
    s = 17
    a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
    o_one, _ = _gpu_dense(h3, w.q[a:b], w.k[a:b], w.v[a:b])
    assert np.array_equal(o_one, o_sorted[a:b]), "a ragged sequence equals its dense launch bit for bit"


@pytest.mark.parametrize("cu,max_seqlen,what", [
    ([0, 300, 200, 500], 300, "a negative length"),
    ([0, 100, 250], 200, "cu[nseq] short of total_tokens"),
    ([0, 100, 360], 300, "cu[nseq] beyond total_tokens"),
    ([10, 100, 300], 200, "cu[0] != 0"),
    ([0, 100, 300], 150, "a sequence longer than max_seqlen"),
])
def test_ragged_bad_cu_seqlens_is_rejected_in_the_kernel(h3, orc, cu, max_seqlen, what):
    """cu_seqlens lives in device memory, so the host cannot read it: the kernel
    checks it before any load or store uses a sequence bound, writes nothing, and
    the next device_status() reports INVALID_ARG; the following valid launch runs."""
    import torch
    total = 300 if what != "a negative length" else 500
    w = inputs.random_case([total], 2, 128, seed=990)
    qt, kt, vt = to_cuda_bf16(w.q), to_cuda_bf16(w.k), to_cuda_bf16(w.v)
    o = torch.full_like(qt, 3.0)
    lse = torch.full((2, total), 7.0, dtype=torch.float32, device="cuda")
    bad = torch.tensor(cu, dtype=torch.int32, device="cuda")
    h3.device_status()
    lib = h3.library()
    import ctypes
    st = lambda t: (ctypes.c_int64 * 2)(t.stride(0), t.stride(1))
    rc = lib.h3attn_fwd_varlen(qt.data_ptr(), kt.data_ptr(), vt.data_ptr(), o.data_ptr(), bad.data_ptr(),
                               len(cu) - 1, total, max_seqlen, 2, 128, st(qt), st(kt), st(vt), st(o), 0.0,
                               lse.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, "host-side checks cannot see device memory: the launch is accepted"
    with pytest.raises(h3.H3AttnError) as exc:
        h3.device_status()
    assert exc.value.status == 1 and "cu_seqlens" in str(exc.value), what
    assert torch.all(o == 3.0) and torch.all(lse == 7.0), "%s: nothing may be written" % what
    h3.device_status()  # the error was cleared
    cu_ok = np.asarray([0, 120, total], dtype=np.int32)
    got, got_lse = _gpu_varlen(h3, w.q, w.k, w.v, cu_ok)
    ro, rl = orc.attention(w.q, w.k, w.v, cu_ok)
    check_attention(bf16_bits_to_f64(got), ro, "valid launch after " + what, got_lse.T, rl, strict=True)


def _ramped_case(lens, d, fac, seed):
    """|Q| and |K| with key magnitudes growing along the sequence: every row's
    maximum score grows from key tile to key tile (by ~8 log2 units per tile at
    fac = 6, by more than 16 in 80% of tiles at fac = 16), so the running maximum
    is raised and O rescaled in tensor memory many times per row."""
    w = inputs.random_case(lens, 2, d, seed=seed)
    q = np.abs(inputs.bf16_bits_to_f32(w.q))
    k = np.abs(inputs.bf16_bits_to_f32(w.k))
    pos = np.concatenate([np.arange(n) for n in lens]) if len(lens) else np.zeros(0)
    span = np.concatenate([np.full(n, max(n, 1)) for n in lens]) if len(lens) else np.ones(0)
    k = k * (1.0 + fac * pos / span).astype(np.float32)[:, None, None]
    w.q = inputs.f32_to_bf16_bits(q)
    w.k = inputs.f32_to_bf16_bits(k)
    return w


@pytest.mark.parametrize("fac,d", [(6.0, 128), (16.0, 128), (16.0, 64)])
def test_running_max_grows_every_tile(h3, orc, fac, d):
    # rows are peaked on the last keys (|o| up to ~3): the max bound is taken beyond
    # the half-ulp storage cost, the plain mean bound holds
    w = _ramped_case([1100], d, fac, seed=71)
    o, lse = _gpu_dense(h3, w.q, w.k, w.v)
    ro, rl = orc.attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(o), ro, "ramped fac=%g d=%d" % (fac, d), lse.T, rl, strict=True,
                    plain_max=False)


def test_running_max_grows_every_tile_ragged(h3, orc):
    w = _ramped_case([700, 1100, 0, 300], 128, 16.0, seed=72)
    o, lse = _gpu_varlen(h3, w.q, w.k, w.v, w.cu_seqlens)
    ro, rl = orc.attention(w.q, w.k, w.v, w.cu_seqlens)
    check_attention(bf16_bits_to_f64(o), ro, "ramped ragged", lse.T, rl, strict=True, plain_max=False)
