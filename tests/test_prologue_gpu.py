"""Parity of the CUDA prologue (RMSNorm + RoPE) with the fp64 oracle: every
output element within one bf16 ulp of the oracle's correctly rounded value."""
import numpy as np
import pytest

import oracle
from h3_testlib import check_prologue, from_cuda_bf16, to_cuda_bf16
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


def _cuda(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.cuda() if dtype is None else t.to(dtype).cuda()


def _run(h3, w, tokens=None, fused=False, in_place=False):
    """GPU prologue of a workload (optionally a token subset); returns (q', k') bits."""
    import torch
    q, k = w.q, w.k
    pos, kind = w.pos, w.kind
    if tokens is not None:
        q, k = q[tokens], k[tokens]
        pos = None if pos is None else pos[tokens]
        kind = None if kind is None else kind[tokens]
    n, H, d = q.shape
    if fused:
        # one [n, 3, H, d] buffer, Q and K as strided views (the QKV projection layout)
        buf = torch.zeros((n, 3, H, d), dtype=torch.bfloat16, device="cuda")
        buf[:, 0] = to_cuda_bf16(q)
        buf[:, 1] = to_cuda_bf16(k)
        qt, kt = buf[:, 0], buf[:, 1]
    else:
        qt, kt = to_cuda_bf16(q), to_cuda_bf16(k)
    gq = None if w.gamma_q is None else to_cuda_bf16(w.gamma_q)
    gk = None if w.gamma_k is None else to_cuda_bf16(w.gamma_k)
    pt = None if pos is None else _cuda(pos)
    kd = None if kind is None else _cuda(kind)
    outs = (qt, kt) if in_place else (None, None)
    qo, ko = h3.prologue(qt, kt, outs[0], outs[1], gq, gk, w.eps, pt, kd, w.sections, w.theta)
    h3.device_status()
    return from_cuda_bf16(qo), from_cuda_bf16(ko)


def _ref(orc, w, tokens=None):
    q, k, pos, kind = w.q, w.k, w.pos, w.kind
    if tokens is not None:
        q, k = q[tokens], k[tokens]
        pos = None if pos is None else pos[tokens]
        kind = None if kind is None else kind[tokens]
    _, q16 = orc.rmsnorm_rope(q, w.gamma_q, w.eps, pos, kind, w.sections, w.theta, want_f64=False)
    _, k16 = orc.rmsnorm_rope(k, w.gamma_k, w.eps, pos, kind, w.sections, w.theta, want_f64=False)
    return q16, k16


@pytest.mark.parametrize("name", ["small", "joint", "ragged"])
def test_prologue_workloads(h3, orc, name):
    w = inputs.workload(name)
    gq, gk = _run(h3, w)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, name + " q")
    check_prologue(gk, rk, name + " k")


def test_prologue_2k_sampled_tokens(h3, orc):
    w = inputs.workload("2k")
    rng = np.random.default_rng(4)
    tokens = np.unique(np.concatenate([[0, 1, 127, 128, len(w.q) - 1], rng.integers(0, len(w.q), 4096)]))
    gq, gk = _run(h3, w)  # the full-size launch, as the benchmark runs it
    rq, rk = _ref(orc, w, tokens)
    check_prologue(gq[tokens], rq, "2k q")
    check_prologue(gk[tokens], rk, "2k k")


def test_prologue_fused_qkv_in_place(h3, orc):
    w = inputs.workload("small")
    gq, gk = _run(h3, w, fused=True, in_place=True)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, "fused in-place q")
    check_prologue(gk, rk, "fused in-place k")


def test_prologue_d64_odd_heads_mixed_kinds(h3, orc):
    # d = 64 packs two heads per warp pass: an odd head count exercises the tail;
    # kinds 0/1/2 and a gamma on Q only exercise every branch
    n, H, d = 333, 3, 64
    w = inputs.make_workload("d64", [n], H, d, seed=77, norm=True, sections=(16, 24, 24))
    rng = np.random.default_rng(78)
    w.pos = np.stack([rng.integers(0, 40, n), rng.integers(0, 50, n), rng.integers(0, 90, n)], 1).astype(np.int32)
    w.kind = rng.integers(0, 3, n).astype(np.uint8)
    w.gamma_k = None
    gq, gk = _run(h3, w)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, "d64 q")
    check_prologue(gk, rk, "d64 k")


def test_prologue_norm_only_and_single_token(h3, orc):
    w = inputs.make_workload("one", [1], 24, 128, seed=79, norm=True)
    gq, gk = _run(h3, w)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, "single token q")
    check_prologue(gk, rk, "single token k")


def test_prologue_identity_without_norm_or_rope(h3):
    w = inputs.make_workload("copy", [100], 4, 128, seed=80, norm=False)
    gq, gk = _run(h3, w)
    assert np.array_equal(gq, w.q) and np.array_equal(gk, w.k)


@pytest.mark.parametrize("H,d", [(32, 128), (60, 64)])
def test_prologue_many_heads(h3, orc, H, d):
    # head counts above the model's (more heads per token than a warp's passes
    # at the benchmark size); a ragged token count and all three token kinds
    n = 77
    w = inputs.make_workload("many%d" % H, [n], H, d, seed=81 + H, norm=True,
                             sections=(32, 48, 48) if d == 128 else (16, 24, 24))
    rng = np.random.default_rng(82)
    w.pos = np.stack([rng.integers(0, 40, n), rng.integers(0, 50, n), rng.integers(0, 90, n)], 1).astype(np.int32)
    w.kind = rng.integers(0, 3, n).astype(np.uint8)
    gq, gk = _run(h3, w)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, "H%d q" % H)
    check_prologue(gk, rk, "H%d k" % H)


@pytest.mark.parametrize("H,d", [(1, 128), (7, 128), (8, 128), (9, 128), (17, 128),
                                 (1, 64), (15, 64), (16, 64), (17, 64), (33, 64)])
def test_prologue_pass_counts(h3, orc, H, d):
    # a warp streams its token's head passes (one head per pass at d = 128, two at
    # d = 64) through a ring of eight: fewer passes than the ring, exactly the ring,
    # one more, and several turns of it, with a half-live last pass at odd d = 64
    # head counts; 45 tokens leave the last block's warps partly idle
    n = 45
    w = inputs.make_workload("passes%d_%d" % (H, d), [n], H, d, seed=300 + H + d, norm=True,
                             sections=(32, 48, 48) if d == 128 else (16, 24, 24))
    rng = np.random.default_rng(301 + H)
    w.pos = np.stack([rng.integers(0, 40, n), rng.integers(0, 50, n), rng.integers(0, 5000, n)], 1).astype(np.int32)
    w.kind = rng.integers(0, 3, n).astype(np.uint8)
    gq, gk = _run(h3, w)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, "H%d d%d q" % (H, d))
    check_prologue(gk, rk, "H%d d%d k" % (H, d))


@pytest.mark.parametrize("sections", [(64, 64, 0), (0, 0, 128), (0, 128, 0), (32, 48, 48)])
def test_prologue_video_rows_sections(h3, orc, sections):
    # video rows of 16 tokens (tokens of a row share t and h); degenerate sections put
    # every rotation pair on the t and h axes, or all on w, or all on h; 5 audio
    # tokens end the clip
    pos, kind = inputs.video_layout(3, 4, 16, n_audio=5)
    n = len(pos)
    w = inputs.make_workload("rows%d%d%d" % sections, [n], 6, 128, seed=400, norm=True, sections=sections,
                             pos=pos, kind=kind)
    gq, gk = _run(h3, w)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, "sections %s q" % (sections,))
    check_prologue(gk, rk, "sections %s k" % (sections,))


def _cancelling_rows(rng, pos, n, H, d, theta):
    """bf16 rows whose rotation pairs nearly cancel: for pair i at angle
    pos * theta^(-2i/d), x1 ~ x0 * cos/sin makes x0*cos - x1*sin vanish to the
    rounding of x1, or x1 ~ -x0 * sin/cos does the same for x1*cos + x0*sin."""
    i = np.arange(d // 2)
    ang = pos[:, 0:1].astype(np.float64) * np.exp(-(2.0 * i / d) * np.log(theta))[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x0 = rng.uniform(0.5, 2.0, (n, H, d // 2)) * rng.choice([-1.0, 1.0], (n, H, d // 2))
    x0 = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(x0.astype(np.float32))).astype(np.float64)
    with np.errstate(divide="ignore"):
        ratio = np.where(rng.integers(0, 2, (n, H, d // 2)) == 0, (c / s)[:, None, :], (-s / c)[:, None, :])
    usable = np.isfinite(ratio) & (np.abs(ratio) > 1.0 / 64) & (np.abs(ratio) < 64.0)
    x1 = np.where(usable, x0 * np.where(usable, ratio, 0.0), rng.uniform(-2.0, 2.0, x0.shape))
    x = np.empty((n, H, d))
    x[..., 0::2] = x0
    x[..., 1::2] = x1
    return inputs.f32_to_bf16_bits(x.astype(np.float32))


def test_prologue_rotation_cancellation(h3, orc):
    # The two products of each rotated element nearly cancel, so the result is
    # thousands of times smaller than its terms; a rotation with fp32 cos/sin and
    # no error-free product misses the 1-ulp bound on ~0.1% of these elements (by up
    # to thousands of ulps), the kernel's float-pair rotation must not.  Q without
    # norm (no scale factor), K with a unit gamma (the RMS factor on top).
    n, H, d = 2048, 4, 128
    rng = np.random.default_rng(5)
    w = inputs.make_workload("cancel", [n], H, d, seed=6, norm=True)
    w.pos = np.zeros((n, 3), dtype=np.int32)
    w.pos[:, 0] = rng.integers(0, 5000, n)
    w.kind = np.full(n, 2, dtype=np.uint8)
    w.q = _cancelling_rows(rng, w.pos, n, H, d, w.theta)
    w.k = _cancelling_rows(rng, w.pos, n, H, d, w.theta)
    w.gamma_q = None
    w.gamma_k = inputs.f32_to_bf16_bits(np.ones(d, dtype=np.float32))
    gq, gk = _run(h3, w)
    rq, rk = _ref(orc, w)
    check_prologue(gq, rq, "cancelling q")
    check_prologue(gk, rk, "cancelling k")
