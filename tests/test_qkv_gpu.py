"""Parity of the fused Q/K/V projection (projection GEMM with the RMSNorm + RoPE
prologue in its epilogue) with the fp64 oracle.

Tolerance, from the arithmetic: the tensor cores accumulate the projection in
fp32, so a feature's error is bounded by KAPPA * A_f with A_f = sum_c |x_c w_fc|
(the sum of the magnitudes of its products; KAPPA = 2^-20 allows the rounding of
the fp32 accumulator across dim_in / 16 accumulation steps with room to spare).
The norm divides by the row's rms and multiplies by gamma, which carries that
error over (to first order) as
  |dy_i| <= gamma_i / rms * KAPPA * A_i + |y_i| * KAPPA * sum_j |x_j| A_j / sum_j x_j^2,
plus a few fp32 roundings of y_i (NORM_REL) and the fp32 rotation (cos/sin within
2^-21, ROPE_ABS); the rotation mixes each pair, so a rotated element may carry
both errors of its pair.  Every output must lie within
half a bf16 ulp of the exact (oracle) value plus that bound."""
import numpy as np
import pytest

import oracle
from h3_testlib import bf16_bits_to_f64, bf16_half_ulp, from_cuda_bf16, to_cuda_bf16
from video_diffusion_transformer_h3attn_b200 import inputs

pytestmark = pytest.mark.gpu

KAPPA = 2.0 ** -20
NORM_REL = 2.0 ** -20
ROPE_ABS = 2.0 ** -19      # fp32 cos/sin (< 2^-21 absolute) and the fp32 rotation, per pair element


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


def _case(n, dim_in, H, d, seed, bias=True, layout="video"):
    rng = np.random.default_rng(seed)
    x = inputs.f32_to_bf16_bits(rng.standard_normal((n, dim_in)).astype(np.float32))
    w = inputs.f32_to_bf16_bits((rng.standard_normal((3 * H * d, dim_in)) / np.sqrt(dim_in)).astype(np.float32))
    b = inputs.f32_to_bf16_bits((rng.standard_normal(3 * H * d) * 0.1).astype(np.float32)) if bias else None
    gq = inputs.f32_to_bf16_bits(rng.uniform(0.5, 1.5, d).astype(np.float32))
    gk = inputs.f32_to_bf16_bits(rng.uniform(0.5, 1.5, d).astype(np.float32))
    pos = np.zeros((n, 3), dtype=np.int32)
    pos[:, 0] = np.arange(n) % 11
    pos[:, 1] = (np.arange(n) // 11) % 13
    pos[:, 2] = np.arange(n) // 143
    kind = np.full(n, 1, dtype=np.uint8) if layout == "video" else (np.arange(n) % 3).astype(np.uint8)
    sections = (d // 4, 3 * d // 8, 3 * d // 8)
    return x, w, b, gq, gk, pos, kind, sections


def _bounds(x, w, b, rows, H, d, gam, part, y64, pre64):
    """Per-element error bound (see the module docstring) for part 0 (Q), 1 (K), 2 (V)."""
    xv = bf16_bits_to_f64(x[rows])
    wv = bf16_bits_to_f64(w[part * H * d:(part + 1) * H * d])
    A = (np.abs(xv) @ np.abs(wv).T).reshape(len(rows), H, d)
    if part == 2:
        return KAPPA * A + 2.0 ** -23 * np.abs(y64)
    g = bf16_bits_to_f64(gam)[None, None, :]
    pre = pre64  # the projection (+ bias) before the norm, fp64
    ss = np.sum(pre * pre, axis=-1, keepdims=True)
    rms = np.sqrt(ss / d + 1e-6)
    lin = g / rms * KAPPA * A
    glob = np.abs(pre * g / rms) * KAPPA * np.sum(np.abs(pre) * A, axis=-1, keepdims=True) / ss
    e = lin + glob + NORM_REL * np.abs(pre * g / rms) + ROPE_ABS * np.abs(pre * g / rms)
    # RoPE mixes the pair
    pair = e.reshape(len(rows), H, d // 2, 2).sum(-1, keepdims=True)
    return np.broadcast_to(pair, (len(rows), H, d // 2, 2)).reshape(len(rows), H, d)


def _check(h3, orc, n, dim_in, H, d, seed, bias=True, layout="video", n_rows=None):
    import torch
    x, w, b, gq, gk, pos, kind, sec = _case(n, dim_in, H, d, seed, bias, layout)
    q, k, v = h3.qkv_fused(to_cuda_bf16(x), to_cuda_bf16(w), H, bias=None if b is None else to_cuda_bf16(b),
                           gamma_q=to_cuda_bf16(gq), gamma_k=to_cuda_bf16(gk), pos=torch.from_numpy(pos).cuda(),
                           kind=torch.from_numpy(kind).cuda(), sections=sec)
    h3.device_status()
    rows = np.arange(n) if n_rows is None else inputs.sample_rows(n, n_rows, seed)
    (rq, rk, rv), _ = orc.qkv_norm_rope(x, w, b, H, gq, gk, 1e-6, pos, kind, sec, rows=rows, want_bf16=False)
    # the projection before the norm, for the bound
    (pq, pk_, _), _ = orc.qkv_norm_rope(x, w, b, H, rows=rows, want_bf16=False)
    for part, got, ref, gam, pre in ((0, q, rq, gq, pq), (1, k, rk, gk, pk_), (2, v, rv, None, None)):
        g = bf16_bits_to_f64(from_cuda_bf16(got))[rows]
        bound = bf16_half_ulp(ref) + _bounds(x, w, b, rows, H, d, gam, part, ref, pre)
        err = np.abs(g - ref)
        worst = np.unravel_index(int(np.argmax(err / bound)), err.shape)
        assert np.all(err <= bound), "%s: error %g > bound %g at %s (ratio %.2f)" % (
            "QKV"[part], err[worst], bound[worst], worst, err[worst] / bound[worst])


@pytest.mark.parametrize("n,dim_in,H,d", [(300, 512, 4, 128), (1000, 256, 4, 64), (129, 3072, 24, 128),
                                          (257, 64, 2, 128)])
def test_qkv_fused_vs_oracle(h3, orc, n, dim_in, H, d):
    _check(h3, orc, n, dim_in, H, d, seed=n + dim_in)


def test_qkv_fused_mixed_tokens_no_bias(h3, orc):
    _check(h3, orc, 777, 384, 2, 128, seed=5, bias=False, layout="mixed")


def test_qkv_fused_model_size_sampled(h3, orc):
    """The model's projection (dim_in = H*d = 3072, 9216 features) on 4096 tokens,
    sampled rows."""
    _check(h3, orc, 4096, 3072, 24, 128, seed=9, n_rows=96)


def test_qkv_fused_2k_sampled(h3, orc):
    """The 2K clip's token count (129,024) at the model width, as the benchmark
    launches it (a persistent grid of CTA pairs over 504 x 36 tiles), sampled rows."""
    _check(h3, orc, 129024, 3072, 24, 128, seed=10, n_rows=64)


def test_qkv_fused_matches_projection_then_prologue(h3):
    """Against the unfused path (cuBLAS projection rounded to bf16, then the
    prologue kernel): the two differ by the projection's bf16 rounding only."""
    import torch
    x, w, b, gq, gk, pos, kind, sec = _case(512, 1024, 8, 128, seed=3)
    xt, wt, bt = to_cuda_bf16(x), to_cuda_bf16(w), to_cuda_bf16(b)
    g = (to_cuda_bf16(gq), to_cuda_bf16(gk))
    pt, kt = torch.from_numpy(pos).cuda(), torch.from_numpy(kind).cuda()
    q, k, v = h3.qkv_fused(xt, wt, 8, bias=bt, gamma_q=g[0], gamma_k=g[1], pos=pt, kind=kt, sections=sec)
    proj = (xt @ wt.T + bt).view(512, 3, 8, 128)
    q2, k2 = h3.prologue(proj[:, 0], proj[:, 1], gamma_q=g[0], gamma_k=g[1], pos=pt, kind=kt, sections=sec)
    h3.device_status()
    for a, b_ in ((q, q2), (k, k2), (v, proj[:, 2])):
        diff = (a.float() - b_.float()).abs()
        assert diff.max().item() < 0.08 and diff.mean().item() < 2e-3


@pytest.mark.parametrize("n", [1, 33, 300])
def test_qkv_fused_output_layouts_are_bitwise_identical(h3, n):
    """The outputs leave through bulk tensor stores whose tensor maps are built from
    the output strides: views of one fused [n, 3, H, d] buffer and head-outermost
    views ([H, n, d] storage) give exactly the bits of separate contiguous outputs,
    with a ragged last block of tokens (n not a multiple of 32) and a single token."""
    import torch
    H, d = 4, 128
    x, w, b, gq, gk, pos, kind, sec = _case(n, 512, H, d, seed=70 + n)
    xt, wt, bt = to_cuda_bf16(x), to_cuda_bf16(w), to_cuda_bf16(b)
    g = (to_cuda_bf16(gq), to_cuda_bf16(gk))
    pt, kt = torch.from_numpy(pos).cuda(), torch.from_numpy(kind).cuda()
    kw = dict(bias=bt, gamma_q=g[0], gamma_k=g[1], pos=pt, kind=kt, sections=sec)
    ref = h3.qkv_fused(xt, wt, H, **kw)
    fused = torch.full((n, 3, H, d), 7.0, dtype=torch.bfloat16, device="cuda")
    got = h3.qkv_fused(xt, wt, H, q_out=fused[:, 0], k_out=fused[:, 1], v_out=fused[:, 2], **kw)
    heads_out = [torch.full((H, n, d), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    got2 = h3.qkv_fused(xt, wt, H, q_out=heads_out[0].permute(1, 0, 2), k_out=heads_out[1].permute(1, 0, 2),
                        v_out=heads_out[2].permute(1, 0, 2), **kw)
    h3.device_status()
    for r, a, c in zip(ref, got, got2):
        assert torch.equal(r, a) and torch.equal(r, c)
