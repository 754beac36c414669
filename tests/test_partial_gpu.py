"""Parity of partial attention (queries against one block of a split key set)
and of the log-sum-exp merge with the fp64 oracle.

attention_kv is compared with the oracle's partial attention on the same bf16
inputs, with the attention tolerances.  The merge kernel is compared with the
oracle's merge of exactly the GPU's inputs (bf16 O parts and fp32 LSE parts,
read as fp64): every output is within half a bf16 ulp of that merge plus the fp32
error of the weighted sum (which only shows where the two parts cancel).  The whole split-key pipeline (partials, then
merges in place) is compared with the oracle's attention over all keys."""
import numpy as np
import pytest

import oracle
from h3_testlib import bf16_bits_to_f64, bf16_half_ulp, check_attention, from_cuda_bf16, to_cuda_bf16
from video_diffusion_transformer_h3attn_b200 import inputs

pytestmark = pytest.mark.gpu

# O: |o_gpu - o| <= ulp_bf16(o)/2 + MERGE_W_REL * (w_a |O_a| + w_b |O_b|): one bf16 rounding of
# the result plus the fp32 error of the weighted sum (weights from expf and a division, a few fp32
# ulps each; 2^-20 allows 16).  The second term matters only where the two parts cancel.
MERGE_W_REL = 2.0 ** -20
MERGE_LSE_TOL = 2e-6       # |L_gpu - L| <= tol * max(1, |L|): fp32 expf/logf on the weights


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


def _case(nq, nk, H, d, seed, q_scale=1.0):
    """q [nq, H, d] and k, v [nk, H, d] bf16 bits from the shared generator."""
    w = inputs.random_case([max(nq, nk, 1)], H, d, seed, q_scale=q_scale)
    return w.q[:nq], w.k[:nk], w.v[:nk]


@pytest.mark.parametrize("nq,nk,d", [(300, 1000, 128), (1000, 300, 128), (129, 1, 128), (5, 4097, 128),
                                     (640, 257, 64), (256, 128, 64), (777, 2000, 128)])
def test_attention_kv_vs_oracle(h3, orc, nq, nk, d):
    q, k, v = _case(nq, nk, 2, d, seed=700 + nq + nk + d)
    o, l = h3.attention_kv(to_cuda_bf16(q), to_cuda_bf16(k), to_cuda_bf16(v), return_lse=True)
    h3.device_status()
    ro, rl = orc.attention_kv(q, k, v)
    check_attention(bf16_bits_to_f64(from_cuda_bf16(o)), ro, "kv %dx%d d%d" % (nq, nk, d),
                    l.cpu().numpy().T, rl, strict=True)


@pytest.mark.parametrize("d", [64, 128])
def test_attention_kv_without_keys(h3, d):
    import torch
    q, _, _ = _case(300, 1, 2, d, seed=801)
    qt = to_cuda_bf16(q)
    empty = torch.empty((0, 2, d), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(qt, 7.0)
    o, l = h3.attention_kv(qt, empty, empty, o=o, return_lse=True)
    h3.device_status()
    assert torch.all(o == 0), "no keys: O must be the empty sum (0)"
    assert torch.all(torch.isneginf(l)), "no keys: LSE must be -inf"


def _merge_inputs(rng, B, N, H, d):
    """Partial O (bf16 bits) and LSE (fp32) with edge rows: an empty side, both
    empty, equal LSE, and large magnitudes."""
    oa = inputs.f32_to_bf16_bits(rng.standard_normal((B, N, H, d)).astype(np.float32))
    ob = inputs.f32_to_bf16_bits(rng.standard_normal((B, N, H, d)).astype(np.float32))
    la = (rng.standard_normal((B, H, N)) * 4).astype(np.float32)
    lb = (rng.standard_normal((B, H, N)) * 4).astype(np.float32)
    la[:, :, 0] = -np.inf                    # a empty
    lb[:, :, 1] = -np.inf                    # b empty
    la[:, :, 2] = lb[:, :, 2] = -np.inf      # both empty
    lb[:, :, 3] = la[:, :, 3]                # equal weights
    la[:, :, 4], lb[:, :, 4] = 80.0, 79.0    # large
    la[:, :, 5], lb[:, :, 5] = -90.0, -60.0
    oa[:, 0] = 0                             # an empty part's O as the kernel writes it
    ob[:, 1] = 0
    oa[:, 2] = ob[:, 2] = 0
    return oa, ob, la, lb


@pytest.mark.parametrize("B,N,H,d", [(1, 333, 3, 128), (2, 70, 2, 64), (1, 4096, 24, 128)])
def test_merge_vs_oracle(h3, orc, B, N, H, d):
    import torch
    rng = np.random.default_rng(900 + N)
    oa, ob, la, lb = _merge_inputs(rng, B, N, H, d)
    o, l = h3.merge(to_cuda_bf16(oa), torch.from_numpy(la).cuda(), to_cuda_bf16(ob),
                    torch.from_numpy(lb).cuda())
    h3.device_status()
    _check_merge(orc, oa, ob, la, lb, from_cuda_bf16(o), l.cpu().numpy())
    assert np.all(from_cuda_bf16(o)[:, 2] == 0), "both parts empty: O = 0"


def test_merge_2k_sampled(h3, orc):
    """The merge at the 2K clip's full output shape (129,024 tokens x 24 heads x
    128), as the benchmark launches it, checked on sampled rows."""
    import torch
    B, N, H, d = 1, 129024, 24, 128
    g = torch.Generator(device="cuda").manual_seed(5)
    oa = torch.randn((B, N, H, d), generator=g, device="cuda").to(torch.bfloat16)
    ob = torch.randn((B, N, H, d), generator=g, device="cuda").to(torch.bfloat16)
    la = torch.randn((B, H, N), generator=g, device="cuda") * 4
    lb = torch.randn((B, H, N), generator=g, device="cuda") * 4
    o, l = h3.merge(oa, la, ob, lb)
    h3.device_status()
    rows = torch.from_numpy(inputs.sample_rows(N, 96, seed=4321)).cuda()
    _check_merge(orc, from_cuda_bf16(oa[:, rows]), from_cuda_bf16(ob[:, rows]), la[:, :, rows].cpu().numpy(),
                 lb[:, :, rows].cpu().numpy(), from_cuda_bf16(o[:, rows]), l[:, :, rows].cpu().numpy())


def _check_merge(orc, oa, ob, la, lb, o_bits, l_gpu):
    """GPU merge (o_bits [B, N, H, d], l_gpu [B, H, N]) against the oracle's merge of
    exactly these inputs (oa, ob bf16 bits [B, N, H, d]; la, lb fp32 [B, H, N])."""
    # oracle on exactly these inputs: rows (b, n, h), parts a and b
    oap = bf16_bits_to_f64(oa)
    obp = bf16_bits_to_f64(ob)
    lap = la.astype(np.float64).transpose(0, 2, 1)  # [B, N, H]
    lbp = lb.astype(np.float64).transpose(0, 2, 1)
    ro, rl = orc.merge(np.stack([oap, obp]), np.stack([lap, lbp]))
    with np.errstate(invalid="ignore"):  # -inf - -inf where both parts are empty
        wa = np.exp(lap - rl)[..., None]  # exact weights of the two parts, [B, N, H, 1]
        wb = np.exp(lbp - rl)[..., None]
    wa[np.isneginf(rl)] = 0.0
    wb[np.isneginf(rl)] = 0.0
    bound = bf16_half_ulp(ro) + MERGE_W_REL * (wa * np.abs(oap) + wb * np.abs(obp))
    err = np.abs(bf16_bits_to_f64(o_bits) - ro)
    worst = np.unravel_index(int(np.argmax(err - bound)), err.shape)
    assert np.all(err <= bound), "merge O: error %g > bound %g at %s" % (err[worst], bound[worst], worst)
    rl = rl.transpose(0, 2, 1)  # [B, H, N]
    both_empty = np.isneginf(rl)
    assert np.array_equal(np.isneginf(l_gpu), both_empty), "merge LSE: -inf exactly where both parts are empty"
    fin = ~both_empty
    err = np.abs(l_gpu[fin] - rl[fin]) / np.maximum(1.0, np.abs(rl[fin]))
    assert err.max() <= MERGE_LSE_TOL, "merge LSE relative error %g" % err.max()


def test_merge_in_place(h3, orc):
    import torch
    rng = np.random.default_rng(77)
    oa, ob, la, lb = _merge_inputs(rng, 1, 200, 2, 128)
    ta, tla = to_cuda_bf16(oa), torch.from_numpy(la).cuda()
    ref_o, ref_l = h3.merge(ta, tla, to_cuda_bf16(ob), torch.from_numpy(lb).cuda())
    o, l = h3.merge(ta, tla, to_cuda_bf16(ob), torch.from_numpy(lb).cuda(), o=ta, lse=tla)
    h3.device_status()
    assert o.data_ptr() == ta.data_ptr() and l.data_ptr() == tla.data_ptr()
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l), "in-place merge must equal the out-of-place one"


@pytest.mark.parametrize("cuts,d", [([0, 700, 1500, 2600], 128), ([0, 1, 1300], 128), ([0, 0, 999], 64),
                                    ([0, 128, 256, 384, 512], 128)])
def test_split_keys_merge_to_full_attention(h3, orc, cuts, d):
    """Key blocks one at a time, merged in place, give the attention over all keys."""
    import torch
    nk = cuts[-1]
    q, k, v = _case(900, nk, 2, d, seed=950 + nk + d, q_scale=2.0)
    qt = to_cuda_bf16(q)
    o = l = None
    for a, b in zip(cuts[:-1], cuts[1:]):
        ob, lb = h3.attention_kv(qt, to_cuda_bf16(k[a:b]), to_cuda_bf16(v[a:b]), return_lse=True)
        if o is None:
            o, l = ob, lb
        else:
            h3.merge(o, l, ob, lb, o=o, lse=l)
    h3.device_status()
    ro, rl = orc.attention_kv(q, k, v)
    check_attention(bf16_bits_to_f64(from_cuda_bf16(o)), ro, "split keys %s" % cuts,
                    l.cpu().numpy().T, rl)
