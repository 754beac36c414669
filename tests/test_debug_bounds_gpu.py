"""The bounds-checking debug build on the GPU: every kernel, with its store
indices checked against its own launch's extents (H3ATTN_DEBUG_BOUNDS), gives
exactly the release build's bits on valid launches and reports nothing.

compute-sanitizer cannot run here, so these checks stand in for a memory checker:
an index outside a launch's extents would be recorded for device_status() and the
store skipped, never written out of place."""
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
    from video_diffusion_transformer_h3attn_b200 import _build
    _build.build(debug_bounds=True)
    yield mod
    mod.use_library(None)


def _both(h3, fn):
    """fn() under the release and the debug library: (release, debug) outputs."""
    import torch
    from video_diffusion_transformer_h3attn_b200 import _build
    out = []
    for path, flags in ((None, 0), (_build.DEBUG_LIBRARY, 1)):
        h3.use_library(path)
        assert h3.build_flags() == flags
        res = fn()
        h3.device_status()  # a fired check raises here
        out.append([r.clone() for r in (res if isinstance(res, (tuple, list)) else (res,))])
        torch.cuda.synchronize()
    h3.use_library(None)
    return out


def _same(pair):
    import torch
    rel, dbg = pair
    for a, b in zip(rel, dbg):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


def test_prologue_and_dense_attention(h3):
    import torch
    pos, kind = inputs.video_layout(4, 8, 12, 40)
    w = inputs.make_workload("dbg", [len(kind)], 4, 128, seed=3, pos=pos, kind=kind)
    q, k, v = to_cuda_bf16(w.q), to_cuda_bf16(w.k), to_cuda_bf16(w.v)
    g = (to_cuda_bf16(w.gamma_q), to_cuda_bf16(w.gamma_k))
    pt, kt = torch.from_numpy(pos).cuda(), torch.from_numpy(kind).cuda()
    _same(_both(h3, lambda: h3.prologue(q, k, gamma_q=g[0], gamma_k=g[1], pos=pt, kind=kt)))
    _same(_both(h3, lambda: h3.attention(q, k, v, return_lse=True)))


@pytest.mark.parametrize("d", [64, 128])
def test_ragged_partial_merge_and_sparse(h3, d):
    import torch
    lens = [1, 130, 0, 255, 4, 513, 128]
    w = inputs.random_case(lens, 2, d, seed=11 + d)
    q, k, v = to_cuda_bf16(w.q), to_cuda_bf16(w.k), to_cuda_bf16(w.v)
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    _same(_both(h3, lambda: h3.attention_varlen(q, k, v, cu, max(lens), return_lse=True)))
    q3, k3 = q[:300].unsqueeze(0), k[:100].unsqueeze(0)
    v3 = v[:100].unsqueeze(0)
    _same(_both(h3, lambda: h3.attention_kv(q3, k3, v3, return_lse=True)))
    _same(_both(h3, lambda: h3.attention_kv(q3, k3[:, :0], v3[:, :0], return_lse=True)))
    oa, la = h3.attention_kv(q3, k3, v3, return_lse=True)
    ob, lb = h3.attention_kv(q3, q3, q3, return_lse=True)
    _same(_both(h3, lambda: h3.merge(oa, la, ob, lb)))
    off, idx = inputs.block_lists(1, 2, 300, 300, 0.5, seed=3)
    offt, idxt = torch.from_numpy(off).cuda(), torch.from_numpy(idx).cuda()
    x = q[:300].unsqueeze(0)
    _same(_both(h3, lambda: h3.attention_block_sparse(x, x, x, offt, idxt, return_lse=True)))


def test_fused_projection(h3):
    import torch
    rng = np.random.default_rng(2)
    n, dim_in, H, d = 300, 512, 4, 128
    x = to_cuda_bf16(inputs.f32_to_bf16_bits(rng.standard_normal((n, dim_in)).astype(np.float32)))
    wt = to_cuda_bf16(inputs.f32_to_bf16_bits((rng.standard_normal((3 * H * d, dim_in)) / 20).astype(np.float32)))
    pos = torch.from_numpy(np.stack([np.arange(n) % 5, np.arange(n) % 7, np.arange(n) // 35], 1).astype(np.int32)).cuda()
    kind = torch.full((n,), 1, dtype=torch.uint8, device="cuda")
    g = to_cuda_bf16(inputs.f32_to_bf16_bits(rng.uniform(0.5, 1.5, d).astype(np.float32)))
    _same(_both(h3, lambda: h3.qkv_fused(x, wt, H, gamma_q=g, gamma_k=g, pos=pos, kind=kind)))
