"""h3attn -- B200 (sm_100a) attention hot path of a joint video/audio DiT block.

Python binding of the C ABI in include/h3attn.h.  It only marshals arguments
(data pointers, strides, the current CUDA stream) into the library; every step
of the computation runs in the library's CUDA kernels.  There is no CPU
fallback: without the built library, or with tensors that are not CUDA bf16,
the calls raise.

    prologue(q, k, ...)                 per-head RMSNorm + RoPE of Q and K
    attention(q, k, v, ...)             dense non-causal softmax(QK^T*scale)V
    attention_varlen(q, k, v, cu, ...)  the same over ragged packed sequences
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence, Tuple

from . import _build

__all__ = ["prologue", "attention", "attention_varlen", "attention_kv", "attention_block_sparse", "merge",
           "qkv_fused", "device_status", "selftest_wait_timeout", "library", "use_library", "build_flags",
           "H3AttnError", "KIND_NONE", "KIND_3D", "KIND_1D",
           "declared_symbols"]

KIND_NONE, KIND_3D, KIND_1D = 0, 1, 2

LIBRARY_PATH = _build.LIBRARY
HEADER_PATH = os.path.join(_build.INCLUDE, "h3attn.h")


class H3AttnError(RuntimeError):
    """A call into the h3attn library returned an error status."""

    def __init__(self, call: str, status: int, detail: str):
        self.status = status
        super().__init__("%s failed: %s (%d): %s" % (call, _status_string(status), status, detail))


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_I64_3 = ctypes.c_int64 * 3
_I64_2 = ctypes.c_int64 * 2


def use_library(path: Optional[str] = None) -> None:
    """Load the library from `path` for the calls that follow (None: the release
    build; _build.DEBUG_LIBRARY: the bounds-checking debug build)."""
    global _lib, LIBRARY_PATH
    LIBRARY_PATH = path or _build.LIBRARY
    _lib = None


def build_flags() -> int:
    """h3attn_build_flags() of the loaded library (bit 1: bounds-checking debug build)."""
    return int(library().h3attn_build_flags())


def library() -> ctypes.CDLL:
    """The loaded libh3attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY_PATH):
            raise RuntimeError("libh3attn.so is not built (%s); run __graft_entry__.build() or "
                               "python -m video_diffusion_transformer_h3attn_b200._build" % LIBRARY_PATH)
        lib = ctypes.CDLL(LIBRARY_PATH)
        lib.h3attn_version.restype = ctypes.c_int
        lib.h3attn_build_flags.restype = ctypes.c_int
        lib.h3attn_status_string.restype = ctypes.c_char_p
        lib.h3attn_status_string.argtypes = [ctypes.c_int]
        lib.h3attn_last_error.restype = ctypes.c_char_p
        lib.h3attn_device_status.restype = ctypes.c_int
        lib.h3attn_device_status.argtypes = [_P, ctypes.c_int]
        lib.h3attn_prologue.restype = ctypes.c_int
        lib.h3attn_prologue.argtypes = [_P, _P, _P, _P, _I64, _I32, _I32, _I64, _I64, _I64, _I64,
                                        _P, _P, ctypes.c_double, _P, _P, _I32, _I32, _I32,
                                        ctypes.c_double, _P]
        lib.h3attn_fwd.restype = ctypes.c_int
        lib.h3attn_fwd.argtypes = [_P, _P, _P, _P, _I32, _I64, _I32, _I32, _I64_3, _I64_3, _I64_3,
                                   _I64_3, ctypes.c_float, _P, _P]
        lib.h3attn_fwd_varlen.restype = ctypes.c_int
        lib.h3attn_fwd_varlen.argtypes = [_P, _P, _P, _P, _P, _I32, _I64, _I32, _I32, _I32, _I64_2,
                                          _I64_2, _I64_2, _I64_2, ctypes.c_float, _P, _P]
        lib.h3attn_fwd_kv.restype = ctypes.c_int
        lib.h3attn_fwd_kv.argtypes = [_P, _P, _P, _P, _I32, _I64, _I64, _I32, _I32, _I64_3, _I64_3,
                                      _I64_3, _I64_3, ctypes.c_float, _P, _P]
        lib.h3attn_qkv_fused.restype = ctypes.c_int
        lib.h3attn_qkv_fused.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I32, _I32, _I32, _I64, _I64_3, _I64_3,
                                         _P, _P, ctypes.c_double, _P, _P, _I32, _I32, _I32, ctypes.c_double, _P]
        lib.h3attn_fwd_block_sparse.restype = ctypes.c_int
        lib.h3attn_fwd_block_sparse.argtypes = [_P, _P, _P, _P, _I32, _I64, _I64, _I32, _I32, _I64_3, _I64_3,
                                                _I64_3, _I64_3, _P, _P, ctypes.c_float, _P, _P]
        lib.h3attn_selftest_wait_timeout.restype = ctypes.c_int
        lib.h3attn_selftest_wait_timeout.argtypes = [_P]
        lib.h3attn_merge.restype = ctypes.c_int
        lib.h3attn_merge.argtypes = [_P, _P, _P, _P, _P, _P, _I32, _I64, _I32, _I32, _I64_3, _I64_3,
                                     _I64_3, _P]
        _lib = lib
    return _lib


def declared_symbols() -> list:
    """Names of the functions include/h3attn.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(h3attn_[a-z_]+)\s*\(", text)))


def _status_string(status: int) -> str:
    try:
        return library().h3attn_status_string(status).decode()
    except Exception:  # pragma: no cover - only when the library is missing
        return "status"


def _check(call: str, status: int) -> None:
    if status != 0:
        raise H3AttnError(call, status, library().h3attn_last_error().decode())


def _torch():
    import torch
    return torch


def _stream_handle(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _require_bf16_cuda(name: str, t) -> None:
    torch = _torch()
    if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError("%s must be a CUDA bfloat16 tensor" % name)
    if t.stride(-1) != 1:
        raise ValueError("%s: the last dimension must be contiguous" % name)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _same_device(device, **tensors) -> None:
    for name, t in tensors.items():
        if t is not None and t.device != device:
            raise ValueError("%s is on %s, the inputs on %s" % (name, t.device, device))


def _require_out(name: str, t, shape, device) -> None:
    """An output the kernels write row by row through its strides: its shape must
    be exactly the one the call produces (a smaller view would be written past its
    end) and it must live on the inputs' device."""
    _require_bf16_cuda(name, t)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))
    _same_device(device, **{name: t})


def _require_rope_inputs(pos, kind, n_tokens: int, device) -> None:
    torch = _torch()
    if pos is None:
        return
    if pos.dtype != torch.int32 or not pos.is_cuda or not pos.is_contiguous():
        raise TypeError("pos must be a contiguous CUDA int32 tensor [n_tokens, 3]")
    if kind is None or kind.dtype != torch.uint8 or not kind.is_cuda or not kind.is_contiguous():
        raise TypeError("kind must be a contiguous CUDA uint8 tensor [n_tokens]")
    if tuple(pos.shape) != (n_tokens, 3) or kind.numel() != n_tokens:
        raise ValueError("pos must be [%d, 3] and kind [%d]" % (n_tokens, n_tokens))
    _same_device(device, pos=pos, kind=kind)


def _require_gamma(name: str, g, head_dim: int, device) -> None:
    if g is None:
        return
    _require_bf16_cuda(name, g)
    if g.numel() != head_dim:
        raise ValueError("%s must hold head_dim = %d values" % (name, head_dim))
    _same_device(device, **{name: g})


def _strides(t, ndim: int):
    """The first `ndim` strides of t ({batch, token, head} or {token, head}) for the
    C ABI; a dimension of extent <= 1 is never stepped over, so a stride torch
    reports for it that the library would reject (0, or not a multiple of 8
    elements) is passed as 8."""
    s = [t.stride(i) for i in range(ndim)]
    for i in range(ndim):
        if t.shape[i] <= 1 and (s[i] <= 0 or s[i] % 8):
            s[i] = 8
    return (_I64_3 if ndim == 3 else _I64_2)(*s)


def _strides3(t):
    return _strides(t, 3)


def _strides2(t):
    return _strides(t, 2)


def device_status(stream=None, clear: bool = True) -> None:
    """Synchronise `stream` and raise if a kernel recorded a device-side failure (a
    timed-out wait, or a block-sparse key list that broke its rules)."""
    _check("h3attn_device_status", library().h3attn_device_status(_stream_handle(stream), int(clear)))


def selftest_wait_timeout(stream=None) -> None:
    """Enqueue the bounded-wait self-test: a kernel whose one wait can never
    complete gives up after about a second and records a timeout, which the next
    device_status() raises (and clears)."""
    _check("h3attn_selftest_wait_timeout", library().h3attn_selftest_wait_timeout(_stream_handle(stream)))


def prologue(q, k, q_out=None, k_out=None, gamma_q=None, gamma_k=None, eps: float = 1e-6,
             pos=None, kind=None, sections: Sequence[int] = (32, 48, 48), theta: float = 10000.0,
             stream=None) -> Tuple[object, object]:
    """RMSNorm (when gamma is given) then RoPE (when pos is given) of q and k.

    q, k: bf16 CUDA [n_tokens, n_heads, head_dim] views with equal strides (e.g. two
    slices of one fused QKV buffer).  q_out/k_out default to new contiguous tensors;
    pass q_out=q, k_out=k for in-place.  pos: int32 [n_tokens, 3]; kind: uint8 [n_tokens].
    """
    torch = _torch()
    _require_bf16_cuda("q", q)
    _require_bf16_cuda("k", k)
    if q.dim() != 3 or q.shape != k.shape or q.stride() != k.stride():
        raise ValueError("q and k must be [n_tokens, n_heads, head_dim] with equal shapes and strides")
    _same_device(q.device, k=k)
    if q_out is None:
        q_out = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    if k_out is None:
        k_out = torch.empty(k.shape, dtype=k.dtype, device=k.device)
    _require_out("q_out", q_out, q.shape, q.device)
    _require_out("k_out", k_out, q.shape, q.device)
    if q_out.stride() != k_out.stride():
        raise ValueError("q_out and k_out must share strides")
    n, h, d = q.shape
    _require_gamma("gamma_q", gamma_q, d, q.device)
    _require_gamma("gamma_k", gamma_k, d, q.device)
    _require_rope_inputs(pos, kind, n, q.device)
    st, sh, sw = sections
    si, so = _strides2(q), _strides2(q_out)
    _check("h3attn_prologue", library().h3attn_prologue(
        _ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), n, h, d, si[0], si[1],
        so[0], so[1], _ptr(gamma_q), _ptr(gamma_k), float(eps), _ptr(pos),
        _ptr(kind), st, sh, sw, float(theta), _stream_handle(stream)))
    return q_out, k_out


def attention(q, k, v, o=None, softmax_scale: Optional[float] = None, return_lse: bool = False,
              stream=None):
    """softmax(q k^T * scale) v, non-causal, per (batch, head).

    q, k, v: bf16 CUDA [B, N, H, d] or [N, H, d] (any strides, last dim contiguous).
    Returns o (same layout as q, new contiguous tensor unless `o` is given) and,
    with return_lse, lse fp32 [B, H, N] (natural log)."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16_cuda(name, t)
    squeeze = q.dim() == 3
    if squeeze:
        q, k, v = q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0)
        if o is not None:
            o = o.unsqueeze(0)
    if q.dim() != 4 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share a [B, N, H, d] shape")
    _same_device(q.device, k=k, v=v)
    B, N, H, d = q.shape
    if o is None:
        o = torch.empty((B, N, H, d), dtype=q.dtype, device=q.device)
    _require_out("o", o, (B, N, H, d), q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if return_lse else None
    st = _strides3
    _check("h3attn_fwd", library().h3attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, N, H, d, st(q), st(k), st(v), st(o),
        float(softmax_scale or 0.0), _ptr(lse), _stream_handle(stream)))
    out = o.squeeze(0) if squeeze else o
    if return_lse:
        return out, (lse.squeeze(0) if squeeze else lse)
    return out


def attention_varlen(q, k, v, cu_seqlens, max_seqlen: int, o=None,
                     softmax_scale: Optional[float] = None, return_lse: bool = False, stream=None):
    """Attention over ragged sequences packed along tokens.

    q, k, v: bf16 CUDA [total, H, d]; cu_seqlens: CUDA int32 [nseq + 1].
    Returns o [total, H, d] and, with return_lse, lse fp32 [H, total]."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16_cuda(name, t)
    if q.dim() != 3 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must share a [total, H, d] shape")
    if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_cuda or not cu_seqlens.is_contiguous():
        raise TypeError("cu_seqlens must be a contiguous CUDA int32 tensor")
    _same_device(q.device, k=k, v=v, cu_seqlens=cu_seqlens)
    total, H, d = q.shape
    if o is None:
        o = torch.empty((total, H, d), dtype=q.dtype, device=q.device)
    _require_out("o", o, (total, H, d), q.device)
    lse = torch.empty((H, total), dtype=torch.float32, device=q.device) if return_lse else None
    st = _strides2
    _check("h3attn_fwd_varlen", library().h3attn_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu_seqlens), cu_seqlens.numel() - 1, total,
        int(max_seqlen), H, d, st(q), st(k), st(v), st(o), float(softmax_scale or 0.0), _ptr(lse),
        _stream_handle(stream)))
    return (o, lse) if return_lse else o


def attention_kv(q, k, v, o=None, softmax_scale: Optional[float] = None, return_lse: bool = False,
                 stream=None):
    """Queries against a key/value set of its own length (one block of a split key set).

    q: bf16 CUDA [B, Nq, H, d] or [Nq, H, d]; k, v: [B, Nk, H, d] or [Nk, H, d], Nk >= 0.
    Returns o (layout of q) and, with return_lse, lse fp32 [B, H, Nq]; Nk = 0 gives
    o = 0 and lse = -inf."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16_cuda(name, t)
    squeeze = q.dim() == 3
    if squeeze:
        q, k, v = q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0)
        if o is not None:
            o = o.unsqueeze(0)
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("q must be [B, Nq, H, d] and k, v one [B, Nk, H, d] shape")
    B, Nq, H, d = q.shape
    if k.shape[0] != B or k.shape[2:] != q.shape[2:]:
        raise ValueError("k, v must match q in batch, heads and head_dim")
    Nk = k.shape[1]
    _same_device(q.device, k=k, v=v)
    if o is None:
        o = torch.empty((B, Nq, H, d), dtype=q.dtype, device=q.device)
    _require_out("o", o, (B, Nq, H, d), q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if return_lse else None
    st = _strides3
    _check("h3attn_fwd_kv", library().h3attn_fwd_kv(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Nq, Nk, H, d, st(q), st(k), st(v), st(o),
        float(softmax_scale or 0.0), _ptr(lse), _stream_handle(stream)))
    out = o.squeeze(0) if squeeze else o
    if return_lse:
        return out, (lse.squeeze(0) if squeeze else lse)
    return out


def attention_block_sparse(q, k, v, blk_off, blk_idx, o=None, softmax_scale: Optional[float] = None,
                           return_lse: bool = False, stream=None):
    """Attention in which each group of 256 query rows sees only listed tiles of 128 keys.

    q: bf16 CUDA [B, Nq, H, d] or [Nq, H, d]; k, v: [B, Nk, H, d] or [Nk, H, d].
    blk_off: int32 CUDA [B*H*ceil(Nq/256) + 1] offsets into blk_idx; list
    (b*H + h)*ceil(Nq/256) + qp holds the strictly ascending key tiles (of 128 keys)
    that query rows [256 qp, 256 qp + 256) of (b, h) attend to.  Returns o and, with
    return_lse, lse fp32 [B, H, Nq]; an empty list gives o = 0 and lse = -inf.  A list
    that breaks the rules is reported by the next device_status()."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16_cuda(name, t)
    for name, t in (("blk_off", blk_off), ("blk_idx", blk_idx)):
        if not (t.is_cuda and t.dtype == torch.int32 and t.is_contiguous()):
            raise TypeError("%s must be a contiguous int32 CUDA tensor" % name)
    squeeze = q.dim() == 3
    if squeeze:
        q, k, v = q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0)
        if o is not None:
            o = o.unsqueeze(0)
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("q must be [B, Nq, H, d] and k, v one [B, Nk, H, d] shape")
    B, Nq, H, d = q.shape
    if k.shape[0] != B or k.shape[2:] != q.shape[2:]:
        raise ValueError("k, v must match q in batch, heads and head_dim")
    Nk = k.shape[1]
    n_lists = B * H * (-(-Nq // 256))
    if blk_off.numel() != n_lists + 1:
        raise ValueError("blk_off must have B*H*ceil(Nq/256) + 1 = %d entries" % (n_lists + 1))
    _same_device(q.device, k=k, v=v, blk_off=blk_off, blk_idx=blk_idx)
    if blk_idx.numel() == 0:
        blk_idx = torch.zeros(1, dtype=torch.int32, device=q.device)  # never read: every list is empty
    if o is None:
        o = torch.empty((B, Nq, H, d), dtype=q.dtype, device=q.device)
    _require_out("o", o, (B, Nq, H, d), q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device) if return_lse else None
    st = _strides3
    _check("h3attn_fwd_block_sparse", library().h3attn_fwd_block_sparse(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), B, Nq, Nk, H, d, st(q), st(k), st(v), st(o), _ptr(blk_off),
        _ptr(blk_idx), float(softmax_scale or 0.0), _ptr(lse), _stream_handle(stream)))
    out = o.squeeze(0) if squeeze else o
    if return_lse:
        return out, (lse.squeeze(0) if squeeze else lse)
    return out


def merge(o_a, lse_a, o_b, lse_b, o=None, lse=None, stream=None):
    """Combine two partial results of the same queries over disjoint key sets.

    o_a, o_b: bf16 CUDA [B, N, H, d] or [N, H, d]; lse_a, lse_b: fp32 CUDA [B, H, N]
    or [H, N] (contiguous).  Returns (o, lse); o = o_a and lse = lse_a (or the b
    pair) merge in place."""
    torch = _torch()
    for name, t in (("o_a", o_a), ("o_b", o_b)):
        _require_bf16_cuda(name, t)
    squeeze = o_a.dim() == 3
    if squeeze:
        o_a, o_b = o_a.unsqueeze(0), o_b.unsqueeze(0)
        lse_a, lse_b = lse_a.unsqueeze(0), lse_b.unsqueeze(0)
        o = None if o is None else o.unsqueeze(0)
        lse = None if lse is None else lse.unsqueeze(0)
    if o_a.dim() != 4 or o_b.shape != o_a.shape:
        raise ValueError("o_a and o_b must share a [B, N, H, d] shape")
    B, N, H, d = o_a.shape
    for name, t in (("lse_a", lse_a), ("lse_b", lse_b)):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != (B, H, N):
            raise TypeError("%s must be a contiguous CUDA float32 [B, H, N] tensor" % name)
    _same_device(o_a.device, o_b=o_b, lse_a=lse_a, lse_b=lse_b)
    if o is None:
        o = torch.empty((B, N, H, d), dtype=o_a.dtype, device=o_a.device)
    _require_out("o", o, (B, N, H, d), o_a.device)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=o_a.device)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or tuple(lse.shape) != (B, H, N):
        raise TypeError("lse must be a contiguous float32 [B, H, N] tensor")
    _same_device(o_a.device, lse=lse)
    st = _strides3
    _check("h3attn_merge", library().h3attn_merge(
        _ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(o), _ptr(lse), B, N, H, d,
        st(o_a), st(o_b), st(o), _stream_handle(stream)))
    if squeeze:
        return o.squeeze(0), lse.squeeze(0)
    return o, lse


def qkv_fused(x, w, n_heads: int, bias=None, q_out=None, k_out=None, v_out=None, gamma_q=None, gamma_k=None,
              eps: float = 1e-6, pos=None, kind=None, sections: Sequence[int] = (32, 48, 48),
              theta: float = 10000.0, stream=None):
    """Q/K/V projection x w^T (+ bias) with RMSNorm + RoPE of Q and K in its epilogue.

    x: bf16 CUDA [n_tokens, dim_in] (last dim contiguous); w: bf16 CUDA [3*H*d, dim_in]
    contiguous; bias: [3*H*d] or None.  Returns (q, k, v), each [n_tokens, H, d]
    (new contiguous tensors unless the *_out views are given)."""
    torch = _torch()
    _require_bf16_cuda("x", x)
    _require_bf16_cuda("w", w)
    if x.dim() != 2 or w.dim() != 2 or w.shape[1] != x.shape[1] or not w.is_contiguous():
        raise ValueError("x must be [n_tokens, dim_in] and w a contiguous [3*H*d, dim_in]")
    n, dim_in = x.shape
    H = int(n_heads)
    if w.shape[0] % (3 * H):
        raise ValueError("w must have 3 * n_heads * head_dim rows")
    d = w.shape[0] // (3 * H)
    _same_device(x.device, w=w)
    outs = []
    for name, t in (("q_out", q_out), ("k_out", k_out), ("v_out", v_out)):
        if t is None:
            t = torch.empty((n, H, d), dtype=x.dtype, device=x.device)
        _require_out(name, t, (n, H, d), x.device)
        outs.append(t)
    if bias is not None:
        _require_bf16_cuda("bias", bias)
        if bias.numel() != 3 * H * d:
            raise ValueError("bias must hold 3 * n_heads * head_dim = %d values" % (3 * H * d))
        _same_device(x.device, bias=bias)
    _require_gamma("gamma_q", gamma_q, d, x.device)
    _require_gamma("gamma_k", gamma_k, d, x.device)
    _require_rope_inputs(pos, kind, n, x.device)
    st, sh, sw = sections
    tok = _I64_3(*(max(t.stride(0), 8) if n <= 1 else t.stride(0) for t in outs))
    hst = _I64_3(*(t.stride(1) for t in outs))
    _check("h3attn_qkv_fused", library().h3attn_qkv_fused(
        _ptr(x), _ptr(w), _ptr(bias), _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]), n, dim_in, H, d,
        max(x.stride(0), dim_in) if n <= 1 else x.stride(0), tok, hst, _ptr(gamma_q), _ptr(gamma_k), float(eps),
        _ptr(pos), _ptr(kind), st, sh, sw, float(theta), _stream_handle(stream)))
    return tuple(outs)
