"""fp64 CPU oracle of the h3attn hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
library never loads it and shares no code with it.

The arithmetic lives in ``h3attn_oracle.c`` (plain C, double precision, OpenMP
over independent rows); this module only marshals numpy arrays through ctypes.
Each function cites the passage of the source pages it follows in the C file.

Parity status: every function is pinned by tests/test_oracle_pins.py (brute
force, closed forms, invariants, library routines on special cases); none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "h3attn_oracle.c")
LIBRARY = os.path.join(_HERE, "libh3attn_oracle.so")

CFLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-std=c11"]


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False) -> str:
    """Compile the oracle with gcc (plain IEEE double: no fast-math, no FMA contraction)."""
    if not force and os.path.exists(output) and os.path.getmtime(output) >= os.path.getmtime(source):
        return output
    tmp = output + ".tmp%d" % os.getpid()
    subprocess.run(["gcc", *CFLAGS, source, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, output)
    return output


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_D = ctypes.c_double


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """ctypes view of one compiled oracle library (the real one, or a test mutant)."""

    def __init__(self, path: Optional[str] = None):
        path = path or build()
        self.path = path
        lib = ctypes.CDLL(path)
        lib.h3o_bf16_from_double.restype = ctypes.c_uint16
        lib.h3o_bf16_from_double.argtypes = [_D]
        lib.h3o_bf16_round_array.restype = None
        lib.h3o_bf16_round_array.argtypes = [_P, _I64, _P]
        lib.h3o_rmsnorm_rope.restype = ctypes.c_int
        lib.h3o_rmsnorm_rope.argtypes = [_P, _I64, _I32, _I32, _I64, _I64, _P, _D, _P, _P,
                                         _I32, _I32, _I32, _D, _P, _P]
        lib.h3o_attention.restype = ctypes.c_int
        lib.h3o_attention.argtypes = [_P, _P, _P, _I64, _I32, _I32, _P, _I32, _D, _P, _I64, _P, _P]
        lib.h3o_attention_kv.restype = ctypes.c_int
        lib.h3o_attention_kv.argtypes = [_P, _I64, _P, _P, _I64, _I32, _I32, _P, _P, _I32, _D, _P, _P]
        lib.h3o_qkv_norm_rope.restype = ctypes.c_int
        lib.h3o_qkv_norm_rope.argtypes = [_P, _I64, _I32, _I64, _P, _P, _I32, _I32, _P, _P, _D, _P, _P,
                                          _I32, _I32, _I32, _D, _P, _I64, _P, _P, _P, _P, _P, _P]
        lib.h3o_merge.restype = ctypes.c_int
        lib.h3o_merge.argtypes = [_P, _P, _I32, _I64, _I32, _P, _P]
        lib.h3o_attention_block_sparse.restype = ctypes.c_int
        lib.h3o_attention_block_sparse.argtypes = [_P, _P, _P, _I32, _I64, _I64, _I32, _I32, _I32, _I32,
                                                   _P, _P, _D, _P, _I64, _P, _P]
        self.lib = lib

    # -- bfloat16 rounding --------------------------------------------------------
    def bf16_round(self, x) -> np.ndarray:
        """Nearest bfloat16 (ties to even) of each double, as uint16 bit patterns."""
        x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
        out = np.empty(x.shape, dtype=np.uint16)
        self.lib.h3o_bf16_round_array(_ptr(x), x.size, _ptr(out))
        return out

    # -- prologue -------------------------------------------------------------------
    def rmsnorm_rope(self, x: np.ndarray, gamma: Optional[np.ndarray] = None, eps: float = 1e-6,
                     pos: Optional[np.ndarray] = None, kind: Optional[np.ndarray] = None,
                     sections=(32, 48, 48), theta: float = 10000.0,
                     want_f64: bool = True, want_bf16: bool = True
                     ) -> Tuple[Optional[np.ndarray], Optional[np.ndarray]]:
        """RMSNorm then RoPE of x (bf16 bits [n_tokens, n_heads, d], any strides).

        Returns (y64 [n, H, d] float64 or None, y16 [n, H, d] uint16 or None)."""
        x = np.asarray(x, dtype=np.uint16)
        if x.ndim != 3:
            raise ValueError("x must be [n_tokens, n_heads, d]")
        n, H, d = x.shape
        if x.strides[2] != 2:
            x = np.ascontiguousarray(x)
        s_tok, s_head = x.strides[0] // 2, x.strides[1] // 2
        g = None if gamma is None else np.ascontiguousarray(gamma, dtype=np.uint16)
        p = None if pos is None else np.ascontiguousarray(pos, dtype=np.int32)
        kd = None if kind is None else np.ascontiguousarray(kind, dtype=np.uint8)
        y64 = np.empty((n, H, d), dtype=np.float64) if want_f64 else None
        y16 = np.empty((n, H, d), dtype=np.uint16) if want_bf16 else None
        st, sh, sw = sections
        base = x.__array_interface__["data"][0]
        rc = self.lib.h3o_rmsnorm_rope(ctypes.c_void_p(base), n, H, d, s_tok, s_head, _ptr(g),
                                       float(eps), _ptr(p), _ptr(kd), st, sh, sw, float(theta),
                                       _ptr(y64), _ptr(y16))
        if rc != 0:
            raise ValueError("oracle rmsnorm_rope rejected its arguments (%d)" % rc)
        return y64, y16

    # -- attention ------------------------------------------------------------------
    def attention(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens,
                  scale: Optional[float] = None, rows: Optional[np.ndarray] = None
                  ) -> Tuple[np.ndarray, np.ndarray]:
        """softmax(q k^T scale) v per sequence for the given query rows.

        q, k, v: bf16 bits [total, H, d].  Returns (o [nrows, H, d], lse [nrows, H])."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        total, H, d = q.shape
        cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
        nrows = total if r is None else len(r)
        o = np.empty((nrows, H, d), dtype=np.float64)
        lse = np.empty((nrows, H), dtype=np.float64)
        rc = self.lib.h3o_attention(_ptr(q), _ptr(k), _ptr(v), total, H, d, _ptr(cu), len(cu) - 1,
                                    float(scale), _ptr(r), nrows, _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle attention rejected its arguments (%d)" % rc)
        return o, lse

    def attention_kv(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_q=None, cu_k=None,
                     scale: Optional[float] = None) -> Tuple[np.ndarray, np.ndarray]:
        """Each segment's queries against that segment's rows of a separate key set.

        q: bf16 bits [total_q, H, d]; k, v: [total_k, H, d]; cu_q / cu_k: segment
        bounds (default: one segment each).  Returns (o [total_q, H, d], lse [total_q, H]);
        an empty key range gives o = 0, lse = -inf."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        total_q, H, d = q.shape
        k = np.ascontiguousarray(k, dtype=np.uint16).reshape(-1, H, d)
        v = np.ascontiguousarray(v, dtype=np.uint16).reshape(-1, H, d)
        total_k = k.shape[0]
        cq = np.ascontiguousarray([0, total_q] if cu_q is None else cu_q, dtype=np.int32)
        ck = np.ascontiguousarray([0, total_k] if cu_k is None else cu_k, dtype=np.int32)
        if len(cq) != len(ck):
            raise ValueError("cu_q and cu_k must have the same number of segments")
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        o = np.empty((total_q, H, d), dtype=np.float64)
        lse = np.empty((total_q, H), dtype=np.float64)
        rc = self.lib.h3o_attention_kv(_ptr(q), total_q, _ptr(k), _ptr(v), total_k, H, d, _ptr(cq),
                                       _ptr(ck), len(cq) - 1, float(scale), _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle attention_kv rejected its arguments (%d)" % rc)
        return o, lse

    def attention_block_sparse(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, blk_off, blk_idx,
                               block_q: int = 256, block_k: int = 128, scale: Optional[float] = None,
                               rows=None) -> Tuple[np.ndarray, np.ndarray]:
        """Attention of each query to the keys of the key blocks listed for its
        (batch, head, query block).

        q: bf16 bits [B, n_q, H, d]; k, v: [B, n_kv, H, d]; blk_off: int32 CSR offsets
        [B*H*ceil(n_q/block_q) + 1] into blk_idx (key-block indices).  rows: optional
        flat query rows b*n_q + t.  Returns (o [rows, H, d], lse [rows, H]) with
        rows = all B*n_q rows when not given; no visible key gives o = 0, lse = -inf."""
        q = np.ascontiguousarray(q, dtype=np.uint16)
        B, n_q, H, d = q.shape
        k = np.ascontiguousarray(k, dtype=np.uint16).reshape(B, -1, H, d)
        v = np.ascontiguousarray(v, dtype=np.uint16).reshape(B, -1, H, d)
        n_kv = k.shape[1]
        off = np.ascontiguousarray(blk_off, dtype=np.int32)
        idx = np.ascontiguousarray(blk_idx, dtype=np.int32)
        n_qb = -(-n_q // block_q)
        if off.shape != (B * H * n_qb + 1,):
            raise ValueError("blk_off must have B*H*ceil(n_q/block_q) + 1 entries")
        if idx.size < int(off[-1]):
            raise ValueError("blk_idx is shorter than blk_off[-1]")
        if scale is None:
            scale = 1.0 / np.sqrt(d)
        rws = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
        nrows = B * n_q if rws is None else rws.size
        o = np.empty((nrows, H, d), dtype=np.float64)
        lse = np.empty((nrows, H), dtype=np.float64)
        rc = self.lib.h3o_attention_block_sparse(
            _ptr(q), _ptr(k), _ptr(v), B, n_q, n_kv, H, d, block_q, block_k, _ptr(off),
            _ptr(idx) if idx.size else None, float(scale), None if rws is None else _ptr(rws), nrows,
            _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle attention_block_sparse rejected its arguments (%d)" % rc)
        return o, lse

    def merge(self, o_parts, lse_parts) -> Tuple[np.ndarray, np.ndarray]:
        """Combine partial results over disjoint key sets by their log-sum-exp.

        o_parts: [P, ..., d] (any float), lse_parts: [P, ...] matching o_parts[..., 0].
        Returns (o [..., d], lse [...]) in float64."""
        o_parts = np.asarray(o_parts, dtype=np.float64)
        lse_parts = np.asarray(lse_parts, dtype=np.float64)
        if o_parts.shape[:-1] != lse_parts.shape:
            raise ValueError("o_parts [P, ..., d] and lse_parts [P, ...] disagree")
        n_parts, d = o_parts.shape[0], o_parts.shape[-1]
        rows_shape = o_parts.shape[1:-1]
        n_rows = int(np.prod(rows_shape)) if rows_shape else 1
        op = np.ascontiguousarray(o_parts.reshape(n_parts, n_rows, d))
        lp = np.ascontiguousarray(lse_parts.reshape(n_parts, n_rows))
        o = np.empty((n_rows, d), dtype=np.float64)
        lse = np.empty(n_rows, dtype=np.float64)
        rc = self.lib.h3o_merge(_ptr(op), _ptr(lp), n_parts, n_rows, d, _ptr(o), _ptr(lse))
        if rc != 0:
            raise ValueError("oracle merge rejected its arguments (%d)" % rc)
        return o.reshape(*rows_shape, d), lse.reshape(rows_shape)

    def qkv_norm_rope(self, x: np.ndarray, w: np.ndarray, bias: Optional[np.ndarray] = None,
                      n_heads: int = 1, gamma_q=None, gamma_k=None, eps: float = 1e-6, pos=None,
                      kind=None, sections=(32, 48, 48), theta: float = 10000.0,
                      rows: Optional[np.ndarray] = None, want_f64: bool = True, want_bf16: bool = True):
        """Q/K/V projection x w^T (+ bias), then RMSNorm + RoPE of Q and K per head.

        x: bf16 bits [n_tokens, dim_in]; w: [3*H*d, dim_in]; bias: [3*H*d] or None.
        Returns ((q64, k64, v64), (q16, k16, v16)), each [nrows, H, d] (None where not
        wanted)."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w = np.ascontiguousarray(w, dtype=np.uint16)
        n, dim_in = x.shape
        H = int(n_heads)
        d = w.shape[0] // (3 * H)
        if w.shape != (3 * H * d, dim_in):
            raise ValueError("w must be [3*H*d, dim_in]")
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.uint16)
        gq = None if gamma_q is None else np.ascontiguousarray(gamma_q, dtype=np.uint16)
        gk = None if gamma_k is None else np.ascontiguousarray(gamma_k, dtype=np.uint16)
        p = None if pos is None else np.ascontiguousarray(pos, dtype=np.int32)
        kd = None if kind is None else np.ascontiguousarray(kind, dtype=np.uint8)
        r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
        nrows = n if r is None else len(r)
        o64 = [np.empty((nrows, H, d)) if want_f64 else None for _ in range(3)]
        o16 = [np.empty((nrows, H, d), dtype=np.uint16) if want_bf16 else None for _ in range(3)]
        st, sh, sw = sections
        rc = self.lib.h3o_qkv_norm_rope(_ptr(x), n, dim_in, dim_in, _ptr(w), _ptr(b), H, d, _ptr(gq),
                                        _ptr(gk), float(eps), _ptr(p), _ptr(kd), st, sh, sw, float(theta),
                                        _ptr(r), nrows, *(_ptr(a) for a in o64), *(_ptr(a) for a in o16))
        if rc != 0:
            raise ValueError("oracle qkv_norm_rope rejected its arguments (%d)" % rc)
        return tuple(o64), tuple(o16)

    # -- composition: the whole hot path ------------------------------------------------
    def prologue_workload(self, w, want_f64: bool = False):
        """Q', K' of a Workload: RMSNorm + RoPE, rounded once to bf16."""
        if not w.has_prologue:
            return (None, w.q), (None, w.k)
        qs = self.rmsnorm_rope(w.q, w.gamma_q, w.eps, w.pos, w.kind, w.sections, w.theta,
                               want_f64=want_f64)
        ks = self.rmsnorm_rope(w.k, w.gamma_k, w.eps, w.pos, w.kind, w.sections, w.theta,
                               want_f64=want_f64)
        return qs, ks


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The oracle built from h3attn_oracle.c (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default
