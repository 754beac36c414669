"""Pins of the fp64 oracle against things other than itself.

Each pin takes an ``oracle.Oracle`` instance so that the same checks run on the
real oracle (tests/test_oracle_pins.py) and on deliberately broken copies of it
(tests/test_oracle_mutants.py), which must each fail at least one pin.

What pins what:
  bf16 rounding   exhaustive nearest-value search over all finite bfloat16
                  values in exact rational arithmetic (ties to the even pattern);
  RMSNorm         closed form of a constant row; unit RMS at eps = 0;
                  power-of-two scale invariance; one-hot gamma;
                  torch.nn.functional.rms_norm in float64 (library routine);
  RoPE            unit-vector images measured against mpmath angles (pins the
                  pairing, sign, section offsets and frequency ladder);
                  complex multiplication form; norm preservation; relative
                  position property; identities at position 0 / kind 0;
  norm + RoPE     one row recomputed step by step in 50-digit mpmath;
  RoPE cancel     rows whose rotated elements nearly cancel, against 50-digit
                  mpmath (fp64 value and bf16 rounding);
  attention       50-digit mpmath brute force (o and lse) on a ragged case;
                  torch scaled_dot_product_attention in float64; Q = 0 gives
                  the mean of V; one key gives V_0; constant V; permutation
                  invariance; a dominant key; isolation between sequences;
                  sampled rows equal full rows.
  block-sparse    torch scaled_dot_product_attention in float64 with the
                  boolean mask the block lists describe (built by plain loops);
                  a tiny case by 50-digit mpmath brute force; all blocks
                  listed equals unmasked attention; rows with no key give the
                  empty sum.
"""
from __future__ import annotations

import bisect
import math
from fractions import Fraction

import mpmath
import numpy as np
import torch

mpmath.mp.dps = 50

# ----------------------------------------------------------------------------------
# helpers independent of the oracle
# ----------------------------------------------------------------------------------


def _bits_to_float(b: int) -> float:
    return float(np.array([b << 16], dtype=np.uint32).view(np.float32)[0])


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_bf16_bits_f32(x: np.ndarray) -> np.ndarray:
    """float -> bf16 bits via float32 (used only to make test inputs)."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


_POS_TABLE = None


def _positive_table():
    """(sorted exact values, bit patterns) of all finite non-negative bfloat16 values."""
    global _POS_TABLE
    if _POS_TABLE is None:
        vals, bits = [], []
        for b in range(0, 0x7F80):
            vals.append(Fraction(_bits_to_float(b)))
            bits.append(b)
        _POS_TABLE = (vals, bits)
    return _POS_TABLE


def nearest_bf16_bits(x: float) -> int:
    """Brute force: the bf16 pattern nearest to x, ties to the even pattern."""
    if math.isnan(x):
        raise ValueError("nan")
    sign = 0x8000 if math.copysign(1.0, x) < 0 else 0
    if math.isinf(x):
        return sign | 0x7F80
    ax = Fraction(abs(x))
    vals, bits = _positive_table()
    if ax > vals[-1]:
        # between the largest finite value (odd pattern 0x7F7F) and 2^128 (infinity,
        # even pattern 0x7F80): the nearer wins, a tie goes to the even one
        return sign | (0x7F7F if ax - vals[-1] < Fraction(2) ** 128 - ax else 0x7F80)
    i = bisect.bisect_left(vals, ax)
    cands = [j for j in (i - 1, i) if 0 <= j < len(vals)]
    best = min(cands, key=lambda j: (abs(vals[j] - ax), bits[j] & 1))
    return sign | bits[best]


def _close(a, b, rtol, atol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    err = np.abs(a - b)
    lim = atol + rtol * np.abs(b)
    if not np.all(err <= lim):
        i = int(np.argmax(err - lim))
        raise AssertionError("%s: max violation at %d: got %r want %r" % (what, i, a.ravel()[i], b.ravel()[i]))


# ----------------------------------------------------------------------------------
# bf16 rounding
# ----------------------------------------------------------------------------------


def pin_bf16_rounding(orc):
    rng = np.random.default_rng(7)
    xs = list(rng.standard_normal(400) * np.exp2(rng.integers(-30, 30, 400)))
    # exact bf16 values, exact midpoints (ties), and their double neighbours
    for b in list(rng.integers(1, 0x7F7F, 200)) + [0x3F80, 0x3F81, 0x0001, 0x007F, 0x0080, 0x7F7E]:
        lo, hi = _bits_to_float(int(b)), _bits_to_float(int(b) + 1)
        mid = (lo + hi) / 2.0
        xs += [lo, mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf), -mid]
    xs += [0.0, -0.0, 1e-45, 3.0e38, 3.4e38, -3.39e38, 1e-40, -1e-39, 2.0 ** -133, 3 * 2.0 ** -134]
    got = orc.bf16_round(np.array(xs))
    for x, g in zip(xs, got):
        want = nearest_bf16_bits(float(x))
        if int(g) != want:
            raise AssertionError("bf16 rounding of %r: got %#06x want %#06x" % (x, int(g), want))


# ----------------------------------------------------------------------------------
# RMSNorm
# ----------------------------------------------------------------------------------


def pin_rmsnorm(orc):
    d, H = 128, 3
    rng = np.random.default_rng(11)
    # constant rows: y = c / sqrt(c^2 + eps) * g
    cs = np.array([0.75, -2.5, 0.001953125])
    x = np.repeat(to_bf16_bits_f32(cs)[:, None, None], H * d, axis=1).reshape(3, H, d)
    g = to_bf16_bits_f32(rng.uniform(0.5, 1.5, d))
    eps = 1e-6
    y, _ = orc.rmsnorm_rope(x, g, eps, want_bf16=False)
    c = bf16_value(to_bf16_bits_f32(cs))
    want = (np.sign(c) / np.sqrt(1.0 + eps / c ** 2))[:, None, None] * bf16_value(g)[None, None, :]
    _close(y, np.broadcast_to(want, y.shape), 1e-14, 0, "rmsnorm constant row")

    # eps = 0, gamma = 1: every output row has RMS exactly 1
    xr = to_bf16_bits_f32(rng.standard_normal((5, H, d)))
    ones = to_bf16_bits_f32(np.ones(d))
    y0, _ = orc.rmsnorm_rope(xr, ones, 0.0, want_bf16=False)
    _close(np.sqrt(np.mean(y0 ** 2, axis=-1)), np.ones((5, H)), 1e-14, 0, "rmsnorm unit rms")

    # power-of-two scale invariance at eps = 0 (exact in binary floating point)
    x4 = to_bf16_bits_f32(bf16_value(xr) * 4.0)
    y4, _ = orc.rmsnorm_rope(x4, g, 0.0, want_bf16=False)
    yg, _ = orc.rmsnorm_rope(xr, g, 0.0, want_bf16=False)
    _close(y4, yg, 1e-15, 0, "rmsnorm scale invariance")

    # one-hot gamma: only that element survives
    for kk in (0, 37, d - 1):
        oh = np.zeros(d)
        oh[kk] = 1.0
        yo, _ = orc.rmsnorm_rope(xr, to_bf16_bits_f32(oh), eps, want_bf16=False)
        assert np.all(yo[..., np.arange(d) != kk] == 0.0), "rmsnorm one-hot gamma leaks"
        xv = bf16_value(xr)
        _close(yo[..., kk], xv[..., kk] / np.sqrt(np.mean(xv ** 2, -1) + eps), 1e-13, 0,
               "rmsnorm one-hot gamma value")

    # library routine: torch rms_norm in float64 (weight = gamma)
    xt = torch.from_numpy(bf16_value(xr))
    ref = torch.nn.functional.rms_norm(xt, (d,), weight=torch.from_numpy(bf16_value(g)), eps=eps)
    y1, _ = orc.rmsnorm_rope(xr, g, eps, want_bf16=False)
    _close(y1, ref.numpy(), 1e-13, 1e-15, "rmsnorm vs torch.rms_norm")


# ----------------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------------

SECTIONS = (32, 48, 48)
THETA = 10000.0


def _mp_angle(kind, pos, pair, d=128, sections=SECTIONS, theta=THETA):
    """Angle of pair `pair` in 50-digit arithmetic, from the stated reading."""
    if kind == 2:
        return mpmath.mpf(int(pos[0])) * mpmath.power(theta, mpmath.mpf(-2 * pair) / d)
    st, sh, sw = sections
    dim = 2 * pair
    if dim < st:
        axis, i, ds = 0, pair, st
    elif dim < st + sh:
        axis, i, ds = 1, pair - st // 2, sh
    else:
        axis, i, ds = 2, pair - (st + sh) // 2, sw
    return mpmath.mpf(int(pos[axis])) * mpmath.power(theta, mpmath.mpf(-2 * i) / ds)


def pin_rope_unit_vectors(orc):
    d = 128
    for kind, pos in ((1, (3, 17, 83)), (1, (31, 0, 5)), (2, (255, 0, 0)), (2, (31233, 0, 0))):
        # rows: e_0, e_1, e_2, ... (each row one unit vector), as 1 head
        eye = to_bf16_bits_f32(np.eye(d))[:, None, :]
        p = np.tile(np.array(pos, dtype=np.int32), (d, 1))
        kd = np.full(d, kind, dtype=np.uint8)
        y, _ = orc.rmsnorm_rope(eye, None, 0.0, p, kd, SECTIONS, THETA, want_bf16=False)
        y = y[:, 0, :]
        for pair in range(d // 2):
            a = _mp_angle(kind, pos, pair)
            c, s = float(mpmath.cos(a)), float(mpmath.sin(a))
            want_even = np.zeros(d)
            want_even[2 * pair], want_even[2 * pair + 1] = c, s
            want_odd = np.zeros(d)
            want_odd[2 * pair], want_odd[2 * pair + 1] = -s, c
            # the angle itself is a double: allow a few of its ulps (large positions)
            tol = 1e-15 + 1e-15 * abs(float(a))
            _close(y[2 * pair], want_even, 0, tol, "rope e_%d kind %d pos %s" % (2 * pair, kind, pos))
            _close(y[2 * pair + 1], want_odd, 0, tol, "rope e_%d kind %d pos %s" % (2 * pair + 1, kind, pos))


def pin_rope_properties(orc):
    d, H, n = 128, 2, 40
    rng = np.random.default_rng(5)
    x = to_bf16_bits_f32(rng.standard_normal((n, H, d)))
    pos = np.stack([rng.integers(0, 32, n), rng.integers(0, 48, n), rng.integers(0, 84, n)], 1).astype(np.int32)
    kind = rng.integers(0, 3, n).astype(np.uint8)
    y, _ = orc.rmsnorm_rope(x, None, 0.0, pos, kind, SECTIONS, THETA, want_bf16=False)
    xv = bf16_value(x)
    # complex form: (x0 + i x1) * exp(i a)
    for t in range(n):
        if kind[t] == 0:
            assert np.array_equal(y[t], xv[t]), "kind 0 must be the identity"
            continue
        ang = np.array([float(_mp_angle(int(kind[t]), pos[t], i)) for i in range(d // 2)])
        z = (xv[t, :, 0::2] + 1j * xv[t, :, 1::2]) * np.exp(1j * ang)[None, :]
        _close(y[t, :, 0::2], z.real, 1e-12, 1e-13, "rope complex form (real)")
        _close(y[t, :, 1::2], z.imag, 1e-12, 1e-13, "rope complex form (imag)")
    # norm preservation
    _close(np.linalg.norm(y, axis=-1), np.linalg.norm(xv, axis=-1), 1e-14, 0, "rope norm")
    # position 0 is the identity for both kinds
    y0, _ = orc.rmsnorm_rope(x, None, 0.0, np.zeros_like(pos), np.maximum(kind, 1), SECTIONS, THETA,
                             want_bf16=False)
    _close(y0, xv, 0, 0, "rope at position 0")
    # relative position: <R(q, p + D), R(k, p' + D)> == <R(q, p), R(k, p')>
    q, k = x[:20], x[20:]
    pq, pk = pos[:20], pos[20:]
    for kd_val in (1, 2):
        kd = np.full(20, kd_val, dtype=np.uint8)
        shift = np.array([7, 11, 13], dtype=np.int32)
        a_q, _ = orc.rmsnorm_rope(q, None, 0.0, pq, kd, SECTIONS, THETA, want_bf16=False)
        a_k, _ = orc.rmsnorm_rope(k, None, 0.0, pk, kd, SECTIONS, THETA, want_bf16=False)
        b_q, _ = orc.rmsnorm_rope(q, None, 0.0, pq + shift, kd, SECTIONS, THETA, want_bf16=False)
        b_k, _ = orc.rmsnorm_rope(k, None, 0.0, pk + shift, kd, SECTIONS, THETA, want_bf16=False)
        _close(np.sum(b_q * b_k, -1), np.sum(a_q * a_k, -1), 0, 1e-11, "rope relative position")


def pin_norm_then_rope(orc):
    """One row through RMSNorm then RoPE, recomputed in 50-digit arithmetic."""
    d = 128
    rng = np.random.default_rng(3)
    x = to_bf16_bits_f32(rng.standard_normal((2, 1, d)) * 1.7)
    g = to_bf16_bits_f32(rng.uniform(0.5, 1.5, d))
    pos = np.array([[5, 9, 70], [200, 0, 0]], dtype=np.int32)
    kind = np.array([1, 2], dtype=np.uint8)
    eps = 1e-6
    y, y16 = orc.rmsnorm_rope(x, g, eps, pos, kind, SECTIONS, THETA)
    for t in range(2):
        xs = [mpmath.mpf(float(v)) for v in bf16_value(x[t, 0])]
        gs = [mpmath.mpf(float(v)) for v in bf16_value(g)]
        r = mpmath.sqrt(mpmath.fsum(v * v for v in xs) / d + mpmath.mpf(eps))
        nrm = [xs[i] / r * gs[i] for i in range(d)]
        want = []
        for pair in range(d // 2):
            a = _mp_angle(int(kind[t]), pos[t], pair)
            c, s = mpmath.cos(a), mpmath.sin(a)
            want += [nrm[2 * pair] * c - nrm[2 * pair + 1] * s, nrm[2 * pair] * s + nrm[2 * pair + 1] * c]
        want = np.array([float(w) for w in want])
        _close(y[t, 0], want, 1e-12, 1e-14, "norm then rope, row %d" % t)
        wb = np.array([nearest_bf16_bits(float(w)) for w in want], dtype=np.uint16)
        if not np.array_equal(y16[t, 0], wb):
            raise AssertionError("norm then rope: bf16 rounding of row %d differs" % t)


def pin_rope_cancellation(orc):
    """Rows whose rotated elements nearly cancel (x1 ~ x0 cos/sin, or x1 ~ -x0 sin/cos,
    to the rounding of x1): the results are thousands of times smaller than their
    terms; each is recomputed in 50-digit arithmetic and the oracle's bf16 rounding
    must be the nearest bf16 of that value (and its fp64 value within a few double
    ulps of the terms)."""
    d = 128
    rng = np.random.default_rng(11)
    toks = [(2, (4097, 0, 0)), (2, (31233, 0, 0)), (1, (17, 40, 83)), (1, (3, 5, 7))]
    n = len(toks)
    pos = np.array([t[1] for t in toks], dtype=np.int32)
    kind = np.array([t[0] for t in toks], dtype=np.uint8)
    x = np.zeros((n, 1, d))
    for t, (kd, p) in enumerate(toks):
        for pair in range(d // 2):
            a = _mp_angle(kd, p, pair)
            c, s = float(mpmath.cos(a)), float(mpmath.sin(a))
            x0 = float(bf16_value(to_bf16_bits_f32(np.array([rng.uniform(0.5, 2.0) * rng.choice([-1.0, 1.0])])))[0])
            ratio = c / s if (pair % 2 == 0 and s != 0.0) else (-s / c if c != 0.0 else 0.0)
            x1 = x0 * ratio if 1.0 / 64 < abs(ratio) < 64.0 else rng.uniform(-2.0, 2.0)
            x[t, 0, 2 * pair], x[t, 0, 2 * pair + 1] = x0, x1
    xb = to_bf16_bits_f32(x)
    y, y16 = orc.rmsnorm_rope(xb, None, 0.0, pos, kind, SECTIONS, THETA)
    xv = bf16_value(xb)
    tiny = 0
    for t, (kd, p) in enumerate(toks):
        for pair in range(d // 2):
            a = _mp_angle(kd, p, pair)
            c, s = mpmath.cos(a), mpmath.sin(a)
            x0, x1 = mpmath.mpf(float(xv[t, 0, 2 * pair])), mpmath.mpf(float(xv[t, 0, 2 * pair + 1]))
            for j, w in ((2 * pair, x0 * c - x1 * s), (2 * pair + 1, x0 * s + x1 * c)):
                scale = float(abs(x0) + abs(x1))
                if abs(y[t, 0, j] - float(w)) > 4e-16 * scale * (1.0 + abs(float(a))):
                    raise AssertionError("rope cancellation: token %d element %d: %r against %s" % (t, j, y[t, 0, j], w))
                if int(y16[t, 0, j]) != nearest_bf16_bits(float(w)):
                    raise AssertionError("rope cancellation: bf16 of token %d element %d differs" % (t, j))
                tiny += abs(float(w)) < 1e-3 * scale
    if tiny < n * d // 4:
        raise AssertionError("rope cancellation: too few cancelling elements (%d)" % tiny)


# ----------------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------------


def _mp_attention(q, k, v, cu, scale):
    """o, lse of every row by 50-digit brute force (small inputs only)."""
    qv, kv, vv = bf16_value(q), bf16_value(k), bf16_value(v)
    total, H, d = q.shape
    o = np.zeros((total, H, d))
    lse = np.zeros((total, H))
    sc = mpmath.mpf(scale)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        for t in range(a, b):
            for h in range(H):
                sj = [sc * mpmath.fsum(mpmath.mpf(float(qv[t, h, i])) * mpmath.mpf(float(kv[j, h, i]))
                                       for i in range(d)) for j in range(a, b)]
                e = [mpmath.exp(x) for x in sj]
                den = mpmath.fsum(e)
                for i in range(d):
                    o[t, h, i] = float(mpmath.fsum(e[j - a] * mpmath.mpf(float(vv[j, h, i]))
                                                   for j in range(a, b)) / den)
                lse[t, h] = float(mpmath.log(den))
    return o, lse


def pin_attention_brute_force(orc):
    rng = np.random.default_rng(17)
    cu = np.array([0, 1, 3, 7], dtype=np.int32)
    H, d = 2, 8
    q = to_bf16_bits_f32(rng.standard_normal((7, H, d)) * 2)
    k = to_bf16_bits_f32(rng.standard_normal((7, H, d)))
    v = to_bf16_bits_f32(rng.standard_normal((7, H, d)))
    scale = 0.37
    o, lse = orc.attention(q, k, v, cu, scale)
    wo, wl = _mp_attention(q, k, v, cu, scale)
    _close(o, wo, 1e-13, 1e-15, "attention vs mpmath (o)")
    _close(lse, wl, 1e-13, 1e-15, "attention vs mpmath (lse)")


def pin_attention_library(orc):
    rng = np.random.default_rng(19)
    N, H, d = 37, 3, 16
    q = to_bf16_bits_f32(rng.standard_normal((N, H, d)))
    k = to_bf16_bits_f32(rng.standard_normal((N, H, d)))
    v = to_bf16_bits_f32(rng.standard_normal((N, H, d)))
    o, lse = orc.attention(q, k, v, [0, N])
    qt, kt, vt = (torch.from_numpy(bf16_value(a)).permute(1, 0, 2) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(1, 0, 2).numpy()
    _close(o, ref, 1e-12, 1e-14, "attention vs torch sdpa float64")
    s = torch.einsum("hnd,hmd->hnm", qt, kt) / math.sqrt(d)
    _close(lse, torch.logsumexp(s, -1).T.numpy(), 1e-12, 1e-14, "lse vs torch.logsumexp")


def pin_attention_special_cases(orc):
    rng = np.random.default_rng(23)
    H, d = 2, 64
    cu = np.array([0, 1, 9, 40], dtype=np.int32)
    total = int(cu[-1])
    q = to_bf16_bits_f32(rng.standard_normal((total, H, d)))
    k = to_bf16_bits_f32(rng.standard_normal((total, H, d)))
    v = to_bf16_bits_f32(rng.standard_normal((total, H, d)))
    vv = bf16_value(v)
    # Q = 0: every key has the same score, o = mean of the sequence's V rows
    o, lse = orc.attention(np.zeros_like(q), k, v, cu)
    for s in range(3):
        a, b = cu[s], cu[s + 1]
        _close(o[a:b], np.broadcast_to(vv[a:b].mean(0), o[a:b].shape), 1e-14, 1e-15, "Q=0 mean of V")
        _close(lse[a:b], np.full((b - a, H), math.log(b - a)), 1e-14, 1e-15, "Q=0 lse = log n")
    # one key: o = v_0, lse = scale * q . k_0
    o, lse = orc.attention(q, k, v, cu)
    _close(o[0], vv[0], 0, 0, "single key gives v_0")
    _close(lse[0], np.sum(bf16_value(q[0]) * bf16_value(k[0]), -1) / 8.0, 1e-14, 0, "single key lse")
    # constant V rows inside a sequence reproduce that row
    vc = v.copy()
    vc[9:40] = v[20]
    oc, _ = orc.attention(q, k, vc, cu)
    _close(oc[9:40], np.broadcast_to(vv[20], oc[9:40].shape), 1e-14, 1e-15, "constant V")
    # permuting (K, V) rows together inside a sequence changes nothing
    perm = np.arange(total)
    perm[9:40] = 9 + rng.permutation(31)
    op, lp = orc.attention(q, k[perm], v[perm], cu)
    _close(op, o, 1e-13, 1e-15, "permutation invariance (o)")
    _close(lp, lse, 1e-13, 1e-15, "permutation invariance (lse)")
    # a dominant key: q = 0 except one dimension; huge scale -> o = v of the best key
    qd = np.zeros_like(q)
    qd[:, :, 0] = to_bf16_bits_f32(np.ones(1))[0]
    kd = k.copy()
    kd[:, :, 0] = to_bf16_bits_f32(np.linspace(-1, 1, total))[:, None]
    od, _ = orc.attention(qd, kd, v, cu, scale=1e4)
    for s in range(3):
        a, b = cu[s], cu[s + 1]
        best = a + int(np.argmax(bf16_value(kd[a:b, 0, 0])))
        _close(od[a:b], np.broadcast_to(vv[best], od[a:b].shape), 0, 1e-12, "dominant key")
    # sequences do not see each other
    k2, v2 = k.copy(), v.copy()
    k2[9:40] = to_bf16_bits_f32(rng.standard_normal((31, H, d)))
    v2[9:40] = to_bf16_bits_f32(rng.standard_normal((31, H, d)))
    oi, _ = orc.attention(q, k2, v2, cu)
    _close(oi[:9], o[:9], 0, 0, "isolation between sequences")
    # sampled rows are the same as the full computation
    rows = np.array([39, 0, 8, 9, 25], dtype=np.int64)
    orows, lrows = orc.attention(q, k, v, cu, rows=rows)
    _close(orows, o[rows], 0, 0, "sampled rows (o)")
    _close(lrows, lse[rows], 0, 0, "sampled rows (lse)")


# ----------------------------------------------------------------------------------
# partial attention over a split key set, and the log-sum-exp merge
# ----------------------------------------------------------------------------------


def pin_attention_kv_library(orc):
    """Queries against a key set of another length: torch SDPA in float64."""
    rng = np.random.default_rng(29)
    Nq, Nk, H, d = 23, 41, 2, 16
    q = to_bf16_bits_f32(rng.standard_normal((Nq, H, d)) * 1.5)
    k = to_bf16_bits_f32(rng.standard_normal((Nk, H, d)))
    v = to_bf16_bits_f32(rng.standard_normal((Nk, H, d)))
    o, lse = orc.attention_kv(q, k, v)
    qt, kt, vt = (torch.from_numpy(bf16_value(a)).permute(1, 0, 2) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).permute(1, 0, 2).numpy()
    _close(o, ref, 1e-12, 1e-14, "attention_kv vs torch sdpa float64")
    sc = torch.einsum("hnd,hmd->hnm", qt, kt) / math.sqrt(d)
    _close(lse, torch.logsumexp(sc, -1).T.numpy(), 1e-12, 1e-14, "attention_kv lse vs torch.logsumexp")
    # segments: each segment's queries see only its own key rows; an empty key range is the empty sum
    cu_q, cu_k = [0, 5, 5, 23], [0, 17, 30, 30]
    os_, ls = orc.attention_kv(q, k[:30], v[:30], cu_q, cu_k)
    o0, l0 = orc.attention_kv(q[:5], k[:17], v[:17])
    _close(os_[:5], o0, 0, 0, "attention_kv segment 0")
    _close(ls[:5], l0, 0, 0, "attention_kv segment 0 lse")
    _close(os_[5:], np.zeros((18, H, d)), 0, 0, "empty key range gives o = 0")
    assert np.all(np.isneginf(ls[5:])), "empty key range gives lse = -inf"
    # the mpmath brute force of the self-attention pins applies with cu_q == cu_k
    cu = np.array([0, 2, 6], dtype=np.int32)
    qs = to_bf16_bits_f32(rng.standard_normal((6, 1, 8)))
    ks = to_bf16_bits_f32(rng.standard_normal((6, 1, 8)))
    vs = to_bf16_bits_f32(rng.standard_normal((6, 1, 8)))
    ob, lb = orc.attention_kv(qs, ks, vs, cu, cu, scale=0.61)
    wo, wl = _mp_attention(qs, ks, vs, cu, 0.61)
    _close(ob, wo, 1e-13, 1e-15, "attention_kv vs mpmath (o)")
    _close(lb, wl, 1e-13, 1e-15, "attention_kv vs mpmath (lse)")


def pin_merge(orc):
    """Merging the parts of a split key set gives the attention over all keys."""
    rng = np.random.default_rng(31)
    Nq, Nk, H, d = 19, 64, 3, 16
    q = to_bf16_bits_f32(rng.standard_normal((Nq, H, d)) * 2)
    k = to_bf16_bits_f32(rng.standard_normal((Nk, H, d)))
    v = to_bf16_bits_f32(rng.standard_normal((Nk, H, d)))
    full_o, full_l = orc.attention_kv(q, k, v)
    for cuts in ([0, 30, 64], [0, 1, 2, 50, 64], [0, 0, 64], [0, 64, 64]):
        parts = [orc.attention_kv(q, k[a:b], v[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
        o, l = orc.merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
        _close(o, full_o, 1e-13, 1e-15, "merge of %s equals the whole (o)" % cuts)
        _close(l, full_l, 1e-13, 1e-15, "merge of %s equals the whole (lse)" % cuts)
    # closed forms on synthetic parts
    a = rng.standard_normal((5, 8))
    b = rng.standard_normal((5, 8))
    la = rng.standard_normal(5)
    o, l = orc.merge(a[None], la[None])
    _close(o, a, 0, 0, "one part is itself")
    _close(l, la, 0, 0, "one part keeps its lse")
    o, l = orc.merge(np.stack([a, b]), np.stack([la, la]))
    _close(o, (a + b) / 2, 1e-15, 1e-15, "equal weights average")
    _close(l, la + math.log(2), 1e-15, 1e-15, "equal weights add log 2")
    lb = la + math.log(3)  # b carries three times a's weight
    o, l = orc.merge(np.stack([a, b]), np.stack([la, lb]))
    _close(o, (a + 3 * b) / 4, 1e-14, 1e-15, "weights 1:3")
    _close(l, la + math.log(4), 1e-14, 1e-15, "lse of weights 1:3")
    o2, l2 = orc.merge(np.stack([b, a]), np.stack([lb, la]))
    _close(o2, o, 1e-15, 0, "order of parts")
    ninf = np.full(5, -np.inf)
    o, l = orc.merge(np.stack([a, b]), np.stack([la, ninf]))
    _close(o, a, 1e-15, 0, "an empty part carries no weight")
    o, l = orc.merge(np.stack([a, b]), np.stack([ninf, ninf]))
    _close(o, np.zeros_like(a), 0, 0, "all parts empty gives o = 0")
    assert np.all(np.isneginf(l)), "all parts empty gives lse = -inf"
    # large lse values: the max shift keeps it finite (the inputs la + 900 are only
    # good to ulp(900) ~ 1.1e-13, which bounds the agreement)
    o, l = orc.merge(np.stack([a, b]), np.stack([la + 900.0, la + 900.0 + math.log(3)]))
    _close(o, (a + 3 * b) / 4, 1e-12, 1e-12, "weights 1:3 at lse ~ 900")


# ----------------------------------------------------------------------------------
# Q/K/V projection fused with the prologue
# ----------------------------------------------------------------------------------


def pin_qkv_projection(orc):
    """The projection against numpy's float64 matmul; with identity weights the fused
    operation is the pinned prologue itself."""
    rng = np.random.default_rng(37)
    n, H, d = 21, 2, 16
    dim_in = 40
    x = to_bf16_bits_f32(rng.standard_normal((n, dim_in)))
    w = to_bf16_bits_f32(rng.standard_normal((3 * H * d, dim_in)) * 0.2)
    b = to_bf16_bits_f32(rng.standard_normal(3 * H * d))
    (q, k, v), _ = orc.qkv_norm_rope(x, w, b, n_heads=H, want_bf16=False)
    ref = bf16_value(x) @ bf16_value(w).T + bf16_value(b)
    _close(q.reshape(n, -1), ref[:, :H * d], 1e-13, 1e-13, "Q projection vs numpy")
    _close(k.reshape(n, -1), ref[:, H * d:2 * H * d], 1e-13, 1e-13, "K projection vs numpy")
    _close(v.reshape(n, -1), ref[:, 2 * H * d:], 1e-13, 1e-13, "V projection vs numpy")
    # identity weights: Q, K, V are x itself, so norm + RoPE equal the prologue of x
    sec = (4, 6, 6)
    x2 = to_bf16_bits_f32(rng.standard_normal((n, H * d)))
    eye = np.eye(H * d)
    wi = to_bf16_bits_f32(np.concatenate([eye, eye, eye], axis=0))
    gq = to_bf16_bits_f32(rng.uniform(0.5, 1.5, d))
    gk = to_bf16_bits_f32(rng.uniform(0.5, 1.5, d))
    pos = rng.integers(0, 20, size=(n, 3)).astype(np.int32)
    kind = (np.arange(n) % 3).astype(np.uint8)
    (q, k, v), (q16, _, v16) = orc.qkv_norm_rope(x2, wi, None, n_heads=H, gamma_q=gq, gamma_k=gk, pos=pos,
                                                 kind=kind, sections=sec)
    xh = x2.reshape(n, H, d)
    rq, rq16 = orc.rmsnorm_rope(xh, gq, 1e-6, pos, kind, sec)
    rk, _ = orc.rmsnorm_rope(xh, gk, 1e-6, pos, kind, sec)
    _close(q, rq, 1e-15, 1e-15, "identity weights: Q = prologue(x)")
    _close(k, rk, 1e-15, 1e-15, "identity weights: K = prologue(x) with gamma_k")
    assert np.array_equal(q16, rq16), "identity weights: rounded Q = rounded prologue"
    assert np.array_equal(v16, xh), "identity weights: V = x"
    # sampled rows are the full computation's rows
    rows = np.array([20, 0, 7], dtype=np.int64)
    (qs, _, _), _ = orc.qkv_norm_rope(x2, wi, None, n_heads=H, gamma_q=gq, gamma_k=gk, pos=pos, kind=kind,
                                      sections=sec, rows=rows)
    _close(qs, q[rows], 0, 0, "sampled rows")


def _block_mask(B, H, n_q, n_kv, block_q, block_k, off, idx):
    """Boolean [B, H, n_q, n_kv] visibility from CSR block lists, by direct loops."""
    n_qb = -(-n_q // block_q)
    mask = np.zeros((B, H, n_q, n_kv), dtype=bool)
    for b in range(B):
        for h in range(H):
            for qb in range(n_qb):
                c = (b * H + h) * n_qb + qb
                for e in range(int(off[c]), int(off[c + 1])):
                    kb = int(idx[e])
                    mask[b, h, qb * block_q:(qb + 1) * block_q, kb * block_k:(kb + 1) * block_k] = True
    return mask


def pin_attention_block_sparse(orc):
    """Block-sparse attention against torch scaled_dot_product_attention in
    float64 with the equivalent boolean mask (lists unsorted, with repeats and
    empty ones; a partial last key block; n_q != n_kv); all blocks listed equals
    plain attention; rows that see no key give o = 0, lse = -inf."""
    rng = np.random.default_rng(23)
    B, H, n_q, n_kv, d = 2, 2, 37, 29, 16
    bq, bk = 6, 8  # slips that swap the two sizes stay inside the buffers
    n_qb, n_kb = -(-n_q // bq), -(-n_kv // bk)
    q = to_bf16_bits_f32(rng.standard_normal((B, n_q, H, d)))
    k = to_bf16_bits_f32(rng.standard_normal((B, n_kv, H, d)))
    v = to_bf16_bits_f32(rng.standard_normal((B, n_kv, H, d)))
    lists = []
    for c in range(B * H * n_qb):
        n = int(rng.integers(0, n_kb + 2)) if c % 5 else 0
        lists.append(list(rng.integers(0, n_kb, size=n)))
    off = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int32)
    idx = np.array([e for x in lists for e in x], dtype=np.int32)
    scale = 0.29
    o, lse = orc.attention_block_sparse(q, k, v, off, idx, bq, bk, scale)
    mask = _block_mask(B, H, n_q, n_kv, bq, bk, off, idx)
    qt, kt, vt = (torch.from_numpy(bf16_value(a)).permute(0, 2, 1, 3) for a in (q, k, v))
    s = torch.einsum("bhnd,bhmd->bhnm", qt, kt) * scale
    mt = torch.from_numpy(mask)
    seen = mask.any(-1)  # [B, H, n_q]
    safe = mt | torch.from_numpy(~seen)[..., None]  # rows with no key: any mask (discarded)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=safe, scale=scale)
    ref = ref.permute(0, 2, 1, 3).numpy().reshape(B * n_q, H, d)
    ref_lse = torch.logsumexp(s.masked_fill(~safe, -math.inf), -1).permute(0, 2, 1).numpy().reshape(B * n_q, H)
    vis = seen.transpose(0, 2, 1).reshape(B * n_q, H)
    if vis.all() or not vis.any():
        raise AssertionError("block-sparse pin: the case must mix rows with and without keys")
    _close(o[vis], ref[vis], 1e-12, 1e-14, "block-sparse attention vs masked torch sdpa (o)")
    _close(lse[vis], ref_lse[vis], 1e-12, 1e-14, "block-sparse attention vs masked logsumexp (lse)")
    if not (np.all(o[~vis] == 0.0) and np.all(np.isneginf(lse[~vis]))):
        raise AssertionError("block-sparse attention: rows without keys must give o = 0, lse = -inf")
    # every block listed: plain attention of each batch entry
    full = [list(range(n_kb))] * (B * H * n_qb)
    off_f = np.arange(0, n_kb * len(full) + 1, n_kb, dtype=np.int32)
    idx_f = np.array([e for x in full for e in x], dtype=np.int32)
    o_f, lse_f = orc.attention_block_sparse(q, k, v, off_f, idx_f, bq, bk, scale)
    ref_f = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    _close(o_f, ref_f.permute(0, 2, 1, 3).numpy().reshape(B * n_q, H, d), 1e-12, 1e-14,
           "block-sparse with every block vs torch sdpa")
    _close(lse_f, torch.logsumexp(s, -1).permute(0, 2, 1).numpy().reshape(B * n_q, H), 1e-12, 1e-14,
           "block-sparse with every block: lse")
    # a tiny case by 50-digit brute force over the visible keys (blocks of 2 queries, 3 keys)
    qs, ks, vs = q[:1, :5, :1, :4].copy(), k[:1, :7, :1, :4].copy(), v[:1, :7, :1, :4].copy()
    lists_s = [[2, 0], [], [1, 1, 2]]  # unsorted, empty, repeated
    off_s = np.array([0, 2, 2, 5], dtype=np.int32)
    idx_s = np.array([e for x in lists_s for e in x], dtype=np.int32)
    o_s, lse_s = orc.attention_block_sparse(qs, ks, vs, off_s, idx_s, 2, 3, scale)
    qv, kv, vv = bf16_value(qs)[0, :, 0], bf16_value(ks)[0, :, 0], bf16_value(vs)[0, :, 0]
    for t in range(5):
        keys = sorted({j for b in lists_s[t // 2] for j in range(3 * b, min(3 * b + 3, 7))})
        if not keys:
            if not (np.all(o_s[t] == 0.0) and np.isneginf(lse_s[t, 0])):
                raise AssertionError("block-sparse brute force: row %d has no key" % t)
            continue
        sj = [mpmath.mpf(scale) * mpmath.fsum(mpmath.mpf(float(qv[t, i])) * mpmath.mpf(float(kv[j, i]))
                                              for i in range(4)) for j in keys]
        e = [mpmath.exp(x) for x in sj]
        den = mpmath.fsum(e)
        want = [float(mpmath.fsum(e[n] * mpmath.mpf(float(vv[j, i])) for n, j in enumerate(keys)) / den)
                for i in range(4)]
        _close(o_s[t, 0], want, 1e-13, 1e-15, "block-sparse vs mpmath, row %d" % t)
        _close(lse_s[t, 0], float(mpmath.log(den)), 1e-13, 1e-15, "block-sparse lse vs mpmath, row %d" % t)
    # sampled rows equal the same rows of the full result
    rows = np.array([0, 5, 40, 73], dtype=np.int64)
    o_r, lse_r = orc.attention_block_sparse(q, k, v, off, idx, bq, bk, scale, rows=rows)
    if not (np.array_equal(o_r, o[rows]) and np.array_equal(lse_r, lse[rows])):
        raise AssertionError("block-sparse attention: sampled rows differ from full rows")


ALL_PINS = [
    pin_bf16_rounding,
    pin_rmsnorm,
    pin_rope_unit_vectors,
    pin_rope_properties,
    pin_norm_then_rope,
    pin_rope_cancellation,
    pin_attention_brute_force,
    pin_attention_library,
    pin_attention_special_cases,
    pin_attention_kv_library,
    pin_merge,
    pin_qkv_projection,
    pin_attention_block_sparse,
]
