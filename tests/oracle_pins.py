"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes a loaded oracle library (the real one, or a copy
with a planted mistake) and raises AssertionError when the oracle disagrees
with an independent fact: numpy / torch number-format conversions, exact
rational arithmetic, numpy matmul, closed-form round trips, hand-worked
fixtures under ``tests/golden/``, and invariants of the definitions.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _hex(v):
    return int(v, 16)


# Independent decoders (numpy / torch), used to dequantize in the pins.
def np_half(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def torch_bf16(bits):
    b = torch.from_numpy(np.ascontiguousarray(np.asarray(bits, np.uint16)).view(np.int16))
    return b.view(torch.bfloat16).double().numpy()


def bf16_bits_from_f32(v):
    t = torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def dequant(q, s, z, g):
    """W_deq[n][k] = s (q - z) of k's group, via numpy's fp16 decode."""
    sf = np.repeat(np_half(s), g, axis=1)
    zf = np.repeat(np_half(z), g, axis=1)
    return sf * (q.astype(np.float64) - zf)


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def pin_half_decode_exhaustive(lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.half_to_double(bits, lib)
    ref = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def pin_half_encode_vs_numpy(lib):
    rng = np.random.default_rng(1)
    mags = np.concatenate([
        rng.uniform(-70000, 70000, 4000),
        rng.standard_normal(4000) * 2.0 ** rng.integers(-30, 16, 4000),
        rng.uniform(-1e-7, 1e-7, 1000),              # fp16 subnormal range
    ])
    # exact midpoints between neighbouring fp16 values (ties -> even)
    h = np.arange(0x0001, 0x7bff, 97, dtype=np.uint16)
    a = h.view(np.float16).astype(np.float64)
    b = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mids = (a + b) / 2
    special = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e6, 2.0 ** -25,
                        2.0 ** -24, 1.5 * 2.0 ** -24, 3 * 2.0 ** -26, np.inf, -np.inf])
    vals = np.concatenate([mags, mids, -mids, special])
    got = oracle.double_to_half(vals, lib)
    ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref), vals[got != ref][:5]


def pin_bf16_decode_exhaustive(lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_to_double(bits, lib)
    ref = torch_bf16(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def pin_bf16_encode_nearest_even(lib):
    rng = np.random.default_rng(2)
    # fp32-representable inputs: torch's float -> bf16 rounding is a single RNE step
    f32 = np.concatenate([
        (rng.standard_normal(6000) * 2.0 ** rng.integers(-140, 120, 6000)).astype(np.float32),
        np.array([0.0, -0.0, 3.3895314e38, 3.4e38, 1e-45, -1e-40], np.float32),
    ])
    got = oracle.double_to_bf16(f32.astype(np.float64), lib)
    ref = bf16_bits_from_f32(f32)
    assert np.array_equal(got, ref), f32[got != ref][:5]
    # general doubles: the result must be the nearest bf16, ties to even
    d = rng.standard_normal(3000) * 2.0 ** rng.integers(-120, 120, 3000)
    hb = np.arange(0x0080, 0x7f7f, 131, dtype=np.uint16)          # exact midpoints
    lo, hi = torch_bf16(hb), torch_bf16((hb + 1).astype(np.uint16))
    d = np.concatenate([d, (lo + hi) / 2])
    got = oracle.double_to_bf16(d, lib)
    v = torch_bf16(got)
    up = torch_bf16((got + 1).astype(np.uint16))
    dn = torch_bf16((got - 1).astype(np.uint16))
    for x, r, u, w, gb in zip(np.abs(d), np.abs(v), np.abs(up), np.abs(dn), got):
        err = abs(x - r)
        assert err <= abs(x - u) and err <= abs(x - w), (x, r)
        if err == abs(x - u) or err == abs(x - w):       # a tie: must be even
            assert (int(gb) & 1) == 0, (x, r)


# ---------------------------------------------------------------------------
# Quantization
# ---------------------------------------------------------------------------

def pin_quantize_hand_golden(lib):
    gd = _golden("quantize_hand.json")
    g = gd["group"]
    W = np.array([r["w"] for r in gd["rows"]], np.float16).view(np.uint16)
    q, s, z = oracle.quantize(W, g, lib)
    for i, r in enumerate(gd["rows"]):
        assert list(q[i]) == r["q"], (i, q[i], r["q"])
        assert int(s[i, 0]) == _hex(r["s"]), (i, hex(int(s[i, 0])))
        assert int(z[i, 0]) == _hex(r["z"]), (i, hex(int(z[i, 0])))


def pin_quantize_roundtrip(lib):
    """W = s (q - z) with s a power of two and codes 0 and 15 in every group:
    quantization returns exactly (q, s, z)."""
    rng = np.random.default_rng(3)
    N, K, g = 24, 64, 16
    G = K // g
    e = rng.integers(-12, 3, size=(N, G))
    s = 2.0 ** e
    z = rng.integers(0, 16, size=(N, G)).astype(np.float64)
    q = rng.integers(0, 16, size=(N, K))
    q[:, 0::g] = 0
    q[:, 1::g] = 15
    W = np.repeat(s, g, 1) * (q - np.repeat(z, g, 1))
    assert np.array_equal(W.astype(np.float16).astype(np.float64), W)
    qo, so, zo = oracle.quantize(W.astype(np.float16).view(np.uint16), g, lib)
    assert np.array_equal(qo, q.astype(np.uint8))
    assert np.array_equal(np_half(so), s)
    assert np.array_equal(np_half(zo), z)


def pin_quantize_error_bound(lib):
    """Codes in [0, 15]; every weight inside the representable range
    [s(0 - z), s(15 - z)] dequantizes to within s/2; the range endpoints of the
    group (min(0, w), max(0, w)) lie within one scale step of it."""
    rng = np.random.default_rng(4)
    N, K, g = 32, 256, 64
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    W[3, :64] = np.abs(W[3, :64])         # an all-positive group
    W[4, 64:128] = -np.abs(W[4, 64:128])  # an all-negative group
    q, s, z = oracle.quantize(W.view(np.uint16), g, lib)
    assert q.max() <= 15
    Wd = dequant(q, s, z, g)
    w = W.astype(np.float64)
    sf = np.repeat(np_half(s), g, 1)
    zf = np.repeat(np_half(z), g, 1)
    assert np.all(zf == np.round(zf)) and zf.min() >= 0 and zf.max() <= 15
    lo_r, hi_r = -sf * zf, sf * (15 - zf)
    inside = (w >= lo_r) & (w <= hi_r)
    assert inside.mean() > 0.95
    assert np.all(np.abs(w - Wd)[inside] <= sf[inside] / 2)
    assert np.all(np.abs(w - Wd) <= sf * 1.5)
    # zero is exactly representable: a zero weight dequantizes to 0
    Z = W.copy()
    Z[:, 5] = 0
    qz, sz_, zz = oracle.quantize(Z.view(np.uint16), g, lib)
    assert np.all(dequant(qz, sz_, zz, g)[:, 5] == 0)


def pin_quantize_rejects_nonfinite(lib):
    W = np.zeros((2, 64), np.float16)
    W[1, 7] = np.inf
    assert oracle.quantize_rc(W.view(np.uint16), 32, lib) == -1
    W[1, 7] = np.nan
    assert oracle.quantize_rc(W.view(np.uint16), 32, lib) == -1
    assert oracle.quantize_rc(np.zeros((2, 60), np.uint16), 32, lib) == -2


# ---------------------------------------------------------------------------
# Layout
# ---------------------------------------------------------------------------

def pin_layout_hand_golden(lib):
    gd = _golden("layout_hand.json")
    q = np.array(gd["q"], np.uint8)
    s = np.array([[_hex(v) for v in r] for r in gd["s"]], np.uint16)
    z = np.array([[_hex(v) for v in r] for r in gd["z"]], np.uint16)
    qw, sz = oracle.pack_layout(q, s, z, gd["group"], lib)
    assert qw.tolist() == [[_hex(v) for v in r] for r in gd["qweight"]]
    assert sz.tolist() == [[[_hex(v) for v in p] for p in r] for r in gd["sz"]]


def pin_layout_unpack(lib):
    rng = np.random.default_rng(5)
    N, K, g = 64, 96, 32
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    s = rng.integers(0, 0x7bff, (N, K // g)).astype(np.uint16)
    z = rng.integers(0, 0x7bff, (N, K // g)).astype(np.uint16)
    qw, sz = oracle.pack_layout(q, s, z, g, lib)
    lo = qw & 0x0F
    hi = qw >> 4
    un = np.empty((K, N), np.uint8)
    un[:, 0::2], un[:, 1::2] = lo, hi
    assert np.array_equal(un.T, q)
    assert np.array_equal(sz[..., 0].T, s) and np.array_equal(sz[..., 1].T, z)


# ---------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------

def pin_select_bruteforce(lib):
    rng = np.random.default_rng(6)
    for K, t in ((1, 0.0), (37, 0.5), (1000, 0.0), (4096, 0.7), (333, -1.0), (64, 10.0)):
        x = rng.standard_normal((1, K)).astype(np.float32)
        x[0, :: 7] = 0.0
        xb = bf16_bits_from_f32(x)
        ref = np.nonzero(np.abs(torch_bf16(xb)[0]) > t)[0]
        got = oracle.select(xb, [t], lib)
        assert np.array_equal(got, ref.astype(np.int32)), (K, t)


def pin_select_edges(lib):
    vals = np.array([0.0, -0.0, 1.0, -1.0, np.nan, np.inf, -np.inf, 0.5, -0.5, 2.0 ** -130],
                    np.float32)
    xb = bf16_bits_from_f32(vals[None, :])
    assert oracle.select(xb, [0.0], lib).tolist() == [2, 3, 5, 6, 7, 8, 9]   # nonzero, not NaN
    assert oracle.select(xb, [0.5], lib).tolist() == [2, 3, 5, 6]           # strict: 0.5 out
    assert oracle.select(xb, [-1.0], lib).tolist() == [0, 1, 2, 3, 5, 6, 7, 8, 9]  # NaN never
    assert oracle.select(xb, [np.inf], lib).tolist() == []


def pin_select_union(lib):
    rng = np.random.default_rng(7)
    B, K = 5, 700
    x = rng.standard_normal((B, K)).astype(np.float32)
    xb = bf16_bits_from_f32(x)
    t = rng.uniform(0.5, 2.0, B)
    t = t.astype(np.float32)
    got = oracle.select(xb, t, lib)
    ref = np.array([], np.int64)
    xd = torch_bf16(xb)
    for b in range(B):
        ref = np.union1d(ref, np.nonzero(np.abs(xd[b]) > t[b])[0])
    assert np.array_equal(got, ref.astype(np.int32))


# ---------------------------------------------------------------------------
# GEMV
# ---------------------------------------------------------------------------

def _small_problem(rng, N, K, g, B=1):
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    q, s, z = oracle.quantize(W.view(np.uint16), g)       # the real oracle builds inputs
    x = bf16_bits_from_f32(rng.standard_normal((B, K)).astype(np.float32))
    return q, s, z, x


def pin_gemv_hand_golden(lib):
    lay = _golden("layout_hand.json")
    gd = _golden("gemv_hand.json")
    q = np.array(lay["q"], np.uint8)
    s = np.array([[_hex(v) for v in r] for r in lay["s"]], np.uint16)
    z = np.array([[_hex(v) for v in r] for r in lay["z"]], np.uint16)
    for c in gd["cases"]:
        xb = bf16_bits_from_f32(np.array(c["x"], np.float32))
        idx = oracle.select(xb, c["t"], lib)
        assert idx.tolist() == c["idx"]
        y, sa, yb = oracle.gemv(q, s, z, lay["group"], xb, idx, lib)
        assert y.tolist() == c["y"] and sa.tolist() == c["sumabs"], (c, y, sa)
        assert np.array_equal(torch_bf16(yb), np.array(c["y"]))


def pin_gemv_dense_vs_matmul(lib):
    rng = np.random.default_rng(8)
    N, K, g, B = 48, 256, 64, 3
    q, s, z, x = _small_problem(rng, N, K, g, B)
    ref = torch_bf16(x) @ dequant(q, s, z, g).T
    y, sa, _ = oracle.gemv(q, s, z, g, x, np.arange(K, dtype=np.int32), lib)
    assert np.all(np.abs(y - ref) <= 1e-13 * sa + 1e-300)
    yd, sad, ybd = oracle.gemv_dense(q, s, z, g, x, lib)
    assert np.array_equal(yd, y) and np.array_equal(sad, sa)
    ref_abs = np.abs(torch_bf16(x)) @ np.abs(dequant(q, s, z, g)).T
    assert np.all(np.abs(sa - ref_abs) <= 1e-13 * ref_abs)


def pin_gemv_sparse_vs_masked_matmul(lib):
    rng = np.random.default_rng(9)
    N, K, g = 40, 320, 64
    q, s, z, x = _small_problem(rng, N, K, g)
    xd = torch_bf16(x)[0]
    t = float(np.median(np.abs(xd)))
    idx = oracle.select(x, [t], lib)
    mask = (np.abs(xd) > t).astype(np.float64)
    ref = dequant(q, s, z, g) @ (xd * mask)
    y, sa, _ = oracle.gemv(q, s, z, g, x, idx, lib)
    assert np.all(np.abs(y[0] - ref) <= 1e-13 * sa[0] + 1e-300)


def pin_gemv_threads(lib):
    """The OpenMP form against numpy matmul of the masked activations, and bit
    for bit against the one-thread form (each output keeps its sum order)."""
    rng = np.random.default_rng(21)
    N, K, g, B = 67, 384, 64, 3
    q, s, z, x = _small_problem(rng, N, K, g, B)
    xd = torch_bf16(x)
    t = [float(np.median(np.abs(xd[b]))) for b in range(B)]
    idx = oracle.select(x, t, lib)
    mask = np.zeros(K)
    mask[idx] = 1.0
    ref = (xd * mask) @ dequant(q, s, z, g).T
    y1, sa1, yb1 = oracle.gemv(q, s, z, g, x, idx, lib)
    for threads in (1, 2, 5):
        y, sa, yb = oracle.gemv(q, s, z, g, x, idx, lib, threads=threads)
        assert np.all(np.abs(y - ref) <= 1e-13 * sa + 1e-300)
        assert np.array_equal(y, y1) and np.array_equal(sa, sa1) and np.array_equal(yb, yb1)


def pin_gemv_all_masked(lib):
    rng = np.random.default_rng(10)
    q, s, z, x = _small_problem(rng, 16, 128, 32, 2)
    y, sa, yb = oracle.gemv(q, s, z, 32, x, np.zeros(0, np.int32), lib)
    assert np.all(y == 0) and not np.any(np.signbit(y)) and np.all(sa == 0)
    assert np.all(yb == 0)


def pin_gemv_exact_rational_bruteforce(lib):
    """Every one of the 2^K active sets on a tiny problem, against exact
    rational arithmetic written independently of the oracle."""
    rng = np.random.default_rng(11)
    N, K, g = 6, 8, 4
    q, s, z, x = _small_problem(rng, N, K, g)
    sf, zf, xd = np_half(s), np_half(z), torch_bf16(x)[0]
    W = [[Fraction(float(sf[n, k // g])) * (int(q[n, k]) - Fraction(float(zf[n, k // g])))
          for k in range(K)] for n in range(N)]
    X = [Fraction(float(v)) for v in xd]
    for mask in range(1 << K):
        idx = np.array([k for k in range(K) if mask >> k & 1], np.int32)
        y, sa, _ = oracle.gemv(q, s, z, g, x, idx, lib)
        for n in range(N):
            exact = sum((W[n][k] * X[k] for k in idx), Fraction(0))
            eabs = sum((abs(W[n][k] * X[k]) for k in idx), Fraction(0))
            assert abs(Fraction(y[0, n]) - exact) <= Fraction(2) ** -45 * eabs, (mask, n)
            assert abs(Fraction(sa[0, n]) - eabs) <= Fraction(2) ** -45 * eabs, (mask, n)


def pin_gemv_exact_integer_case(lib):
    """Power-of-two scales and small-integer x: every partial sum is exact, so
    y equals the rational result bit for bit."""
    rng = np.random.default_rng(12)
    N, K, g = 16, 64, 16
    G = K // g
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    s = (2.0 ** rng.integers(-3, 3, (N, G))).astype(np.float16).view(np.uint16)
    z = rng.integers(0, 16, (N, G)).astype(np.float16).view(np.uint16)
    xf = rng.integers(-8, 9, (1, K)).astype(np.float32)
    xb = bf16_bits_from_f32(xf)
    idx = np.nonzero(xf[0] != 0)[0].astype(np.int32)
    y, _, _ = oracle.gemv(q, s, z, g, xb, idx, lib)
    Wd = dequant(q, s, z, g)
    for n in range(N):
        exact = sum(Fraction(float(Wd[n, k])) * Fraction(float(xf[0, k])) for k in idx)
        assert Fraction(y[0, n]) == exact


def pin_gemv_permutation_invariance(lib):
    """Permuting channels inside each group, and whole groups, together with
    the matching weight columns leaves y unchanged (up to summation order)."""
    rng = np.random.default_rng(13)
    N, K, g = 32, 256, 64
    G = K // g
    q, s, z, x = _small_problem(rng, N, K, g)
    xd = torch_bf16(x)[0]
    t = float(np.quantile(np.abs(xd), 0.4))
    y0, sa0, _ = oracle.gemv(q, s, z, g, x, oracle.select(x, [t], lib), lib)
    gp = rng.permutation(G)
    perm = np.concatenate([gp[j] * g + rng.permutation(g) for j in range(G)])
    qp, xp = q[:, perm], x[:, perm]
    sp, zp = s[:, gp], z[:, gp]
    y1, sa1, _ = oracle.gemv(qp, sp, zp, g, xp, oracle.select(xp, [t], lib), lib)
    assert np.all(np.abs(y1 - y0) <= 1e-13 * sa0)
    assert np.all(np.abs(sa1 - sa0) <= 1e-13 * sa0)


def pin_gemv_power_of_two_scaling(lib):
    rng = np.random.default_rng(14)
    N, K, g = 24, 192, 64
    q, s, z, x = _small_problem(rng, N, K, g)
    xd = torch_bf16(x)
    t = float(np.median(np.abs(xd)))
    y0, _, _ = oracle.gemv(q, s, z, g, x, oracle.select(x, [t], lib), lib)
    for j in (-3, 5):
        x2 = bf16_bits_from_f32((xd * 2.0 ** j).astype(np.float32))
        y2, _, _ = oracle.gemv(q, s, z, g, x2, oracle.select(x2, [t * 2.0 ** j], lib), lib)
        assert np.array_equal(y2, y0 * 2.0 ** j)


def pin_gemv_batch_rows(lib):
    rng = np.random.default_rng(15)
    N, K, g, B = 24, 256, 64, 4
    q, s, z, x = _small_problem(rng, N, K, g, B)
    idx = oracle.select(x, [1.0] * B, lib)
    y, sa, _ = oracle.gemv(q, s, z, g, x, idx, lib)
    for b in range(B):
        yb, sab, _ = oracle.gemv(q, s, z, g, x[b:b + 1], idx, lib)
        assert np.array_equal(yb[0], y[b]) and np.array_equal(sab[0], sa[b])


# ---------------------------------------------------------------------------
# Gated activation
# ---------------------------------------------------------------------------

def pin_glu_relu_exact(lib):
    rng = np.random.default_rng(16)
    gv = np.concatenate([rng.standard_normal(3000), [0.0, -0.0, -1.0, 2.0]]).astype(np.float32)
    uv = np.concatenate([rng.standard_normal(3000), [-1.0, 1.0, -3.0, -0.5]]).astype(np.float32)
    g = bf16_bits_from_f32(gv)
    u = bf16_bits_from_f32(uv)
    h, hb = oracle.glu(g, u, 1, lib)
    gd, ud = torch_bf16(g), torch_bf16(u)
    ref = np.where(gd > 0, gd, 0.0) * ud
    assert np.array_equal(h, ref)
    assert (h == 0).mean() > 0.4
    ref_b = (torch.from_numpy(ref).float().to(torch.bfloat16)).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(hb, ref_b)   # products of two bf16 are exact in fp32


def pin_glu_silu(lib):
    rng = np.random.default_rng(17)
    gv = np.concatenate([rng.standard_normal(3000) * 3, [0.0, -0.0, 20.0, -20.0, 80.0, -80.0]])
    g = bf16_bits_from_f32(gv.astype(np.float32))
    u = bf16_bits_from_f32(rng.standard_normal(gv.size).astype(np.float32))
    h, _ = oracle.glu(g, u, 0, lib)
    gd, ud = torch.from_numpy(torch_bf16(g)), torch.from_numpy(torch_bf16(u))
    ref = (torch.nn.functional.silu(gd) * ud).numpy()
    assert np.all(np.abs(h - ref) <= 1e-14 * np.abs(ref) + 1e-300)
    assert h[-6] == 0.0


def pin_act_mul_closed_forms(lib):
    """fp64 gated activation: sigma(ln 3) = 3/4 gives SiLU(+-ln 3) in closed
    form; SiLU(g) - SiLU(-g) = g for every g; ReLU products are exact; h is
    linear in up; the bf16 output is the nearest bf16 of h."""
    l3 = np.log(3.0)
    h, _ = oracle.act_mul(np.array([l3, -l3, 0.0, -0.0]), np.ones(4), 0, lib)
    assert np.allclose(h, [0.75 * l3, -0.25 * l3, 0.0, 0.0], rtol=1e-15, atol=0)
    rng = np.random.default_rng(18)
    g = rng.standard_normal(2000) * 4
    hp, _ = oracle.act_mul(g, np.ones_like(g), 0, lib)
    hm, _ = oracle.act_mul(-g, np.ones_like(g), 0, lib)
    assert np.all(np.abs((hp - hm) - g) <= 1e-14 * (1 + np.abs(g)))
    u = rng.standard_normal(g.size)
    h1, _ = oracle.act_mul(g, u, 0, lib)
    h2, _ = oracle.act_mul(g, 2 * u, 0, lib)
    assert np.array_equal(h2, 2 * h1)
    hr, hb = oracle.act_mul(g, u, 1, lib)
    assert np.array_equal(hr, np.where(g > 0, g, 0.0) * u)
    # nearest bf16: no bf16 neighbour of the result is closer to h
    dec = np.array([oracle.bf16_to_double(int(b), lib) for b in hb[:300]])
    for d, hv, b in zip(dec, hr[:300], hb[:300]):
        for nb in (int(b) - 1, int(b) + 1):
            if 0 <= nb < 0x7f80 or 0x8000 <= nb < 0xff80:
                assert abs(oracle.bf16_to_double(nb, lib) - hv) >= abs(d - hv)


def pin_select_mask_bits(lib):
    """Bitmask of the active set: a hand fixture fixes the bit order (channel k
    is bit k % 32 of word k / 32), and brute force on random batches fixes the
    union and the strict comparison."""
    K = 72
    x = np.zeros((1, K), np.float32)
    for k in (0, 31, 32, 33, 63, 71):
        x[0, k] = 1.0
    x[0, 5] = 0.5                                   # equal to t: not active
    m, c = oracle.select_mask(bf16_bits_from_f32(x), [0.5], lib)
    assert m.tolist() == [0x80000001, 0x80000003, 0x80] and c == 6
    rng = np.random.default_rng(19)
    for B, K in ((1, 256), (3, 1000), (16, 136)):
        xv = rng.standard_normal((B, K)).astype(np.float32)
        xb = bf16_bits_from_f32(xv)
        t = np.abs(rng.standard_normal(B)).astype(np.float32)
        act = (np.abs(torch_bf16(xb).reshape(B, K)) > t[:, None]).any(axis=0)
        m, c = oracle.select_mask(xb, t, lib)
        words = np.zeros((K + 31) // 32, np.uint64)
        for k in np.nonzero(act)[0]:
            words[k // 32] |= np.uint64(1) << np.uint64(k % 32)
        assert np.array_equal(m.astype(np.uint64), words) and c == int(act.sum())


def _nm_fixture_weights():
    K, N = 32, 8
    W = np.zeros((N, K), np.float64)
    W[0, 0::2] = 15 / 16
    W[2, :] = 1 / 32
    W[3, 1::2] = 15 / 8
    W[4:8, :] = 15 / 16
    return W.astype(np.float16).view(np.uint16)


def pin_nm_layout_hand(lib):
    """The 2:4 choice and packed layout of a hand-worked case (largest sums of
    w^2, ties to the lower output, nibble and slot order, (s, z) per slot)."""
    d = _golden("nm_layout_hand.json")
    Wb = _nm_fixture_weights()
    g = d["group"]
    keep, bad = oracle.nm_keep(Wb, g, lib)
    assert keep.tolist() == d["keep_nibbles"] and not bad.any()
    q, s, z = oracle.quantize(Wb, g, lib)
    qw, kp, sz = oracle.pack_layout_nm(q, s, z, keep, bad, g, lib)
    h = lambda v: int(v, 16)
    assert kp.tolist() == [[h(v) for v in r] for r in d["keep_packed"]]
    even = [h(v) for v in d["qweight_even_row"]]
    odd = [h(v) for v in d["qweight_odd_row"]]
    for k in range(d["K"]):
        assert qw[k].tolist() == (even if k % 2 == 0 else odd), k
    assert sz.tolist() == [[[h(v) for v in pair] for pair in blk] for blk in d["sz"]]


def pin_nm_keep_brute_force(lib):
    """Brute force of the 2:4 choice on random weights with planted ties:
    sums of squares in numpy, a stable sort by (-energy, output)."""
    rng = np.random.default_rng(20)
    for N, K, g in ((16, 64, 32), (64, 256, 64), (32, 128, 128)):
        Wf = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
        Wf[5] = Wf[4]                       # equal energies inside a block
        Wf[8:12] = Wf[8]                    # a block of four equal rows
        Wf[13] = -Wf[12]                    # equal energy, opposite sign
        keep, bad = oracle.nm_keep(Wf.view(np.uint16), g, lib)
        assert not bad.any()
        Wd = Wf.astype(np.float64)
        for grp in range(K // g):
            e = (Wd[:, grp * g:(grp + 1) * g] ** 2).sum(axis=1)
            for j in range(N // 4):
                order = sorted(range(4), key=lambda i: (-e[4 * j + i], i))
                nib = (1 << order[0]) | (1 << order[1])
                assert keep[grp, j] == nib, (N, K, g, grp, j)
    Wf = (rng.standard_normal((8, 64)) * 0.02).astype(np.float16)
    Wf[6, 40] = np.float16(np.nan)
    keep, bad = oracle.nm_keep(Wf.view(np.uint16), 32, lib)
    assert bad.tolist() == [[0, 0], [0, 1]] and keep[1, 1] == 0x3


def pin_nm_gemv_is_gemv_of_pruned_weights(lib):
    """The 2:4 GEMV equals the plain GEMV of W with the pruned weights set to
    zero and quantized as usual (a zeroed group gets s = 1, z = 0, q = 0):
    every fp64 partial sum is the same, so y and sum |w x| agree bit for bit."""
    rng = np.random.default_rng(21)
    N, K, g = 32, 256, 64
    Wf = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    Wb = Wf.view(np.uint16)
    keep, bad = oracle.nm_keep(Wb, g, lib)
    q, s, z = oracle.quantize(Wb, g, lib)
    x = bf16_bits_from_f32(rng.standard_normal((2, K)).astype(np.float32))
    idx = oracle.select(x, [0.5, 0.7], lib)
    y, sa, yb = oracle.gemv_nm(q, s, z, keep, bad, g, x, idx, lib)
    Wp = Wf.copy()
    for grp in range(K // g):
        for n in range(N):
            if not (keep[grp, n // 4] >> (n % 4)) & 1:
                Wp[n, grp * g:(grp + 1) * g] = 0
    q2, s2, z2 = oracle.quantize(Wp.view(np.uint16), g, lib)
    y2, sa2, yb2 = oracle.gemv(q2, s2, z2, g, x, idx, lib)
    assert np.array_equal(y, y2) and np.array_equal(sa, sa2) and np.array_equal(yb, yb2)
    assert np.mean(y == 0) < 0.1          # the pruned GEMV is not trivially zero


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
