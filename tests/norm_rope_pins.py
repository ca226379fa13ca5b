"""Checks that pin the RMSNorm / rotary-embedding oracle
(oracle/norm_rope_oracle.py) to facts fixed outside itself.

* The bf16 rounding: hand-worked values (ties to even, and a value just above
  a tie that a rounding through fp32 would get wrong), and agreement with the
  bit-pattern rounding of the 4-bit weight oracle (oracle/w4_oracle.py, pinned
  separately) on values exact in fp32.
* RMSNorm: a hand-worked example (tests/golden/norm_rope_hand_examples.json);
  with eps = 0 the output of a unit-weight norm has mean square 1, is
  unchanged when x is scaled by c > 0, and equals x sqrt(d) / ||x||_2
  (numpy's 2-norm); its backward is the derivative of its forward (central
  finite differences).
* The rotation: scalar loops with Python complex numbers (the pair
  (a, b) = (q_i, q_{i+h}) as a + b j, turned by multiplying with cos + j sin);
  zero angle is the identity; with genuine tables (angle = position x
  10000^(-2i/head_dim)) the dot product of a rotated q and k depends only on
  the difference of their positions; the backward is the adjoint
  (<R x, y> = <x, R^T y>) and undoes the forward.
* The attention-input block: a hand-worked q (rotated) and v (not rotated)
  example, forward and backward; x_n is bf16 and within half a bf16 unit of
  the exact norm; the backward matches central finite differences of
  sum_j <dY_j, Y_j> in X (x_n unrounded), A_j and B_j.

Each ``check_*`` takes the module (or a copy with a planted mistake) and raises
AssertionError when it disagrees with the fact.
"""
from __future__ import annotations

import cmath
import json
import math
import os

import numpy as np

from oracle import w4_oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "norm_rope_hand_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _a(x):
    return np.array(x, dtype=np.float64)


def check_round_bf16_hand(o):
    u = 2.0 ** -8
    cases = [(1.0 + u, 1.0),                       # tie -> even (1.0)
             (1.0 + 3 * u, 1.0 + 4 * u),           # tie -> even (1 + 2^-6)
             (1.0 + u + 2.0 ** -30, 1.0 + 2 * u),  # just above a tie: up (fp32 would round to the tie first)
             (-(1.0 + u + 2.0 ** -30), -(1.0 + 2 * u)),
             (3.0, 3.0), (0.0, 0.0), (1.0 - 2.0 ** -10, 1.0), (0.1, 0.10009765625)]
    got = o.round_bf16(_a([c[0] for c in cases]))
    assert np.array_equal(got, _a([c[1] for c in cases])), got


def check_round_bf16_matches_bit_rounding(o):
    rng = np.random.default_rng(31)
    v = (rng.standard_normal(4000) * np.exp2(rng.integers(-20, 20, 4000))).astype(np.float32).astype(np.float64)
    assert np.array_equal(o.round_bf16(v), w4_oracle.round_to_bf16(v))


def check_rms_norm_hand(o):
    g = _golden()["rms_norm"]
    Xn, rstd = o.rms_norm(_a(g["X"]), _a(g["g"]), g["eps"])
    assert np.array_equal(rstd, _a(g["rstd"])), rstd
    assert np.array_equal(Xn, _a(g["Xn"])), Xn


def check_rms_norm_closed_forms(o):
    rng = np.random.default_rng(32)
    X = rng.standard_normal((5, 24)) * 3.0
    ones = np.ones(24)
    Xn, rstd = o.rms_norm(X, ones, 0.0)
    assert np.allclose(np.mean(Xn * Xn, axis=1), 1.0, rtol=1e-14, atol=0)
    Xn2, _ = o.rms_norm(X * 7.5, ones, 0.0)
    assert np.allclose(Xn2, Xn, rtol=1e-13, atol=1e-15)
    want = X * math.sqrt(24) / np.linalg.norm(X, axis=1)[:, None]
    assert np.allclose(Xn, want, rtol=1e-13, atol=1e-15)
    g = rng.standard_normal(24)
    Xg, _ = o.rms_norm(X, g, 0.0)
    assert np.allclose(Xg, want * g[None, :], rtol=1e-13, atol=1e-15)


def _fd(loss, base, h=1e-6):
    num = np.zeros_like(base)
    for idx in np.ndindex(base.shape):
        e = np.zeros_like(base)
        e[idx] = h
        num[idx] = (loss(base + e) - loss(base - e)) / (2 * h)
    return num


def _rel(num, got):
    return np.max(np.abs(num - got)) / max(1e-12, np.max(np.abs(num)))


def check_rms_norm_backward_finite_differences(o):
    rng = np.random.default_rng(33)
    X = rng.standard_normal((3, 10))
    g = rng.standard_normal(10)
    dXn = rng.standard_normal((3, 10))
    eps = 0.05
    num = _fd(lambda x: float(np.sum(dXn * o.rms_norm(x, g, eps)[0])), X)
    assert _rel(num, o.rms_norm_backward(dXn, X, g, eps)) <= 1e-7


def _tables(n_pos, head_dim, base=10000.0):
    h = head_dim // 2
    cos = np.empty((n_pos, h))
    sin = np.empty((n_pos, h))
    for p in range(n_pos):
        for i in range(h):
            ang = p * base ** (-2.0 * i / head_dim)
            cos[p, i] = math.cos(ang)
            sin[p, i] = math.sin(ang)
    return cos, sin


def check_rotary_complex_brute_force(o):
    rng = np.random.default_rng(34)
    M, hd, heads = 4, 8, 3
    h = hd // 2
    Z = rng.standard_normal((M, heads * hd))
    ang = rng.uniform(-3.2, 3.2, (6, h))
    cos, sin = np.cos(ang), np.sin(ang)
    pos = np.array([5, 0, 3, 3])
    got = o.apply_rotary(Z, pos, cos, sin, hd)
    for m in range(M):
        for hh in range(heads):
            for i in range(h):
                a, b = Z[m, hh * hd + i], Z[m, hh * hd + h + i]
                w = complex(a, b) * complex(cos[pos[m], i], sin[pos[m], i])
                assert abs(got[m, hh * hd + i] - w.real) <= 1e-14, (m, hh, i)
                assert abs(got[m, hh * hd + h + i] - w.imag) <= 1e-14, (m, hh, i)
                # the same turn through the polar form
                w2 = complex(a, b) * cmath.exp(1j * ang[pos[m], i])
                assert abs(w - w2) <= 1e-13


def check_rotary_zero_angle_and_quarter_turn(o):
    rng = np.random.default_rng(35)
    Z = rng.standard_normal((2, 16))
    cos, sin = _tables(4, 8)
    assert np.array_equal(o.apply_rotary(Z, np.array([0, 0]), cos, sin, 8), Z)
    q = np.array([[1.0, 2.0, 3.0, 4.0]])
    got = o.apply_rotary(q, np.array([0]), np.zeros((1, 2)), np.ones((1, 2)), 4)
    assert np.array_equal(got, np.array([[-3.0, -4.0, 1.0, 2.0]])), got


def check_rotary_relative_position(o):
    rng = np.random.default_rng(36)
    hd = 16
    cos, sin = _tables(64, hd)
    q = rng.standard_normal((1, 2 * hd))
    k = rng.standard_normal((1, 2 * hd))
    for p1, p2, c in ((5, 2, 11), (0, 9, 30), (17, 17, 4)):
        d1 = float(np.sum(o.apply_rotary(q, np.array([p1]), cos, sin, hd) * o.apply_rotary(k, np.array([p2]), cos, sin, hd)))
        d2 = float(np.sum(o.apply_rotary(q, np.array([p1 + c]), cos, sin, hd)
                          * o.apply_rotary(k, np.array([p2 + c]), cos, sin, hd)))
        assert abs(d1 - d2) <= 1e-10 * (1 + abs(d1)), (p1, p2, c, d1, d2)


def check_rotary_backward_is_adjoint(o):
    rng = np.random.default_rng(37)
    hd = 8
    cos, sin = _tables(10, hd)
    pos = np.array([3, 9, 0, 4, 4])
    x = rng.standard_normal((5, 3 * hd))
    y = rng.standard_normal((5, 3 * hd))
    lhs = float(np.sum(o.apply_rotary(x, pos, cos, sin, hd) * y))
    rhs = float(np.sum(x * o.apply_rotary_backward(y, pos, cos, sin, hd)))
    assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))
    back = o.apply_rotary_backward(o.apply_rotary(x, pos, cos, sin, hd), pos, cos, sin, hd)
    assert np.allclose(back, x, rtol=1e-13, atol=1e-14)


def _qkv_golden():
    g = _golden()["qkv"]
    projs = [{"W": _a(g["W_q"]), "A": _a(g["A_q"]), "B": _a(g["B_q"])},
             {"W": _a(g["W_v"]), "A": _a(g["A_v"]), "B": _a(g["B_v"])}]
    args = (_a(g["X"]), _a(g["g"]), g["eps"], projs, g["s"], [True, False], np.array(g["pos"]), _a(g["cos"]),
            _a(g["sin"]), g["head_dim"])
    return g, args


def check_qkv_hand_example(o):
    g, args = _qkv_golden()
    f = o.qkv_forward(*args)
    assert np.array_equal(f["Y"][0], _a(g["Y_q"])), f["Y"][0]
    assert np.array_equal(f["Y"][1], _a(g["Y_v"])), f["Y"][1]
    b = o.qkv_backward([_a(g["dY_q"]), _a(g["dY_v"])], *args)
    for key, j, want in (("dA", 0, "dA_q"), ("dB", 0, "dB_q"), ("dA", 1, "dA_v"), ("dB", 1, "dB_v")):
        assert np.array_equal(b[key][j], _a(g[want])), (key, j, b[key][j])
    assert np.array_equal(b["dX"], _a(g["dX"])), b["dX"]


def _qkv_problem(rng, M=3, d=16, hd=8, r=2):
    projs = []
    for d_out in (16, 8, 8):
        projs.append({"W": rng.standard_normal((d_out, d)) * 0.3, "A": rng.standard_normal((r, d)) * 0.3,
                      "B": rng.standard_normal((d_out, r)) * 0.3})
    ang = rng.uniform(-3.2, 3.2, (7, hd // 2))
    return {"X": rng.standard_normal((M, d)), "g": rng.standard_normal(d), "projs": projs,
            "pos": rng.integers(0, 7, M), "cos": np.cos(ang), "sin": np.sin(ang), "hd": hd,
            "dYs": [rng.standard_normal((M, pj["W"].shape[0])) for pj in projs]}


def check_qkv_xn_is_bf16(o):
    rng = np.random.default_rng(38)
    p = _qkv_problem(rng, M=4, d=32)
    f = o.qkv_forward(p["X"], p["g"], 1e-6, p["projs"], 0.5, [True, True, False], p["pos"], p["cos"], p["sin"], p["hd"])
    exact, _ = o.rms_norm(p["X"], p["g"], 1e-6)
    assert np.array_equal(w4_oracle.round_to_bf16(f["Xn"]), f["Xn"])     # representable in bf16
    _, e = np.frexp(exact)
    assert np.all(np.abs(f["Xn"] - exact) <= np.ldexp(1.0, e - 9))        # within half a bf16 unit
    assert not np.array_equal(f["Xn"], exact)


def check_qkv_finite_differences(o):
    rng = np.random.default_rng(39)
    p = _qkv_problem(rng)
    rot = [True, True, False]
    s, eps = 0.75, 0.01

    def loss(X=p["X"], projs=p["projs"], xn="bf16"):
        f = o.qkv_forward(X, p["g"], eps, projs, s, rot, p["pos"], p["cos"], p["sin"], p["hd"], xn)
        return float(sum(np.sum(dy * y) for dy, y in zip(p["dYs"], f["Y"])))

    b = o.qkv_backward(p["dYs"], p["X"], p["g"], eps, p["projs"], s, rot, p["pos"], p["cos"], p["sin"], p["hd"],
                       xn="exact")
    num = _fd(lambda x: loss(X=x, xn="exact"), p["X"])
    assert _rel(num, b["dX"]) <= 1e-6, _rel(num, b["dX"])
    bq = o.qkv_backward(p["dYs"], p["X"], p["g"], eps, p["projs"], s, rot, p["pos"], p["cos"], p["sin"], p["hd"])
    for j in range(3):
        for name, key in (("A", "dA"), ("B", "dB")):
            def lj(v, j=j, name=name):
                projs = [dict(pj) for pj in p["projs"]]
                projs[j][name] = v
                return loss(projs=projs)
            num = _fd(lj, p["projs"][j][name])
            assert _rel(num, bq[key][j]) <= 1e-6, (j, name, _rel(num, bq[key][j]))


ALL_CHECKS = [
    check_round_bf16_hand,
    check_round_bf16_matches_bit_rounding,
    check_rms_norm_hand,
    check_rms_norm_closed_forms,
    check_rms_norm_backward_finite_differences,
    check_rotary_complex_brute_force,
    check_rotary_zero_angle_and_quarter_turn,
    check_rotary_relative_position,
    check_rotary_backward_is_adjoint,
    check_qkv_hand_example,
    check_qkv_xn_is_bf16,
    check_qkv_finite_differences,
]
