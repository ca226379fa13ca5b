"""Checks that pin the LoRA-dropout oracle (oracle/dropout_oracle.py) to facts
fixed outside itself.

* With every element kept and p = 0 it is the layer without dropout, whose
  oracle is pinned separately (tests/oracle_pins.py).
* With every element dropped the adapter branch vanishes: Y is the plain
  layer (scalar loops), dA and dB are zero and dX = dZ W.
* The backward is the derivative of the forward: central finite differences
  of L = <dY, Y> with respect to X, A and B at a fixed mask and p, every act.
* A hand-worked example (one token, two features, rank 1).
* The mask's bit order: bit j of byte b (least significant first) is element
  8 b + j, checked element by element.

Each ``check_*`` takes a namespace with ``dropout_forward``,
``dropout_backward``, ``unpack_mask`` (the module, or a copy with a planted
mistake) and raises AssertionError when it disagrees with the fact.
"""
from __future__ import annotations

import numpy as np

import oracle


def _problem(rng, M=3, d_in=16, d_out=4, r=2, act="identity"):
    p = {"X": rng.standard_normal((M, d_in)), "W": rng.standard_normal((d_out, d_in)) * 0.3,
         "A": rng.standard_normal((r, d_in)) * 0.3, "B": rng.standard_normal((d_out, r)) * 0.3,
         "dY": rng.standard_normal((M, d_out))}
    if act == "swiglu":
        p.update(W_up=rng.standard_normal((d_out, d_in)) * 0.3, A_up=rng.standard_normal((r, d_in)) * 0.3,
                 B_up=rng.standard_normal((d_out, r)) * 0.3)
    return p


def _args(p, act):
    return (p.get("W_up"), p.get("A_up"), p.get("B_up")) if act == "swiglu" else (None, None, None)


def check_all_kept_is_plain_lora(o):
    rng = np.random.default_rng(21)
    for act in ("identity", "silu", "swiglu"):
        p = _problem(rng, act=act)
        ones = np.ones_like(p["X"])
        f = o.dropout_forward(p["X"], p["W"], p["A"], p["B"], 1.5, ones, 0.0, act, *_args(p, act), mask_up=ones)
        g = o.dropout_backward(p["dY"], p["X"], p["W"], p["A"], p["B"], 1.5, ones, 0.0, act, *_args(p, act),
                               mask_up=ones)
        ref = oracle.lora_backward(p["dY"], p["X"], p["W"], p["A"], p["B"], 1.5, act, *_args(p, act))
        assert np.allclose(f["Y"], ref["fwd"]["Y"], rtol=1e-13, atol=1e-13), act
        for k in ("dX", "dA", "dB") + (("dA_up", "dB_up") if act == "swiglu" else ()):
            assert np.allclose(g[k], ref[k], rtol=1e-13, atol=1e-13), (act, k)


def check_all_dropped_is_plain_linear(o):
    rng = np.random.default_rng(22)
    p = _problem(rng)
    zeros = np.zeros_like(p["X"])
    f = o.dropout_forward(p["X"], p["W"], p["A"], p["B"], 2.0, zeros, 0.3)
    g = o.dropout_backward(p["dY"], p["X"], p["W"], p["A"], p["B"], 2.0, zeros, 0.3)
    M, d_in = p["X"].shape
    d_out = p["W"].shape[0]
    for m in range(M):
        for n in range(d_out):
            acc = 0.0
            for k in range(d_in):
                acc += p["X"][m, k] * p["W"][n, k]
            assert abs(f["Y"][m, n] - acc) <= 1e-12 * (1 + abs(acc))
        for k in range(d_in):
            acc = 0.0
            for n in range(d_out):
                acc += p["dY"][m, n] * p["W"][n, k]
            assert abs(g["dX"][m, k] - acc) <= 1e-12 * (1 + abs(acc))
    assert not np.any(g["dA"]) and not np.any(g["dB"])


def check_finite_differences(o):
    rng = np.random.default_rng(23)
    h = 1e-6
    for act in ("identity", "silu", "swiglu"):
        p = _problem(rng, M=3, d_in=8, d_out=4, r=2, act=act)
        mask = (rng.random(p["X"].shape) < 0.7).astype(np.float64)
        mask_up = (rng.random(p["X"].shape) < 0.6).astype(np.float64)
        s, pd = 1.25, 0.3

        def loss(X=p["X"], A=p["A"], B=p["B"]):
            f = o.dropout_forward(X, p["W"], A, B, s, mask, pd, act, *_args(p, act), mask_up=mask_up)
            return float(np.sum(p["dY"] * f["Y"]))
        g = o.dropout_backward(p["dY"], p["X"], p["W"], p["A"], p["B"], s, mask, pd, act, *_args(p, act),
                               mask_up=mask_up)
        for name, key in (("X", "dX"), ("A", "dA"), ("B", "dB")):
            base = p[name]
            num = np.zeros_like(base)
            for idx in np.ndindex(base.shape):
                e = np.zeros_like(base)
                e[idx] = h
                num[idx] = (loss(**{name: base + e}) - loss(**{name: base - e})) / (2 * h)
            err = np.max(np.abs(num - g[key])) / max(1e-12, np.max(np.abs(num)))
            assert err <= 1e-6, (act, name, err)


def check_hand_example(o):
    # X = [[2, 3]], mask = [[1, 0]], p = 0.5 -> Xd = [[4, 0]]
    # A = [[1, 1]] -> T = [[4]];  B = [[1], [-1]], s = 0.5 -> s T B^T = [[2, -2]]
    # W = [[1, 0], [0, 1]] -> X W^T = [[2, 3]] -> Z = [[4, 1]]
    # dY = [[1, 1]]: U = dY B = [[0]] -> dA = 0, dX = dY W = [[1, 1]];
    # dB = s dY^T T = 0.5 * [[4], [4]] = [[2], [2]]
    X = np.array([[2.0, 3.0]])
    W = np.eye(2)
    A = np.array([[1.0, 1.0]])
    B = np.array([[1.0], [-1.0]])
    mask = np.array([[1.0, 0.0]])
    f = o.dropout_forward(X, W, A, B, 0.5, mask, 0.5)
    g = o.dropout_backward(np.array([[1.0, 1.0]]), X, W, A, B, 0.5, mask, 0.5)
    assert np.array_equal(f["Y"], np.array([[4.0, 1.0]]))
    assert np.array_equal(g["dX"], np.array([[1.0, 1.0]]))
    assert np.array_equal(g["dA"], np.array([[0.0, 0.0]]))
    assert np.array_equal(g["dB"], np.array([[2.0], [2.0]]))
    # dY = [[1, 0]]: U = [[1]] -> s U A = [[0.5, 0.5]] masked / (1 - p) -> [[1, 0]]; dX = [[1, 0]] + [[1, 0]]
    # dA = s U^T Xd = 0.5 * [[4, 0]] = [[2, 0]]
    g = o.dropout_backward(np.array([[1.0, 0.0]]), X, W, A, B, 0.5, mask, 0.5)
    assert np.array_equal(g["dX"], np.array([[2.0, 0.0]]))
    assert np.array_equal(g["dA"], np.array([[2.0, 0.0]]))


def check_mask_bit_order(o):
    bits = np.array([[0b00000101, 0b10000000], [0xFF, 0x00]], dtype=np.uint8)
    m = o.unpack_mask(bits, 16)
    want = np.zeros((2, 16))
    want[0, 0] = want[0, 2] = want[0, 15] = 1.0
    want[1, :8] = 1.0
    assert np.array_equal(m, want)


ALL_CHECKS = [
    check_all_kept_is_plain_lora,
    check_all_dropped_is_plain_linear,
    check_finite_differences,
    check_hand_example,
    check_mask_bit_order,
]
