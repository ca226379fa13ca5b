"""Checks that pin the output-projection cross-entropy oracle
(oracle/linear_ce_oracle.py) to facts fixed outside itself.

* A hand-worked example (tests/golden/linear_ce_hand_examples.json): two valid
  tokens and one ignored.
* Closed forms: with W = 0 every token's loss is ln V and dH = 0; with two
  classes a token's loss is softplus(z_other - z_label) (numpy's logaddexp).
* SciPy's log_softmax gives every valid token's loss.
* Adding the same vector to every row of W shifts all of a token's logits by
  one amount: the loss and dH do not change.
* Logits of order 1e4 give a finite loss equal to that of the same problem
  shifted down by a constant per token.
* Scalar loops with math.exp / math.log on tiny inputs.
* Ignored tokens: the same loss and dH as with those rows removed (dH zero
  on them); with no valid token, loss 0 and dH 0.
* dH against central finite differences of the loss.

Each ``check_*`` takes the module (or a copy with a planted mistake) and raises
AssertionError when it disagrees with the fact.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "linear_ce_hand_examples.json")


def _problem(rng, M=6, d=5, V=7, ignore=(2,)):
    H = rng.standard_normal((M, d))
    W = rng.standard_normal((V, d)) * 0.7
    labels = rng.integers(0, V, size=M)
    for i in ignore:
        labels[i] = -100
    return H, W, labels


def check_hand_example(o):
    g = json.load(open(GOLDEN))
    ln2 = math.log(2.0)
    H = np.array([[ln2], [ln2], [float(g["h2"])]])
    W = np.array(g["W"], dtype=np.float64)
    b = o.linear_ce_backward(H, W, np.array(g["labels"]))
    assert abs(b["fwd"]["loss"] - g["loss_over_ln2"] * ln2) <= 1e-15, b["fwd"]["loss"]
    assert np.allclose(b["dlogits"], np.array(g["dlogits"]), rtol=0, atol=1e-15), b["dlogits"]
    assert np.allclose(b["dH"], np.array(g["dH"]), rtol=0, atol=1e-15), b["dH"]


def check_zero_weight_is_log_v(o):
    rng = np.random.default_rng(61)
    H, W, labels = _problem(rng)
    W = np.zeros_like(W)
    b = o.linear_ce_backward(H, W, labels)
    assert abs(b["fwd"]["loss"] - math.log(W.shape[0])) <= 1e-14
    assert not np.any(b["dH"])


def check_two_classes_softplus(o):
    rng = np.random.default_rng(62)
    H, W, labels = _problem(rng, V=2, ignore=())
    f = o.linear_ce_forward(H, W, labels)
    Z = H @ W.T
    m = np.arange(len(labels))
    want = np.logaddexp(0.0, Z[m, 1 - labels] - Z[m, labels])
    assert np.allclose(f["loss_tok"], want, rtol=1e-14, atol=1e-15)


def check_scipy_log_softmax(o):
    from scipy.special import log_softmax
    rng = np.random.default_rng(63)
    H, W, labels = _problem(rng, M=9, V=11, ignore=(0, 4))
    f = o.linear_ce_forward(H, W, labels)
    ls = log_softmax(H @ W.T, axis=1)
    valid = labels >= 0
    want = -ls[np.arange(9)[valid], labels[valid]]
    assert np.allclose(f["loss_tok"][valid], want, rtol=1e-13, atol=1e-14)
    assert abs(f["loss"] - np.mean(want)) <= 1e-13


def check_shift_invariance(o):
    rng = np.random.default_rng(64)
    H, W, labels = _problem(rng)
    u = rng.standard_normal(W.shape[1]) * 3.0
    a = o.linear_ce_backward(H, W, labels)
    b = o.linear_ce_backward(H, W + u[None, :], labels)
    assert abs(a["fwd"]["loss"] - b["fwd"]["loss"]) <= 1e-12
    assert np.allclose(a["dH"], b["dH"], rtol=1e-10, atol=1e-12)


def check_large_logits_stay_finite(o):
    rng = np.random.default_rng(65)
    H, W, labels = _problem(rng, ignore=())
    big = o.linear_ce_forward(H * 4000.0, W, labels)
    assert np.isfinite(big["loss"]) and np.all(np.isfinite(big["lse"]))
    # the same logits shifted down per token by their own maximum: no overflow either way
    Z = (H * 4000.0) @ W.T
    mx = Z.max(axis=1)
    ref = [math.log(sum(math.exp(v - mx[m]) for v in Z[m])) - (Z[m, labels[m]] - mx[m]) for m in range(len(labels))]
    assert np.allclose(big["loss_tok"], ref, rtol=1e-12, atol=1e-9)
    bb = o.linear_ce_backward(H * 4000.0, W, labels)
    assert np.all(np.isfinite(bb["dH"]))


def check_brute_force_loops(o):
    rng = np.random.default_rng(66)
    M, d, V = 3, 4, 5
    H = rng.standard_normal((M, d))
    W = rng.standard_normal((V, d)) * 0.5
    labels = np.array([4, -1, 0])
    tot, n = 0.0, 0
    for m in range(M):
        if labels[m] < 0:
            continue
        z = [sum(H[m, k] * W[j, k] for k in range(d)) for j in range(V)]
        tot += math.log(sum(math.exp(v) for v in z)) - z[labels[m]]
        n += 1
    f = o.linear_ce_forward(H, W, labels)
    assert abs(f["loss"] - tot / n) <= 1e-13, (f["loss"], tot / n)


def check_ignored_tokens(o):
    rng = np.random.default_rng(67)
    H, W, labels = _problem(rng, M=8, ignore=(1, 5, 6))
    keep = labels >= 0
    a = o.linear_ce_backward(H, W, labels)
    b = o.linear_ce_backward(H[keep], W, labels[keep])
    assert abs(a["fwd"]["loss"] - b["fwd"]["loss"]) <= 1e-14
    assert np.allclose(a["dH"][keep], b["dH"], rtol=1e-13, atol=1e-15)
    assert not np.any(a["dH"][~keep])
    none = o.linear_ce_backward(H, W, np.full(8, -100))
    assert none["fwd"]["loss"] == 0.0 and not np.any(none["dH"])


def check_finite_differences(o):
    rng = np.random.default_rng(68)
    H, W, labels = _problem(rng, M=4, d=3, V=6, ignore=(1,))
    h = 1e-6
    num = np.zeros_like(H)
    for idx in np.ndindex(H.shape):
        e = np.zeros_like(H)
        e[idx] = h
        num[idx] = (o.linear_ce_forward(H + e, W, labels)["loss"] - o.linear_ce_forward(H - e, W, labels)["loss"]) / (2 * h)
    got = o.linear_ce_backward(H, W, labels)["dH"]
    assert np.max(np.abs(num - got)) <= 1e-8 * max(1.0, np.max(np.abs(num))), np.max(np.abs(num - got))


ALL_CHECKS = [
    check_hand_example,
    check_zero_weight_is_log_v,
    check_two_classes_softplus,
    check_scipy_log_softmax,
    check_shift_invariance,
    check_large_logits_stay_finite,
    check_brute_force_loops,
    check_ignored_tokens,
    check_finite_differences,
]
