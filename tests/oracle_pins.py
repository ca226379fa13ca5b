"""Checks that pin the oracle to facts fixed outside itself.

Each ``check_*`` takes an oracle-like namespace (the real ``oracle`` module or
a copy with a planted mistake) and raises AssertionError when the oracle
disagrees with the fact.  ``test_oracle_pins.py`` runs them on the real oracle
and ``test_oracle_mutations.py`` shows that each planted mistake fails one.

Facts used:
* hand-derived worked examples (tests/golden/lora_hand_examples.json), from
  the forward y = Wx + B(Ax) of "Liger-Kernel内核级优化：GPU利用率飙升至90%以上",
  section "为什么传统微调会“卡脖子”？";
* the merged-weight identity W + ΔW ("Liger-Kernel加持！LlamaPro微调性能大幅提升的秘密");
* closed forms of sigma / SiLU / SiLU' and the SwiGLU special case up = 1;
* central finite differences of L = <dY, Y> (the backward must be the
  derivative of the forward);
* special cases: B = 0 or r = 0 gives the plain linear layer, computed by
  brute-force scalar loops; dA = 0 when B = 0; dB = 0 when A = 0.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "lora_hand_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _arr(x):
    return np.array(x, dtype=np.float64)


def _rand_problem(rng, M=3, d_in=5, d_out=4, r=2, act="identity"):
    p = {
        "X": rng.standard_normal((M, d_in)),
        "W": rng.standard_normal((d_out, d_in)) / math.sqrt(d_in),
        "A": rng.uniform(-1, 1, (r, d_in)),
        "B": rng.standard_normal((d_out, r)),
        "dY": rng.standard_normal((M, d_out)),
    }
    if act == "swiglu":
        p["W_up"] = rng.standard_normal((d_out, d_in)) / math.sqrt(d_in)
        p["A_up"] = rng.uniform(-1, 1, (r, d_in))
        p["B_up"] = rng.standard_normal((d_out, r))
    return p


def _fwd(o, p, s, act):
    return o.lora_forward(p["X"], p["W"], p["A"], p["B"], s, act,
                          p.get("W_up"), p.get("A_up"), p.get("B_up"))


def _bwd(o, p, s, act):
    return o.lora_backward(p["dY"], p["X"], p["W"], p["A"], p["B"], s, act,
                           p.get("W_up"), p.get("A_up"), p.get("B_up"))


# ---------------------------------------------------------------------------
def check_bf16_decoding(o):
    """bf16 bit patterns decode to the IEEE values they stand for: a bf16
    number is the upper half of a binary32 (sign, 8 exponent bits, 7 fraction
    bits).  Expected values are written from that definition, bit by bit."""
    cases = [
        (0x3F80, 1.0),                          # exponent 127, fraction 0
        (0xC040, -3.0),                         # sign, exponent 128, fraction 1000000b
        (0x4049, 3.140625),                     # exponent 128, fraction 1001001b: 2 (1 + 73/128)
        (0x3E80, 0.25),
        (0xBF81, -(1.0 + 2.0 ** -7)),           # the smallest step above 1, negated
        (0x7F7F, (2.0 - 2.0 ** -7) * 2.0 ** 127),   # the largest finite bf16
        (0x0080, 2.0 ** -126),                  # the smallest normal
        (0x0001, 2.0 ** -133),                  # the smallest subnormal: 2^-126 * 2^-7
        (0x007F, 127 * 2.0 ** -133),            # the largest subnormal
        (0x8000, -0.0),
        (0x0000, 0.0),
        (0x7F80, math.inf),
        (0xFF80, -math.inf),
    ]
    bits = np.array([[b for b, _ in cases]], dtype=np.uint16)
    got = np.asarray(o.bf16_to_f64(bits))
    assert got.shape == bits.shape and got.dtype == np.float64, (got.shape, got.dtype)
    for (b, want), v in zip(cases, got[0]):
        assert v == want, f"bf16 0x{b:04X}: got {v!r}, want {want!r}"
        assert math.copysign(1.0, v) == math.copysign(1.0, want), f"bf16 0x{b:04X}: sign of {v!r}"
    nan = np.asarray(o.bf16_to_f64(np.array([0x7FC0], dtype=np.uint16)))
    assert np.isnan(nan[0]), nan


def check_golden_examples(o):
    for ex in _golden()["examples"]:
        X, W, A, B, dY = (_arr(ex[k]) for k in ("X", "W", "A", "B", "dY"))
        s = ex["s"]
        f = o.lora_forward(X, W, A, B, s, "identity")
        np.testing.assert_allclose(f["T"], _arr(ex["T"]), rtol=0, atol=1e-12, err_msg=ex["name"] + " T")
        np.testing.assert_allclose(f["Z"], _arr(ex["Z"]), rtol=0, atol=1e-12, err_msg=ex["name"] + " Z")
        np.testing.assert_allclose(f["Y"], _arr(ex["Z"]), rtol=0, atol=1e-12, err_msg=ex["name"] + " Y")
        g = o.lora_backward(dY, X, W, A, B, s, "identity")
        for k in ("U", "dX", "dA", "dB"):
            np.testing.assert_allclose(g[k], _arr(ex[k]), rtol=0, atol=1e-12, err_msg=ex["name"] + " " + k)


def check_activation_closed_forms(o):
    ln3 = math.log(3.0)
    z = np.array([0.0, ln3, -ln3])
    np.testing.assert_allclose(o.sigmoid(z), [0.5, 0.75, 0.25], rtol=1e-15, atol=0)
    np.testing.assert_allclose(o.silu(z), [0.0, 0.75 * ln3, -0.25 * ln3], rtol=1e-15, atol=1e-300)
    np.testing.assert_allclose(o.silu_grad(z), [0.5, 0.75 * (1 + ln3 / 4), 0.25 * (1 - 0.75 * ln3)],
                               rtol=1e-14, atol=0)
    # SiLU(-z) = SiLU(z) - z   and   SiLU(z)/z -> 1 for large z
    w = np.linspace(-6, 6, 25)
    np.testing.assert_allclose(o.silu(-w), o.silu(w) - w, rtol=0, atol=1e-14)
    assert abs(float(o.silu(np.array([40.0]))[0]) / 40.0 - 1.0) < 1e-15
    # SiLU' is the derivative of SiLU (central difference)
    h = 1e-6
    np.testing.assert_allclose(o.silu_grad(w), (o.silu(w + h) - o.silu(w - h)) / (2 * h), rtol=1e-8, atol=1e-9)


def check_swiglu_with_unit_up_is_silu(o):
    """SwiGLU(g, u) with the up projection identically 1 reduces to SiLU(g).

    Z_up = X W_up^T + s (X A_up^T) B_up^T is made 1 by a constant input column:
    X's last column is 1 and W_up selects it; the up branch's LoRA is zero."""
    rng = np.random.default_rng(3)
    M, d_in, d_out, r, s = 4, 6, 5, 2, 1.5
    p = _rand_problem(rng, M, d_in, d_out, r, "swiglu")
    p["X"][:, -1] = 1.0
    p["W_up"] = np.zeros((d_out, d_in))
    p["W_up"][:, -1] = 1.0
    p["B_up"] = np.zeros((d_out, r))
    f = _fwd(o, p, s, "swiglu")
    g = _fwd(o, p, s, "silu")
    np.testing.assert_allclose(f["Y"], g["Y"], rtol=1e-14, atol=1e-14)


def _brute_linear(X, W):
    M, d_in = X.shape
    d_out = W.shape[0]
    Y = np.zeros((M, d_out))
    for m in range(M):
        for n in range(d_out):
            acc = 0.0
            for k in range(d_in):
                acc += X[m, k] * W[n, k]
            Y[m, n] = acc
    return Y


def check_zero_adapter_is_plain_linear(o):
    rng = np.random.default_rng(5)
    p = _rand_problem(rng, M=3, d_in=7, d_out=5, r=3)
    p["B"] = np.zeros_like(p["B"])
    ref = _brute_linear(p["X"], p["W"])
    f = _fwd(o, p, 2.0, "identity")
    np.testing.assert_allclose(f["Y"], ref, rtol=1e-13, atol=1e-13)
    # r = 0: empty adapters
    q = dict(p, A=np.zeros((0, 7)), B=np.zeros((5, 0)))
    f0 = _fwd(o, q, 2.0, "identity")
    np.testing.assert_allclose(f0["Y"], ref, rtol=1e-13, atol=1e-13)
    # silu of the plain layer, elementwise by the closed form
    fs = _fwd(o, p, 2.0, "silu")
    np.testing.assert_allclose(fs["Y"], ref / (1.0 + np.exp(-ref)), rtol=1e-13, atol=1e-14)


def check_brute_force_unfused_sequence(o):
    """Scalar loops of the four-call sequence on a tiny problem, every act."""
    rng = np.random.default_rng(11)
    M, d_in, d_out, r, s = 2, 4, 3, 2, 0.75
    for act in ("identity", "silu", "swiglu"):
        p = _rand_problem(rng, M, d_in, d_out, r, act)

        def branch(W, A, B):
            ax = _brute_linear(p["X"], A)          # linear(x, A)
            bax = _brute_linear(ax, B)             # linear(ax, B)
            wx = _brute_linear(p["X"], W)          # linear(x, W)
            return wx + s * bax
        zg = branch(p["W"], p["A"], p["B"])
        if act == "identity":
            ref = zg
        elif act == "silu":
            ref = zg / (1.0 + np.exp(-zg))
        else:
            zu = branch(p["W_up"], p["A_up"], p["B_up"])
            ref = zg / (1.0 + np.exp(-zg)) * zu
        np.testing.assert_allclose(_fwd(o, p, s, act)["Y"], ref, rtol=1e-13, atol=1e-13, err_msg=act)


def check_merged_weight_identity(o):
    """Y = act(X (W + s B A)^T): the LoRA branch is the same as a merged weight."""
    rng = np.random.default_rng(7)
    for act in ("identity", "silu", "swiglu"):
        p = _rand_problem(rng, M=6, d_in=9, d_out=7, r=3, act=act)
        s = 0.25
        Wm = p["W"] + s * (p["B"] @ p["A"])
        Zg = p["X"] @ Wm.T
        if act == "identity":
            ref = Zg
        elif act == "silu":
            ref = Zg / (1 + np.exp(-Zg))
        else:
            Wum = p["W_up"] + s * (p["B_up"] @ p["A_up"])
            ref = Zg / (1 + np.exp(-Zg)) * (p["X"] @ Wum.T)
        got = _fwd(o, p, s, act)["Y"]
        assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref))), act


def check_finite_difference_gradients(o):
    """Central differences of L = <dY, Y(X, A, B)> against dX, dA, dB."""
    h = 1e-6
    for act in ("identity", "silu", "swiglu"):
        rng = np.random.default_rng({"identity": 1, "silu": 2, "swiglu": 3}[act])
        p = _rand_problem(rng, M=3, d_in=5, d_out=4, r=2, act=act)
        s = 1.25
        g = _bwd(o, p, s, act)

        def loss(q):
            return float(np.sum(q["dY"] * _fwd(o, q, s, act)["Y"]))
        names = [("X", "dX"), ("A", "dA"), ("B", "dB")]
        if act == "swiglu":
            names += [("A_up", "dA_up"), ("B_up", "dB_up")]
        for name, gname in names:
            num = np.zeros_like(p[name])
            for idx in np.ndindex(p[name].shape):
                qp = {k: v.copy() for k, v in p.items()}
                qm = {k: v.copy() for k, v in p.items()}
                qp[name][idx] += h
                qm[name][idx] -= h
                num[idx] = (loss(qp) - loss(qm)) / (2 * h)
            ana = g[gname]
            rel = np.linalg.norm(ana - num) / max(np.linalg.norm(num), 1e-30)
            assert rel <= 1e-6, f"{act} {gname}: rel err {rel:.3e}"


def check_special_case_zero_grads(o):
    rng = np.random.default_rng(13)
    for act in ("identity", "silu", "swiglu"):
        p = _rand_problem(rng, M=4, d_in=6, d_out=5, r=2, act=act)
        q = dict(p, B=np.zeros_like(p["B"]))
        g = _bwd(o, q, 2.0, act)
        assert np.all(g["dA"] == 0.0), act          # U = dZ B = 0
        q2 = dict(p, A=np.zeros_like(p["A"]))
        g2 = _bwd(o, q2, 2.0, act)
        assert np.all(g2["dB"] == 0.0), act         # T = X A^T = 0


def check_dx_main_term_is_transpose_product(o):
    """With B = 0, dX = dY W: checked against a naive loop over W's rows."""
    rng = np.random.default_rng(17)
    p = _rand_problem(rng, M=3, d_in=6, d_out=4, r=2)
    p["B"] = np.zeros_like(p["B"])
    g = _bwd(o, p, 2.0, "identity")
    ref = np.zeros((3, 6))
    for m in range(3):
        for k in range(6):
            ref[m, k] = sum(p["dY"][m, n] * p["W"][n, k] for n in range(4))
    np.testing.assert_allclose(g["dX"], ref, rtol=1e-13, atol=1e-13)


def check_row_sampling_matches_full(o):
    rng = np.random.default_rng(19)
    for act in ("identity", "silu", "swiglu"):
        p = _rand_problem(rng, M=9, d_in=6, d_out=5, r=2, act=act)
        rows = np.array([0, 4, 8])
        full_f = _fwd(o, p, 0.5, act)
        part_f = o.lora_forward_rows(rows, p["X"], p["W"], p["A"], p["B"], 0.5, act,
                                     p.get("W_up"), p.get("A_up"), p.get("B_up"))
        np.testing.assert_allclose(part_f["Y"], full_f["Y"][rows], rtol=1e-14, atol=1e-14)
        full_b = _bwd(o, p, 0.5, act)
        part_b = o.lora_backward_rows(rows, p["dY"], p["X"], p["W"], p["A"], p["B"], 0.5, act,
                                      p.get("W_up"), p.get("A_up"), p.get("B_up"))
        np.testing.assert_allclose(part_b["dX"], full_b["dX"][rows], rtol=1e-14, atol=1e-14)
    p = _rand_problem(rng, M=9, d_in=6, d_out=5, r=2)
    gi = o.lora_adapter_grads_identity(p["dY"], p["X"], p["A"], p["B"], 0.5)
    gb = _bwd(o, p, 0.5, "identity")
    np.testing.assert_allclose(gi["dA"], gb["dA"], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(gi["dB"], gb["dB"], rtol=1e-13, atol=1e-13)


ALL_CHECKS = [
    check_bf16_decoding,
    check_golden_examples,
    check_activation_closed_forms,
    check_swiglu_with_unit_up_is_silu,
    check_zero_adapter_is_plain_linear,
    check_brute_force_unfused_sequence,
    check_merged_weight_identity,
    check_finite_difference_gradients,
    check_special_case_zero_grads,
    check_dx_main_term_is_transpose_product,
    check_row_sampling_matches_full,
]


def run_all(o):
    """Run every pin; return the list of (name, error) for those that fail."""
    failures = []
    for chk in ALL_CHECKS:
        try:
            chk(o)
        except AssertionError as e:
            failures.append((chk.__name__, str(e)[:200]))
        except (ValueError, IndexError) as e:  # a planted shape error
            failures.append((chk.__name__, repr(e)[:200]))
    return failures
