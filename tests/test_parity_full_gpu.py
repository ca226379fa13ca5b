"""Parity at the full workload sizes, through the same library calls bench.py
times.  Rows of Y and dX are independent per token, so the oracle computes a
sample of rows (first, last, a ragged-tile row and seeded random rows); the
adapter gradients dA, dB and the saved T are compared in full where the
oracle can afford them (identity activation: they need no W product)."""
import numpy as np
import pytest

import oracle
import seeded_inputs
from oracle import lora_oracle_c
from tests import gpu_cases as G

pytestmark = pytest.mark.gpu


def sample_rows(M, n=48, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, min(M - 1, 16383), M - 1]
    rows = sorted(set([r for r in fixed if r < M] + list(rng.choice(M, size=min(n, M), replace=False))))
    return np.array(rows)


def _run(name, M=None, backward=True):
    cfg = dict(seeded_inputs.CONFIGS[name])
    if M is not None:
        cfg["M"] = M
    inp = seeded_inputs.make_inputs(cfg["M"], cfg["d_in"], cfg["d_out"], cfg["r"], cfg["act"], seed=0,
                                    with_grad=True)
    s = cfg["alpha"] / cfg["r"]
    out = G.run_library(inp, cfg["M"], cfg["d_in"], cfg["d_out"], cfg["r"], s, cfg["act"], backward=backward)
    return cfg, inp, s, out


@pytest.mark.parametrize("name", ["q_proj", "v_proj", "mlp_down"])
def test_full_size_identity(name):
    cfg, inp, s, out = _run(name)
    g = {k: G.f64(v) for k, v in inp.items()}
    rows = sample_rows(cfg["M"])
    fr = oracle.lora_forward_rows(rows, g["X"], g["W"], g["A"], g["B"], s, "identity")
    br = oracle.lora_backward_rows(rows, g["dY"], g["X"], g["W"], g["A"], g["B"], s, "identity")
    ad = oracle.lora_adapter_grads_identity(g["dY"], g["X"], g["A"], g["B"], s)
    res = {
        "Y": oracle.compare(G.host_f64(out["Y"])[rows], fr["Y"]),
        "dX": oracle.compare(G.host_f64(out["dX"])[rows], br["dX"]),
        "T": oracle.compare(G.host_f64(out["T"][0]), ad["T"]),
        "dA": oracle.compare(G.host_f64(out["dA"]), ad["dA"]),
        "dB": oracle.compare(G.host_f64(out["dB"]), ad["dB"]),
    }
    G.assert_all_ok(res)


def test_full_size_swiglu_gate_up():
    """M = 8192, 4096 -> 2 x 14336, r = 64: the adapter gradients dA, dB,
    dA_up, dB_up are sums over all 8192 tokens and are compared in full, with
    T, T_up, H, Z_gate, Z_up in full and sampled rows of dX.  The oracle is the
    numpy statement (its W products need a BLAS at this size)."""
    cfg, inp, s, out = _run("mlp_gate_up")
    g = {k: G.f64(v) for k, v in inp.items()}
    ref = oracle.lora_backward(g["dY"], g["X"], g["W"], g["A"], g["B"], s, "swiglu", g["W_up"], g["A_up"],
                               g["B_up"])
    f = ref["fwd"]
    rows = sample_rows(cfg["M"], n=64)
    res = {
        "H": oracle.compare(G.host_f64(out["Y"]), f["Y"]),
        "Zg": oracle.compare(G.host_f64(out["Z"][0]), f["Z"]),
        "Zu": oracle.compare(G.host_f64(out["Z"][1]), f["Z_up"]),
        "T": oracle.compare(G.host_f64(out["T"][0]), f["T"]),
        "T_up": oracle.compare(G.host_f64(out["T"][1]), f["T_up"]),
        "dX": oracle.compare(G.host_f64(out["dX"])[rows], ref["dX"][rows]),
        "dA": oracle.compare(G.host_f64(out["dA"]), ref["dA"]),
        "dB": oracle.compare(G.host_f64(out["dB"]), ref["dB"]),
        "dA_up": oracle.compare(G.host_f64(out["dA_up"]), ref["dA_up"]),
        "dB_up": oracle.compare(G.host_f64(out["dB_up"]), ref["dB_up"]),
    }
    G.assert_all_ok(res)


def test_swiglu_gate_up_adapter_grads_1024_tokens():
    """Full feature sizes (4096 -> 2 x 14336, r = 64), 1024 tokens: every output in full."""
    cfg, inp, s, out = _run("mlp_gate_up", M=1024)
    ref = G.run_oracle(inp, s, "swiglu", impl=oracle)
    G.assert_all_ok(G.compare_all(out, ref, "swiglu", cfg["r"]))


@pytest.mark.parametrize("name", ["small_m", "small_m_ragged"])
def test_small_m_forward(name):
    cfg, inp, s, out = _run(name, backward=False)
    g = {k: lora_oracle_c.bf16_to_f64(v) for k, v in inp.items()}
    f = lora_oracle_c.lora_forward(g["X"], g["W"], g["A"], g["B"], s, "identity")
    G.assert_all_ok({"Y": oracle.compare(G.host_f64(out["Y"]), f["Y"]),
                     "T": oracle.compare(G.host_f64(out["T"][0]), f["T"])})
