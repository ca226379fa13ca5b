"""The precision design checked on the CPU: the GPU path's roundings
(tests/precision_model.py) leave every output within the stated tolerance of
the exact oracle, and the cheaper single bf16 rounding of U, which the hi/lo
split replaces, does not (its adapter gradient dA misses the per-element
bound on entries near zero)."""
import pytest

import oracle
import seeded_inputs
from tests import precision_model as PM

M, D_IN, D_OUT, R, S = 1024, 512, 256, 16, 2.0


def _inputs(act, seed):
    inp = seeded_inputs.make_inputs(M, D_IN, D_OUT, R, act, seed=seed)
    return {k: oracle.bf16_to_f64(v) for k, v in inp.items()}


@pytest.mark.parametrize("act", ["identity", "silu"])
def test_planned_roundings_meet_the_tolerance(act):
    g = _inputs(act, 31)
    ref = oracle.lora_backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, act)
    fwd = PM.forward(g["X"], g["W"], g["A"], g["B"], S, act)
    bwd = PM.backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, act, fwd=fwd)
    checks = {"Y": (fwd["Y"], ref["fwd"]["Y"]), "T": (fwd["T"], ref["fwd"]["T"]),
              "dX": (bwd["dX"], ref["dX"]), "dA": (bwd["dA"], ref["dA"]), "dB": (bwd["dB"], ref["dB"])}
    for name, (got, want) in checks.items():
        res = oracle.compare(got, want)
        assert res["ok"], (act, name, res)


def test_single_bf16_rounding_of_U_breaks_dA():
    g = _inputs("identity", 32)
    ref = oracle.lora_backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, "identity")
    good = PM.backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, "identity")
    bad = PM.backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, "identity", single_u_rounding=True)
    assert oracle.compare(good["dA"], ref["dA"])["ok"]
    res = oracle.compare(bad["dA"], ref["dA"])
    assert res["nfail"] > 0, res


def test_bf16_dZ_breaks_dX_over_a_long_reduction():
    """With an activation, dX = dZ W sums over d_out.  Over a long sum (here
    d_out = 28672, the SwiGLU pair's K) one bf16 rounding of dZ leaves
    per-element errors past the bound; the fp16 dZ the kernels use does not."""
    Ml, d_in, d_out, r = 128, 256, 28672, 16
    inp = seeded_inputs.make_inputs(Ml, d_in, d_out, r, "silu", seed=33)
    g = {k: oracle.bf16_to_f64(v) for k, v in inp.items()}
    ref = oracle.lora_backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, "silu")
    fwd = PM.forward(g["X"], g["W"], g["A"], g["B"], S, "silu")
    good = PM.backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, "silu", fwd=fwd)
    bad = PM.backward(g["dY"], g["X"], g["W"], g["A"], g["B"], S, "silu", fwd=fwd, dz_type="bf16")
    assert oracle.compare(good["dX"], ref["dX"])["ok"]
    res = oracle.compare(bad["dX"], ref["dX"])
    assert res["nfail"] > 0, res


def test_block_input_gradient_needs_fp32_sum():
    """The attention-input block: the norm's backward reads the sum of the q,
    k and v input gradients.  Stored as three bf16 tensors and then summed,
    they put entries of dx past the per-element bound (the norm's backward
    scales their roundings by rstd g); summed in fp32 (as the dX GEMMs do, one
    writing and two adding), dx stays well inside it."""
    import numpy as np
    from oracle import norm_rope_oracle as NR
    M, d, douts, r, hd, n_pos = 130, 256, (256, 256, 256), 16, 128, 512
    X = oracle.bf16_to_f64(seeded_inputs.draw("X", (M, d), 23, d))
    g = oracle.bf16_to_f64(seeded_inputs.draw_norm_weight(d, 23))
    proj = [seeded_inputs.make_inputs(M, d, n, r, "identity", seed=230 + j) for j, n in enumerate(douts)]
    projs = [{k: oracle.bf16_to_f64(p[k]) for k in ("W", "A", "B")} for p in proj]
    dYs = [oracle.bf16_to_f64(p["dY"]) for p in proj]
    pos = seeded_inputs.draw_positions(M, n_pos, 23)
    cos, sin = (t.astype(np.float64) for t in seeded_inputs.rotary_tables(n_pos, hd))
    s, eps = 16.0 / r, float(np.float32(1e-6))
    ref = NR.qkv_backward(dYs, X, g, eps, projs, s, [True, True, False], pos, cos, sin, hd)
    parts = [ref["dZ"][j] @ projs[j]["W"] + s * ((ref["dZ"][j] @ projs[j]["B"]) @ projs[j]["A"]) for j in range(3)]
    as_bf16 = oracle.compare(PM.to_bf16(NR.rms_norm_backward(sum(PM.to_bf16(q) for q in parts), X, g, eps)),
                             ref["dX"])
    as_fp32 = oracle.compare(PM.to_bf16(NR.rms_norm_backward(PM.to_f32(sum(PM.to_f32(q) for q in parts)), X, g, eps)),
                             ref["dX"])
    assert not as_bf16["ok"] and as_bf16["worst_ratio"] > 1.0, as_bf16
    assert as_fp32["ok"] and as_fp32["worst_ratio"] < 0.5, as_fp32
