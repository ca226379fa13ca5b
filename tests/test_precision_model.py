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
