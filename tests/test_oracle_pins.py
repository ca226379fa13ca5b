"""The oracles against facts fixed outside themselves (CPU only).

Both statements of the layer are pinned by the same checks: the numpy one
(oracle/lora_oracle.py, matrix products through numpy's matmul) and the plain
C one (oracle/lora_oracle_c.c, scalar fp64 loops)."""
import numpy as np
import pytest

import oracle
from oracle import lora_oracle_c
from tests import oracle_pins

ORACLES = {"numpy": oracle, "c": lora_oracle_c}


@pytest.mark.parametrize("impl", sorted(ORACLES))
@pytest.mark.parametrize("check", oracle_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check, impl):
    check(ORACLES[impl])


@pytest.mark.parametrize("act", ["identity", "silu", "swiglu"])
@pytest.mark.parametrize("M,d_in,d_out,r", [(70, 40, 24, 8), (5, 16, 8, 0), (0, 16, 8, 8), (129, 8, 72, 16)])
def test_c_and_numpy_oracles_agree(M, d_in, d_out, r, act):
    """Two independent statements of the same formulas agree to rounding on
    seeded inputs (every output and intermediate)."""
    rng = np.random.default_rng(M * 1000 + d_in + r)
    p = {"X": rng.standard_normal((M, d_in)), "W": rng.standard_normal((d_out, d_in)) / np.sqrt(d_in),
         "A": rng.uniform(-1, 1, (r, d_in)), "B": rng.standard_normal((d_out, r)),
         "dY": rng.standard_normal((M, d_out))}
    if act == "swiglu":
        p.update(W_up=rng.standard_normal((d_out, d_in)) / np.sqrt(d_in), A_up=rng.uniform(-1, 1, (r, d_in)),
                 B_up=rng.standard_normal((d_out, r)))
    args = (p["dY"], p["X"], p["W"], p["A"], p["B"], 0.75, act, p.get("W_up"), p.get("A_up"), p.get("B_up"))
    a = lora_oracle_c.lora_backward(*args)
    b = oracle.lora_backward(*args)
    for k in b:
        if k == "fwd":
            for kk in b[k]:
                np.testing.assert_allclose(a[k][kk], b[k][kk], rtol=1e-12, atol=1e-12, err_msg=kk)
        else:
            np.testing.assert_allclose(a[k], b[k], rtol=1e-12, atol=1e-12, err_msg=k)


def test_compare_bounds():
    ref = np.array([0.0, 1.0, 100.0])
    assert oracle.compare(ref + np.array([0.009, 0.019, 0.0]), ref)["nfail"] == 0
    assert oracle.compare(ref + np.array([0.011, 0.0, 0.0]), ref)["nfail"] == 1
    assert oracle.compare(ref + np.array([0.0, 0.021, 0.0]), ref)["nfail"] == 1
    assert not oracle.compare(ref * 1.01, ref)["ok"]   # normwise 1e-2 > 5e-3
