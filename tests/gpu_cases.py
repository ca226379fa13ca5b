"""Shared helpers of the GPU parity tests: seeded inputs on the device, one
call of the library, and the oracle on the same bf16 bits.

The layer's oracle here is the plain C statement (oracle/lora_oracle_c.c,
scalar fp64 loops).  Full-size tests whose M-long sums need a whole-batch W
product use the numpy statement (oracle/lora_oracle.py, matmul as the
library primitive), which the same pins hold to the same facts."""
from __future__ import annotations

import numpy as np

import oracle
import seeded_inputs
from oracle import lora_oracle_c


def dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_f64(t):
    """torch tensor (bf16 or fp32, any device) -> float64 numpy."""
    import torch
    return t.detach().to("cpu", torch.float64).numpy()


def f64(bits):
    return oracle.bf16_to_f64(bits)


def run_library(inp, M, d_in, d_out, r, s, act, backward=True, recompute_T=False):
    import lora_linear_fine_b200 as L
    import torch
    t = {k: dev(v) for k, v in inp.items()}
    sw = act == "swiglu"
    Y, T, Z = L.forward(t["X"], t["W"], t.get("A") if r else None, t.get("B") if r else None, s, act,
                        t.get("W_up"), t.get("A_up") if r else None, t.get("B_up") if r else None)
    out = {"Y": Y, "T": T, "Z": Z}
    if backward:
        dX, dA, dB, dA_up, dB_up = L.backward(
            t["dY"], t["X"], t["W"], t.get("A") if r else None, t.get("B") if r else None, s, act,
            t.get("W_up"), t.get("A_up") if r else None, t.get("B_up") if r else None,
            T_save=None if recompute_T else T, Z_save=Z)
        out.update(dX=dX, dA=dA, dB=dB, dA_up=dA_up, dB_up=dB_up)
    torch.cuda.synchronize()
    return out


def run_oracle(inp, s, act, impl=None):
    """The layer's forward and backward on the inputs' bf16 values (the plain
    C oracle unless ``impl`` names another pinned statement)."""
    o = impl or lora_oracle_c
    g = {k: o.bf16_to_f64(v) for k, v in inp.items()}
    b = o.lora_backward(g["dY"], g["X"], g["W"], g["A"], g["B"], s, act,
                             g.get("W_up"), g.get("A_up"), g.get("B_up"))
    return b


def compare_all(out, ref, act, r, backward=True):
    """Compare every output tensor; returns {name: compare-result}."""
    f = ref["fwd"]
    res = {"Y": oracle.compare(host_f64(out["Y"]), f["Y"])}
    if r > 0 and out["T"] is not None:
        res["T"] = oracle.compare(host_f64(out["T"][0]), f["T"])
        if act == "swiglu":
            res["T_up"] = oracle.compare(host_f64(out["T"][1]), f["T_up"])
    if act != "identity" and out["Z"] is not None:
        res["Z"] = oracle.compare(host_f64(out["Z"][0]), f["Z"])
        if act == "swiglu":
            res["Z_up"] = oracle.compare(host_f64(out["Z"][1]), f["Z_up"])
    if backward:
        res["dX"] = oracle.compare(host_f64(out["dX"]), ref["dX"])
        if r > 0:
            res["dA"] = oracle.compare(host_f64(out["dA"]), ref["dA"])
            res["dB"] = oracle.compare(host_f64(out["dB"]), ref["dB"])
            if act == "swiglu":
                res["dA_up"] = oracle.compare(host_f64(out["dA_up"]), ref["dA_up"])
                res["dB_up"] = oracle.compare(host_f64(out["dB_up"]), ref["dB_up"])
    return res


def assert_all_ok(res):
    bad = {k: v for k, v in res.items() if not v["ok"]}
    assert not bad, "parity failures: " + "; ".join(
        f"{k}: nfail={v['nfail']} worst={v['worst_ratio']:.3g} norm={v['norm_err']:.3g}" for k, v in bad.items())
