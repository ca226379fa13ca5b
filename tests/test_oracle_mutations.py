"""Plant plausible mistakes in a private copy of the oracle (on the CPU) and
check that at least one pin fails for each: the pins are strong enough to
catch a dropped term, a wrong sign, a swapped operand or a misplaced scale."""
import importlib.util
import os

import numpy as np
import pytest

from tests import oracle_pins

ORACLE_FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                           "oracle", "lora_oracle.py")


def fresh_oracle():
    spec = importlib.util.spec_from_file_location("oracle_mutant", ORACLE_FILE)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def m_drop_scale(o):
    def branch(X, W, A, B, s):
        ax = X @ A.T
        return ax, X @ W.T + ax @ B.T
    o.lora_linear_branch = branch


def m_double_scale(o):
    def branch(X, W, A, B, s):
        ax = X @ A.T
        return ax, X @ W.T + s * s * (ax @ B.T)
    o.lora_linear_branch = branch


def m_scaled_T(o):
    def branch(X, W, A, B, s):
        ax = s * (X @ A.T)
        return ax, X @ W.T + ax @ B.T
    o.lora_linear_branch = branch


def m_act_before_add(o):
    orig = o.lora_forward

    def fwd(X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
        out = orig(X, W, A, B, s, act, W_up, A_up, B_up)
        if act == "silu":
            T = X @ A.T
            out["Y"] = o.silu(X @ W.T) + s * (T @ B.T)
        return out
    o.lora_forward = fwd


def m_sigmoid_sign(o):
    o.sigmoid = lambda z: 1.0 / (1.0 + np.exp(z))


def m_silu_grad_sign(o):
    def g(z):
        sg = o.sigmoid(z)
        return sg * (1.0 - z * (1.0 - sg))
    o.silu_grad = g


def m_swiglu_swapped(o):
    orig = o.lora_forward

    def fwd(X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
        out = orig(X, W, A, B, s, act, W_up, A_up, B_up)
        if act == "swiglu":
            out["Y"] = o.silu(out["Z_up"]) * out["Z"]
        return out
    o.lora_forward = fwd


def m_swiglu_up_grad(o):
    orig = o.act_backward

    def ab(dY, fwd, act):
        a, b = orig(dY, fwd, act)
        if act == "swiglu":
            b = dY * fwd["Z"]
        return a, b
    o.act_backward = ab


def m_dx_missing_lora(o):
    def bb(dZ, X, W, A, B, T, s):
        U = dZ @ B
        return {"U": U, "dX": dZ @ W, "dA": s * (U.T @ X), "dB": s * (dZ.T @ T)}
    o.lora_linear_branch_backward = bb


def m_dA_no_scale(o):
    def bb(dZ, X, W, A, B, T, s):
        U = dZ @ B
        return {"U": U, "dX": dZ @ W + s * (U @ A), "dA": U.T @ X, "dB": s * (dZ.T @ T)}
    o.lora_linear_branch_backward = bb


def m_dB_wrong_operand(o):
    def bb(dZ, X, W, A, B, T, s):
        U = dZ @ B
        return {"U": U, "dX": dZ @ W + s * (U @ A), "dA": s * (U.T @ X), "dB": s * (dZ.T @ U)}
    o.lora_linear_branch_backward = bb


def m_dx_sign(o):
    def bb(dZ, X, W, A, B, T, s):
        U = dZ @ B
        return {"U": U, "dX": dZ @ W - s * (U @ A), "dA": s * (U.T @ X), "dB": s * (dZ.T @ T)}
    o.lora_linear_branch_backward = bb


def m_U_transposed_B(o):
    def bb(dZ, X, W, A, B, T, s):
        U = dZ @ B[::-1]            # rows of B taken in the wrong order
        return {"U": U, "dX": dZ @ W + s * (U @ A), "dA": s * (U.T @ X), "dB": s * (dZ.T @ T)}
    o.lora_linear_branch_backward = bb


def m_identity_uses_silu_grad(o):
    orig = o.act_backward

    def ab(dY, fwd, act):
        if act == "identity":
            return dY * o.silu_grad(fwd["Z"]), None
        return orig(dY, fwd, act)
    o.act_backward = ab


def m_bf16_shift15(o):
    o.bf16_to_f64 = lambda bits: (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 15).view(
        np.float32).astype(np.float64)


def m_bf16_as_fp16(o):
    o.bf16_to_f64 = lambda bits: np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def m_bf16_drops_sign(o):
    orig = o.bf16_to_f64
    o.bf16_to_f64 = lambda bits: np.abs(orig(bits))


def m_bf16_flushes_subnormals(o):
    orig = o.bf16_to_f64

    def dec(bits):
        v = orig(bits)
        return np.where(np.abs(v) < 2.0 ** -126, 0.0 * v, v)
    o.bf16_to_f64 = dec


MUTATIONS = [m_bf16_shift15, m_bf16_as_fp16, m_bf16_drops_sign, m_bf16_flushes_subnormals, m_drop_scale, m_double_scale, m_scaled_T, m_act_before_add, m_sigmoid_sign,
             m_silu_grad_sign, m_swiglu_swapped, m_swiglu_up_grad, m_dx_missing_lora,
             m_dA_no_scale, m_dB_wrong_operand, m_dx_sign, m_U_transposed_B,
             m_identity_uses_silu_grad]


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda m: m.__name__)
def test_planted_mistake_is_caught(mutate):
    o = fresh_oracle()
    assert oracle_pins.run_all(o) == []          # the unmodified copy passes
    mutate(o)
    failures = oracle_pins.run_all(o)
    assert failures, f"no pin caught {mutate.__name__}"
