"""The RMSNorm / rotary-embedding oracle against its pins, and planted
mistakes that each must fail a pin (CPU only)."""
import importlib.util
import os

import numpy as np
import pytest

from oracle import norm_rope_oracle
from tests import norm_rope_pins


@pytest.mark.parametrize("check", norm_rope_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_norm_rope_pin(check):
    check(norm_rope_oracle)


FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "norm_rope_oracle.py")


def fresh():
    spec = importlib.util.spec_from_file_location("oracle.norm_rope_mutant", FILE, submodule_search_locations=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    spec.loader.exec_module(mod)
    return mod


def m_sum_not_mean(o):
    def rms_norm(X, g, eps):
        rstd = 1.0 / np.sqrt(np.sum(X * X, axis=1) + eps)
        return (X * rstd[:, None]) * g[None, :], rstd
    o.rms_norm = rms_norm


def m_eps_outside_sqrt(o):
    def rms_norm(X, g, eps):
        rstd = 1.0 / (np.sqrt(np.mean(X * X, axis=1)) + eps)
        return (X * rstd[:, None]) * g[None, :], rstd
    o.rms_norm = rms_norm


def m_norm_backward_no_mean_term(o):
    def bwd(dXn, X, g, eps):
        _, rstd = o.rms_norm(X, g, eps)
        return rstd[:, None] * dXn * g[None, :]
    o.rms_norm_backward = bwd


def m_interleaved_pairs(o):
    def pairs(Z, head_dim):
        M, N = Z.shape
        Zh = Z.reshape(M, N // head_dim, head_dim // 2, 2)
        return Zh[:, :, :, 0], Zh[:, :, :, 1]
    orig_fwd, orig_bwd = o.apply_rotary, o.apply_rotary_backward

    def unpairs(out, shape, head_dim):   # out [M, heads, 2, h] -> interleaved layout
        M, heads, _, h = out.shape
        return np.transpose(out, (0, 1, 3, 2)).reshape(shape)

    def fwd(Z, pos, cos, sin, head_dim):
        a, b = pairs(Z, head_dim)
        c, s = cos[pos][:, None, :], sin[pos][:, None, :]
        return unpairs(np.stack([a * c - b * s, b * c + a * s], axis=2), Z.shape, head_dim)

    def bwd(dY, pos, cos, sin, head_dim):
        a, b = pairs(dY, head_dim)
        c, s = cos[pos][:, None, :], sin[pos][:, None, :]
        return unpairs(np.stack([a * c + b * s, b * c - a * s], axis=2), dY.shape, head_dim)
    o.apply_rotary, o.apply_rotary_backward = fwd, bwd


def m_rotation_sign(o):
    def fwd(Z, pos, cos, sin, head_dim):
        a, b = o._pairs(Z, head_dim)
        c, s = cos[pos][:, None, :], sin[pos][:, None, :]
        return np.stack([a * c + b * s, b * c - a * s], axis=2).reshape(Z.shape)
    o.apply_rotary = fwd


def m_backward_rotates_forward(o):
    o.apply_rotary_backward = o.apply_rotary


def m_rotate_v_too(o):
    orig = o.qkv_forward

    def fwd(X, g, eps, projs, s, rotary, *a, **k):
        return orig(X, g, eps, projs, s, [True] * len(rotary), *a, **k)
    o.qkv_forward = fwd


def m_xn_not_rounded(o):
    o.round_bf16 = lambda v: np.asarray(v, dtype=np.float64)


def m_round_through_f32(o):
    def rnd(v):
        f = np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)
        m, e = np.frexp(f)
        return np.ldexp(np.rint(m * 256.0), e - 8)
    o.round_bf16 = rnd


def m_first_projection_grad_only(o):
    orig = o.rms_norm_backward
    calls = {}

    def qkv_backward(dYs, X, g, eps, projs, s, rotary, pos, cos, sin, head_dim, xn="bf16"):
        fwd = o.qkv_forward(X, g, eps, projs, s, rotary, pos, cos, sin, head_dim, xn)
        out = {"fwd": fwd, "dZ": [], "dA": [], "dB": []}
        dXn = None
        for j, (pj, rot) in enumerate(zip(projs, rotary)):
            dZ = o.apply_rotary_backward(dYs[j], pos, cos, sin, head_dim) if rot else dYs[j]
            b = o.lora_linear_branch_backward(dZ, fwd["Xn"], pj["W"], pj["A"], pj["B"], fwd["T"][j], s)
            out["dA"].append(b["dA"])
            out["dB"].append(b["dB"])
            if dXn is None:
                dXn = b["dX"]
        out["dX"] = orig(dXn, X, g, eps)
        return out
    o.qkv_backward = qkv_backward
    del calls


MUTANTS = [m_sum_not_mean, m_eps_outside_sqrt, m_norm_backward_no_mean_term, m_interleaved_pairs, m_rotation_sign,
           m_backward_rotates_forward, m_rotate_v_too, m_xn_not_rounded, m_round_through_f32,
           m_first_projection_grad_only]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_norm_rope_planted_mistake_fails_a_pin(mutant):
    o = fresh()
    mutant(o)
    failed = []
    for chk in norm_rope_pins.ALL_CHECKS:
        try:
            chk(o)
        except AssertionError:
            failed.append(chk.__name__)
    assert failed, f"{mutant.__name__} passed every pin"
