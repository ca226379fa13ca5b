"""The LoRA-dropout oracle against its pins, and planted mistakes that each
must fail a pin (CPU only)."""
import importlib.util
import os

import numpy as np
import pytest

from oracle import dropout_oracle
from tests import dropout_pins


@pytest.mark.parametrize("check", dropout_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_dropout_pin(check):
    check(dropout_oracle)


FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "dropout_oracle.py")


def fresh():
    spec = importlib.util.spec_from_file_location("oracle.dropout_mutant", FILE,
                                                  submodule_search_locations=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    spec.loader.exec_module(mod)
    return mod


def m_dropout_on_main_path(o):
    def branch(X, W, A, B, s, mask, p):
        Xd = X * mask / (1.0 - p)
        T = Xd @ A.T
        return Xd, T, Xd @ W.T + s * (T @ B.T)
    o._branch = branch


def m_no_keep_scale(o):
    def branch(X, W, A, B, s, mask, p):
        Xd = X * mask
        T = Xd @ A.T
        return Xd, T, X @ W.T + s * (T @ B.T)
    o._branch = branch


def m_unmasked_dx_term(o):
    def bb(dZ, W, A, B, T, Xd, s, mask, p):
        U = dZ @ B
        return {"U": U, "dX": dZ @ W + s * (U @ A) / (1.0 - p), "dA": s * (U.T @ Xd), "dB": s * (dZ.T @ T)}
    o._branch_backward = bb


def m_mask_whole_dx(o):
    def bb(dZ, W, A, B, T, Xd, s, mask, p):
        U = dZ @ B
        return {"U": U, "dX": (dZ @ W + s * (U @ A)) * mask / (1.0 - p), "dA": s * (U.T @ Xd),
                "dB": s * (dZ.T @ T)}
    o._branch_backward = bb


def m_da_from_undropped_x(o):
    def bb(dZ, W, A, B, T, Xd, s, mask, p):
        U = dZ @ B
        X = np.where(mask > 0, Xd * (1.0 - p), 0.0)
        return {"U": U, "dX": dZ @ W + (s * (U @ A)) * mask / (1.0 - p), "dA": s * (U.T @ (X + (mask == 0))),
                "dB": s * (dZ.T @ T)}
    o._branch_backward = bb


def m_msb_first(o):
    def unpack(bits, d_in):
        return np.unpackbits(np.asarray(bits, dtype=np.uint8), axis=1, bitorder="big")[:, :d_in].astype(np.float64)
    o.unpack_mask = unpack


MUTANTS = [m_dropout_on_main_path, m_no_keep_scale, m_unmasked_dx_term, m_mask_whole_dx, m_da_from_undropped_x,
           m_msb_first]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_dropout_planted_mistake_fails_a_pin(mutant):
    o = fresh()
    mutant(o)
    failed = []
    for chk in dropout_pins.ALL_CHECKS:
        try:
            chk(o)
        except AssertionError:
            failed.append(chk.__name__)
    assert failed, f"{mutant.__name__} passed every pin"
