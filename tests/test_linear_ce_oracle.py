"""The output-projection cross-entropy oracle against its pins, and planted
mistakes that each must fail a pin (CPU only)."""
import importlib.util
import os

import numpy as np
import pytest

from oracle import linear_ce_oracle
from tests import linear_ce_pins


@pytest.mark.parametrize("check", linear_ce_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_linear_ce_pin(check):
    check(linear_ce_oracle)


FILE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "linear_ce_oracle.py")


def fresh():
    spec = importlib.util.spec_from_file_location("oracle.linear_ce_mutant", FILE, submodule_search_locations=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"
    spec.loader.exec_module(mod)
    return mod


def m_no_max_shift(o):
    o.logsumexp_rows = lambda Z: np.log(np.sum(np.exp(Z), axis=1))


def m_sum_not_mean(o):
    orig = o.linear_ce_forward

    def fwd(H, W, labels):
        f = orig(H, W, labels)
        f["loss"] = float(np.sum(f["loss_tok"]))
        return f
    o.linear_ce_forward = fwd


def m_mean_over_all_tokens(o):
    orig = o.linear_ce_forward

    def fwd(H, W, labels):
        f = orig(H, W, labels)
        f["loss"] = float(np.sum(f["loss_tok"]) / len(labels))
        return f
    o.linear_ce_forward = fwd


def m_gradient_sign(o):
    orig = o.linear_ce_backward

    def bwd(H, W, labels, dloss=1.0):
        b = orig(H, W, labels, dloss)
        return {"dlogits": -b["dlogits"], "dH": -b["dH"], "fwd": b["fwd"]}
    o.linear_ce_backward = bwd


def m_no_onehot(o):
    def bwd(H, W, labels, dloss=1.0):
        f = o.linear_ce_forward(H, W, labels)
        P = np.exp(f["logits"] - f["lse"][:, None])
        dZ = P * (dloss / max(f["n_valid"], 1))
        dZ[~f["valid"]] = 0.0
        return {"dlogits": dZ, "dH": dZ @ W, "fwd": f}
    o.linear_ce_backward = bwd


def m_ignored_rows_in_gradient(o):
    def bwd(H, W, labels, dloss=1.0):
        f = o.linear_ce_forward(H, W, labels)
        M, V = f["logits"].shape
        P = np.exp(f["logits"] - f["lse"][:, None])
        onehot = np.zeros((M, V))
        rows = np.nonzero(f["valid"])[0]
        onehot[rows, np.asarray(labels)[rows]] = 1.0
        dZ = (P - onehot) * (dloss / max(f["n_valid"], 1))
        return {"dlogits": dZ, "dH": dZ @ W, "fwd": f}
    o.linear_ce_backward = bwd


def m_labels_not_checked(o):
    def fwd(H, W, labels):
        labels = np.asarray(labels)
        Z = H @ W.T
        lse = o.logsumexp_rows(Z)
        loss_tok = lse - Z[np.arange(len(labels)), labels]
        valid = np.ones(len(labels), dtype=bool)
        return {"logits": Z, "lse": lse, "loss_tok": loss_tok, "loss": float(np.mean(loss_tok)), "valid": valid,
                "n_valid": len(labels)}
    o.linear_ce_forward = fwd


MUTANTS = [m_no_max_shift, m_sum_not_mean, m_mean_over_all_tokens, m_gradient_sign, m_no_onehot,
           m_ignored_rows_in_gradient, m_labels_not_checked]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_linear_ce_planted_mistake_fails_a_pin(mutant):
    o = fresh()
    mutant(o)
    failed = []
    with np.errstate(over="ignore", invalid="ignore"):
        for chk in linear_ce_pins.ALL_CHECKS:
            try:
                chk(o)
            except (AssertionError, IndexError, ValueError):   # a pin that cannot even run the mutant rejects it
                failed.append(chk.__name__)
    assert failed, f"{mutant.__name__} passed every pin"
