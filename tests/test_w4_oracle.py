"""The 4-bit weight oracle against its pins, and planted mistakes that each
pin set must catch (CPU only)."""
import types

import numpy as np
import pytest

import oracle
from oracle import w4_oracle
from tests import w4_pins


@pytest.mark.parametrize("check", w4_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_w4_pin(check):
    check(w4_oracle)


def _namespace(dequant, tile=None):
    ns = types.SimpleNamespace()
    ns.w4_dequant = dequant
    ns.w4_tile = tile or w4_oracle.w4_tile

    def fwd(X, Wq, Ws, A, B, s, act="identity", *rest):
        return oracle.lora_forward(X, dequant(Wq, Ws), A, B, s, act)
    ns.w4_forward = fwd
    return ns


def _codes(Wq, swap=False):
    b = np.asarray(Wq, dtype=np.uint8)
    q = np.empty((b.shape[0], 2 * b.shape[1]), dtype=np.int64)
    lo, hi = b & 0x0F, b >> 4
    q[:, 0::2], q[:, 1::2] = (hi, lo) if swap else (lo, hi)
    return q


def _scale(Ws, d_out, d_in, group=64, row_major=False):
    s = oracle.bf16_to_f64(Ws)
    if row_major:
        s = s.reshape(d_out, d_in // 64).T
    return np.repeat(s.T, group, axis=1)[:, :d_in]


def _trunc_bf16(v):
    u = np.asarray(v, dtype=np.float64).astype(np.float32).view(np.uint32)
    return ((u >> 16) << 16).astype(np.uint32).view(np.float32).astype(np.float64)


def m_swapped_nibbles(Wq, Ws):
    q = _codes(Wq, swap=True)
    return w4_oracle.round_to_bf16(_scale(Ws, *q.shape) * (q - 8))


def m_zero_point_7(Wq, Ws):
    q = _codes(Wq)
    return w4_oracle.round_to_bf16(_scale(Ws, *q.shape) * (q - 7))


def m_scales_row_major(Wq, Ws):
    q = _codes(Wq)
    return w4_oracle.round_to_bf16(_scale(Ws, *q.shape, row_major=True) * (q - 8))


def m_truncate_not_round(Wq, Ws):
    q = _codes(Wq)
    return _trunc_bf16(_scale(Ws, *q.shape) * (q - 8))


def m_no_rounding(Wq, Ws):
    q = _codes(Wq)
    return _scale(Ws, *q.shape) * (q - 8)


def m_group_32(Wq, Ws):
    q = _codes(Wq)
    d_out, d_in = q.shape
    s = oracle.bf16_to_f64(Ws)                       # [d_in/64 x d_out], read as if groups were 32 wide
    per = np.repeat(s.T, 32, axis=1)
    per = np.concatenate([per] * 2, axis=1)[:, :d_in]
    return w4_oracle.round_to_bf16(per * (q - 8))


MUTANTS = [m_swapped_nibbles, m_zero_point_7, m_scales_row_major, m_truncate_not_round, m_no_rounding,
           m_group_32]


def t_kblock_major(Wq):
    """Tiles ordered by 64-feature block first, then by slice."""
    b = np.asarray(Wq, dtype=np.uint8)
    d_out, half = b.shape
    slices, nkb = (d_out + 127) // 128, half // 32
    padded = np.zeros((slices * 128, half), dtype=np.uint8)
    padded[:d_out] = b
    return np.ascontiguousarray(padded.reshape(slices, 128, nkb, 32).transpose(2, 0, 1, 3)).reshape(-1)


def t_rows_not_padded(Wq):
    """The last slice's missing rows left out instead of zero-filled."""
    return w4_oracle.w4_tile(Wq)[: np.asarray(Wq).size]


@pytest.mark.parametrize("tile", [t_kblock_major, t_rows_not_padded], ids=lambda m: m.__name__)
def test_w4_tile_planted_mistake_fails_a_pin(tile):
    ns = _namespace(w4_oracle.w4_dequant, tile)
    with pytest.raises(AssertionError):
        w4_pins.check_w4_tile_brute_force(ns)


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_w4_planted_mistake_fails_a_pin(mutant):
    ns = _namespace(mutant)
    failed = []
    for chk in w4_pins.ALL_CHECKS:
        try:
            chk(ns)
        except AssertionError:
            failed.append(chk.__name__)
    assert failed, f"{mutant.__name__} passed every pin"
