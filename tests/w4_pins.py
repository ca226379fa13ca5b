"""Checks that pin the 4-bit weight oracle (oracle/w4_oracle.py) to facts
fixed outside itself.

The pages give no format for the quantised weight; the library states its own
(codes two per byte, low nibble first; one bf16 scale per row and group of 64
input features, group-major; value = bf16 round-to-nearest-even of
scale * (code - 8)).  The facts used are therefore:
* hand-worked dequantisations of that definition
  (tests/golden/w4_hand_examples.json), a tie and an inexact product included;
* the special case of power-of-two scales, where no rounding happens;
* a brute-force, scalar, pure-Python decoding of the definition on tiny
  inputs (bit fields by shifts, the bf16 rounding by integer arithmetic on the
  float32 bit pattern), independent of the oracle's vectorised numpy code;
* with B = 0 the quantised layer is the plain product with the dequantised
  weight, by scalar loops;
* the tiled code layout of the few-token kernel, element by element with
  loops.

Each ``check_*`` takes the module (or a copy with a planted mistake) and raises
AssertionError when it disagrees with the fact.
"""
from __future__ import annotations

import json
import os
import struct

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "w4_hand_examples.json")


def _bits_value(bits: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0]


def _scalar_rne_bf16(x: float) -> float:
    """bf16 round-to-nearest-even of a value exact in float32, by integer arithmetic."""
    u = struct.unpack("<I", struct.pack("<f", x))[0]
    hi, lo = u >> 16, u & 0xFFFF
    if lo > 0x8000 or (lo == 0x8000 and (hi & 1)):
        hi += 1
    return _bits_value(hi)


def _scalar_dequant(Wq, Ws_bits, d_out, d_in):
    out = [[0.0] * d_in for _ in range(d_out)]
    for n in range(d_out):
        for k in range(d_in):
            byte = int(Wq[n][k // 2])
            code = (byte >> 4) if (k % 2) else (byte & 0xF)
            scale = _bits_value(int(Ws_bits[k // 64][n]))
            out[n][k] = _scalar_rne_bf16(scale * (code - 8))
    return np.array(out, dtype=np.float64)


def check_w4_golden(w4):
    with open(GOLDEN) as f:
        g = json.load(f)
    d_out, d_in = g["d_out"], g["d_in"]
    Wq = np.zeros((d_out, d_in // 2), dtype=np.uint8)
    Ws = np.zeros((d_in // 64, d_out), dtype=np.uint16)
    for n, row in enumerate(g["rows"]):
        Wq[n, :] = int(row["byte"], 16)
        for grp, b in enumerate(row["scale_bits"]):
            Ws[grp, n] = int(b, 16)
    W = w4.w4_dequant(Wq, Ws)
    for n, row in enumerate(g["rows"]):
        e = row["expected"]
        want = [e[0], e[1]] * 32 + [e[2], e[3]] * 32
        assert np.array_equal(W[n], np.array(want)), (n, W[n][:2], W[n][64:66], e)


def check_w4_power_of_two_scales_are_exact(w4):
    rng = np.random.default_rng(11)
    d_out, d_in = 5, 192
    Wq = rng.integers(0, 256, size=(d_out, d_in // 2), dtype=np.uint8)
    exps = rng.integers(-12, 3, size=(d_in // 64, d_out))
    signs = rng.choice([-1.0, 1.0], size=exps.shape)
    scale = signs * np.power(2.0, exps)
    Ws = (scale.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    W = w4.w4_dequant(Wq, Ws)
    q = np.empty((d_out, d_in), dtype=np.int64)
    for n in range(d_out):
        for k in range(d_in):
            b = int(Wq[n, k // 2])
            q[n, k] = (b >> 4) if (k % 2) else (b & 0xF)
    want = np.repeat(scale.T, 64, axis=1) * (q - 8)
    assert np.array_equal(W, want)


def check_w4_brute_force_decoding(w4):
    rng = np.random.default_rng(12)
    d_out, d_in = 3, 128
    Wq = rng.integers(0, 256, size=(d_out, d_in // 2), dtype=np.uint8)
    vals = rng.standard_normal((d_in // 64, d_out)) * 0.37 + 0.05
    Ws = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)   # arbitrary bf16 patterns
    assert np.array_equal(w4.w4_dequant(Wq, Ws), _scalar_dequant(Wq, Ws, d_out, d_in))


def check_w4_zero_adapter_is_plain_product(w4):
    rng = np.random.default_rng(13)
    M, d_out, d_in, r = 2, 3, 64, 2
    Wq = rng.integers(0, 256, size=(d_out, d_in // 2), dtype=np.uint8)
    Ws = np.full((1, d_out), 0x3C80, dtype=np.uint16)           # 2^-6
    X = rng.integers(-3, 4, size=(M, d_in)).astype(np.float64)
    A = rng.standard_normal((r, d_in))
    B = np.zeros((d_out, r))
    Y = w4.w4_forward(X, Wq, Ws, A, B, 2.0)["Y"]
    Wd = _scalar_dequant(Wq, Ws, d_out, d_in)
    for m in range(M):
        for n in range(d_out):
            acc = 0.0
            for k in range(d_in):
                acc += X[m, k] * Wd[n, k]
            assert Y[m, n] == acc, (m, n, Y[m, n], acc)


def check_w4_tile_brute_force(w4):
    """The tiled code layout, element by element with loops: tile (g, kb), row
    i, byte j holds byte kb*32 + j of weight row g*128 + i (zero past d_out)."""
    rng = np.random.default_rng(14)
    d_out, d_in = 130, 128
    Wq = rng.integers(0, 256, size=(d_out, d_in // 2), dtype=np.uint8)
    t = w4.w4_tile(Wq)
    nkb, slices = d_in // 64, (d_out + 127) // 128
    assert t.shape == (slices * nkb * 4096,)
    for g in range(slices):
        for kb in range(nkb):
            for i in range(128):
                for j in range(32):
                    n = g * 128 + i
                    want = int(Wq[n, kb * 32 + j]) if n < d_out else 0
                    assert int(t[((g * nkb + kb) * 128 + i) * 32 + j]) == want, (g, kb, i, j)


ALL_CHECKS = [
    check_w4_golden,
    check_w4_power_of_two_scales_are_exact,
    check_w4_brute_force_decoding,
    check_w4_zero_adapter_is_plain_product,
    check_w4_tile_brute_force,
]
