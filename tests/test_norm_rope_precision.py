"""The precision choices of the RMSNorm / rotary block checked on the CPU
against the exact oracle (oracle/norm_rope_oracle.py):

* x_n: the kernel's method, the fp64 value rounded to bf16 through fp32 with
  rounding to odd (Boldo and Melquiond, "Emulation of FMA and correctly
  rounded sums: proved algorithms using rounding to odd", IEEE Trans.
  Computers 57(4), 2008), restated here in numpy, gives the correctly
  rounded bf16 of every double tried, near-ties included; an all-fp32
  evaluation of the norm would not take the oracle's rounding decisions.
* The rotation: on the fp32 accumulator it leaves Y within the bound, while
  rotating the stored bf16 Y (two roundings) does not.
"""
import numpy as np

import oracle
import seeded_inputs
from oracle import norm_rope_oracle as NR
from tests import precision_model as PM


def _round_to_odd_bf16(x):
    """bf16 of doubles by the kernel's method: truncate to fp32, set the last
    fp32 bit when that dropped anything, round to nearest even."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)                        # nearest; step back to truncation where it rounded away
    away = np.abs(f.astype(np.float64)) > np.abs(x)
    fb = f.view(np.uint32).copy()
    fb[away] -= 1
    f = fb.view(np.float32)
    inexact = f.astype(np.float64) != x
    fb = f.view(np.uint32) | inexact.astype(np.uint32)
    u = fb.astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def test_round_to_odd_gives_the_correct_bf16():
    rng = np.random.default_rng(71)
    x = rng.standard_normal(200000) * np.exp2(rng.integers(-30, 30, 200000))
    # near-ties: a bf16 midpoint, nudged by a few fp64 units either way
    mids = (NR.round_bf16(x[:2000]) + np.ldexp(1.0, np.frexp(x[:2000])[1] - 9) * np.sign(x[:2000]))
    near = np.concatenate([mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf),
                           mids + np.ldexp(1.0, np.frexp(mids)[1] - 40), mids - np.ldexp(1.0, np.frexp(mids)[1] - 40)])
    for v in (x, near):
        assert np.array_equal(_round_to_odd_bf16(v), NR.round_bf16(v))
    # a plain rounding through fp32 gets some of the near-ties wrong
    via_f32 = PM.to_bf16(near)
    assert not np.array_equal(via_f32, NR.round_bf16(near))


def test_fp32_norm_would_not_match_the_exact_rounding():
    M, d = 512, 4096
    X = oracle.bf16_to_f64(seeded_inputs.draw("X", (M, d), 72, d))
    g = oracle.bf16_to_f64(seeded_inputs.draw_norm_weight(d, 72))
    eps = float(np.float32(1e-6))
    exact = NR.round_bf16(NR.rms_norm(X, g, eps)[0])
    x32, g32 = X.astype(np.float32), g.astype(np.float32)
    rstd32 = np.float32(1.0) / np.sqrt(np.mean(x32 * x32, axis=1, dtype=np.float32) + np.float32(eps))
    f32 = PM.to_bf16(((x32 * rstd32[:, None]) * g32[None, :]).astype(np.float64))
    assert np.count_nonzero(f32 != exact) > 0


def test_rotation_on_the_accumulator_not_on_bf16_y():
    M, d_in, d_out, r, hd, n_pos = 2048, 256, 256, 8, 128, 512
    inp = seeded_inputs.make_inputs(M, d_in, d_out, r, "identity", seed=73)
    gg = {k: oracle.bf16_to_f64(v) for k, v in inp.items()}
    X = gg["X"] * 4.0                               # |Z| up to about 20: pairs where rounding matters
    pos = seeded_inputs.draw_positions(M, n_pos, 73)
    cos, sin = (t.astype(np.float64) for t in seeded_inputs.rotary_tables(n_pos, hd))
    s = 2.0
    Z = PM.forward(X, gg["W"], gg["A"], gg["B"], s)["Z"]   # the fp32 accumulator
    ref = NR.apply_rotary(oracle.lora_forward(X, gg["W"], gg["A"], gg["B"], s)["Z"], pos, cos, sin, hd)
    once = oracle.compare(PM.to_bf16(NR.apply_rotary(Z, pos, cos, sin, hd)), ref)
    twice = oracle.compare(PM.to_bf16(NR.apply_rotary(PM.to_bf16(Z), pos, cos, sin, hd)), ref)
    assert once["ok"], once
    assert not twice["ok"], twice
