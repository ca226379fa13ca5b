"""A CPU model of the GPU path's roundings (test infrastructure).

The layer's kernels round at fixed points: bf16 inputs, fp32 accumulators,
the adapter's rank-r operands split into a 16-bit high part and a 16-bit
remainder before they meet the tensor cores, fp16 operands for the backward
with an activation, bf16 outputs.  This module applies those roundings to
fp64 arithmetic (products exact, then each stored intermediate rounded to the
type the kernels store it in) so that the error they leave can be compared
with the stated tolerance on the CPU, and so that a cheaper choice (one bf16
rounding of U) can be shown to break it.  It models types, not summation
order: fp32 accumulation is represented by rounding the exact fp64 sum to
fp32 once.

It shares no code with the CUDA library and is not an oracle: the oracle
(oracle/lora_oracle.py) is the exact reference the model is compared with.
"""
from __future__ import annotations

import numpy as np

import oracle


def to_f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def to_bf16(x):
    """Round to bf16 (nearest even) through fp32."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def to_f16(x):
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def hi_lo(x, rnd):
    """The 16-bit high part and the rounded remainder of x (as the kernels store them)."""
    hi = rnd(x)
    return hi, rnd(x - hi)


def forward(X, W, A, B, s, act="identity"):
    """T (fp32), Z (fp32), Y (bf16) as the forward kernels produce them."""
    T = to_f32(X @ A.T)                           # rank pass, fp32 accumulator
    sT = to_bf16(s * T)                           # the adapter K-block's operand
    Z = to_f32(X @ W.T + sT @ B.T)                # one fp32 accumulator for both products
    Y = to_bf16(Z if act == "identity" else oracle.silu(Z))
    return {"T": T, "Z": Z, "Y": Y}


def backward(dY, X, W, A, B, s, act="identity", fwd=None, single_u_rounding=False, dz_type="f16"):
    """dX (bf16), dA, dB (fp32) as the backward kernels produce them.

    single_u_rounding=True replaces the hi/lo split of s*U by one bf16
    rounding, and dz_type="bf16" stores dZ (with an activation) as bf16
    instead of fp16: the cheaper designs that the kernels' choices avoid."""
    fwd = fwd or forward(X, W, A, B, s, act)
    if act == "identity":
        dZ_parts = [dY]                            # bf16 already
        Wop = W
    else:
        dZ = to_f32(dY * oracle.silu_grad(fwd["Z"]))
        rnd16 = to_f16 if dz_type == "f16" else to_bf16
        dZ_parts = list(hi_lo(dZ, rnd16))          # fp16 (or bf16) hi + lo
        Wop = to_f16(W) if dz_type == "f16" else W  # exact fp16 copy of the bf16 weight
    Bop = B if act == "identity" else to_f16(B)
    U = to_f32(sum(p @ Bop for p in dZ_parts))      # rank pass over dZ (both parts)
    sU16 = to_bf16(s * U)                          # dX's adapter K-block operand
    dX = to_bf16(dZ_parts[0] @ Wop + sU16 @ A)     # main term from the high part only
    if single_u_rounding:
        sU_parts = [to_bf16(s * U)]
    else:
        sU_parts = list(hi_lo(s * U, to_bf16))
    dA = to_f32(sum(p.T @ X for p in sU_parts))
    rnd = to_bf16 if act == "identity" else to_f16
    sT_hi, sT_lo = hi_lo(s * fwd["T"], rnd)
    if act == "identity":
        dB = to_f32(dZ_parts[0].T @ (sT_hi + sT_lo))
    else:                                           # hi x hi + hi x lo + lo x hi
        dB = to_f32(dZ_parts[0].T @ (sT_hi + sT_lo) + dZ_parts[1].T @ sT_hi)
    return {"dX": dX, "dA": dA, "dB": dB}
