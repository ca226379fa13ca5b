"""Oracle for the RMSNorm prologue and rotary-embedding epilogue around the
attention-input (q, k, v) LoRA linears: plain, slow, fp64, CPU.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Sources:
* [P2] "Swift-All一文详解：如何用Liger-Kernel提升训练效率", section 2.2 (1)
  "RMSNorm + Rotary Embedding + Attention QKV 融合": the unfused sequence that
  the fused kernel replaces -- normalise x, project the result to q, k and v,
  then rotate q and k.
* [P4] "企业官网建设流程全解析" (the page's extracted title), section
  "融合内核是如何工作的": its sketch of the fused kernel divides by the square
  root of the mean square plus 1e-6, multiplies by the norm's weight, and
  rotates with cosine and sine tables that it takes as arguments, indexed by
  the feature's offset modulo half a head.

Readings (the pages leave these open; each is the plainest one the rest
supports):
* RMSNorm over the d_in features of a token:
      rstd = 1 / sqrt(mean_j x_j^2 + eps),   x_n = x * rstd * g
  with eps an argument (1e-6 in [P4]).  g, the norm's weight, is frozen like W
  (LoRA trains only A and B), so it gets no gradient.
* x_n is a bf16 tensor: the unfused sequence stores it between the norm and
  the projections, and the pages train in bf16.  It is the exact value
  rounded once to the nearest bf16 (ties to even).
* The rotary embedding acts on q and k, not v, head by head (head_dim
  features each), and pairs feature i of a head with feature i + h,
  h = head_dim / 2 (the half-split pairing that an index modulo h implies).
  With c = cos[pos, i], s = sin[pos, i] from the caller's tables at the
  token's position pos (i < h):
      q'_i     = q_i c - q_{i+h} s
      q'_{i+h} = q_{i+h} c + q_i s
  It rotates the projection's exact result Z, before any output rounding.
* The backward is the chain rule.  The rotation's adjoint turns by the
  opposite angle.  The three projections' input gradients add up into dx_n,
  and the norm's backward is
      dx = rstd * (g dx_n - x_hat * mean_j(g dx_n x_hat)_j),   x_hat = x * rstd
  the derivative of the unrounded norm (a dtype cast passes gradients through
  unchanged).
"""
from __future__ import annotations

import numpy as np

from .lora_oracle import lora_forward, lora_linear_branch_backward


def round_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), returned as
    float64.  Normal range only: v = m 2^e with 1/2 <= |m| < 1, and bf16 keeps
    8 significant bits, so the result is rint(m 2^8) 2^(e - 8); numpy's rint
    rounds halves to even."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def rms_norm(X, g, eps):
    """x_n = x * rstd * g with rstd = 1 / sqrt(mean(x^2) + eps), per token
    (row).  Returns (x_n exact, rstd [M])."""
    ms = np.mean(X * X, axis=1)
    rstd = 1.0 / np.sqrt(ms + eps)
    return (X * rstd[:, None]) * g[None, :], rstd


def rms_norm_backward(dXn, X, g, eps):
    """Gradient with respect to x of <dXn, rms_norm(X, g, eps)>, g frozen."""
    _, rstd = rms_norm(X, g, eps)
    xhat = X * rstd[:, None]
    gd = dXn * g[None, :]
    mean = np.mean(gd * xhat, axis=1)
    return rstd[:, None] * (gd - xhat * mean[:, None])


def _pairs(Z, head_dim):
    M, N = Z.shape
    assert head_dim % 2 == 0 and N % head_dim == 0
    h = head_dim // 2
    Zh = Z.reshape(M, N // head_dim, 2, h)    # [token, head, half, i]
    return Zh[:, :, 0, :], Zh[:, :, 1, :]


def apply_rotary(Z, pos, cos, sin, head_dim):
    """Rotate every head's pairs (i, i + head_dim/2) of each token by the
    table angle at that token's position."""
    a, b = _pairs(Z, head_dim)
    c = cos[pos][:, None, :]
    s = sin[pos][:, None, :]
    out = np.stack([a * c - b * s, b * c + a * s], axis=2)
    return out.reshape(Z.shape)


def apply_rotary_backward(dY, pos, cos, sin, head_dim):
    """The adjoint of apply_rotary: dZ = R^T dY (the opposite angle)."""
    a, b = _pairs(dY, head_dim)
    c = cos[pos][:, None, :]
    s = sin[pos][:, None, :]
    out = np.stack([a * c + b * s, b * c - a * s], axis=2)
    return out.reshape(dY.shape)


def qkv_forward(X, g, eps, projs, s, rotary, pos, cos, sin, head_dim, xn="bf16"):
    """The attention-input block: x_n = bf16(rms_norm(x)); per projection j a
    LoRA linear Z_j = x_n W_j^T + s (x_n A_j^T) B_j^T; Y_j = apply_rotary(Z_j)
    where rotary[j], else Z_j.  projs: list of dicts with W, A, B.
    xn="exact" keeps x_n unrounded (for derivative checks only)."""
    Xn_exact, rstd = rms_norm(X, g, eps)
    Xn = round_bf16(Xn_exact) if xn == "bf16" else Xn_exact
    out = {"Xn": Xn, "rstd": rstd, "T": [], "Z": [], "Y": []}
    for pj, rot in zip(projs, rotary):
        f = lora_forward(Xn, pj["W"], pj["A"], pj["B"], s)
        out["T"].append(f["T"])
        out["Z"].append(f["Z"])
        out["Y"].append(apply_rotary(f["Z"], pos, cos, sin, head_dim) if rot else f["Z"])
    return out


def qkv_backward(dYs, X, g, eps, projs, s, rotary, pos, cos, sin, head_dim, xn="bf16"):
    """Gradients of sum_j <dY_j, Y_j> for qkv_forward: dX, and dA_j, dB_j per
    projection (W_j and g frozen)."""
    fwd = qkv_forward(X, g, eps, projs, s, rotary, pos, cos, sin, head_dim, xn)
    dXn = np.zeros_like(X)
    out = {"fwd": fwd, "dZ": [], "dA": [], "dB": []}
    for j, (pj, rot) in enumerate(zip(projs, rotary)):
        dZ = apply_rotary_backward(dYs[j], pos, cos, sin, head_dim) if rot else dYs[j]
        b = lora_linear_branch_backward(dZ, fwd["Xn"], pj["W"], pj["A"], pj["B"], fwd["T"][j], s)
        out["dZ"].append(dZ)
        out["dA"].append(b["dA"])
        out["dB"].append(b["dB"])
        dXn = dXn + b["dX"]
    out["dXn"] = dXn
    out["dX"] = rms_norm_backward(dXn, X, g, eps)
    return out
