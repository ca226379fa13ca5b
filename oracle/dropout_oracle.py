"""Oracle for the LoRA layer with dropout on the LoRA branch's input: plain,
slow, fp64, CPU.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Source: the pages' LoRA configurations set a LoRA dropout without saying
where it applies: [P2] "Swift-All一文详解：如何用Liger-Kernel提升训练效率",
section 3, the training configuration just before "3.3 启动训练任务"
(``lora_dropout=0.05``), and [P4] "企业官网建设流程全解析", section
"如何使用真的能做到“零侵入”吗" (``lora_dropout=0.1``).  The reading taken is
the usual one for LoRA: the dropout acts on the input of the adapter branch
only, the frozen path sees the undropped input, and kept elements are scaled
by 1 / (1 - p):

    X_d = X * mask / (1 - p)          (mask in {0, 1}, one bit per element of X)
    T   = X_d A^T
    Z   = X W^T + s T B^T,    Y = act(Z)

The random draws are an input (``mask``), not generated here.  The backward is
the chain rule of that forward (W frozen): with dZ = dY * act'(Z), U = dZ B,

    dX = dZ W + (s U A) * mask / (1 - p)
    dA = s U^T X_d,    dB = s dZ^T T

For SwiGLU, gate and up each carry their own adapter and their own mask.
"""
from __future__ import annotations

import numpy as np

from .lora_oracle import act_backward, silu


def unpack_mask(bits: np.ndarray, d_in: int) -> np.ndarray:
    """The {0, 1} mask [M x d_in] from its packed form [M x d_in/8]: bit j of
    byte b (least significant first) is element 8 b + j."""
    b = np.asarray(bits, dtype=np.uint8)
    m = np.unpackbits(b, axis=1, bitorder="little")
    return m[:, :d_in].astype(np.float64)


def _branch(X, W, A, B, s, mask, p):
    Xd = X * mask / (1.0 - p)
    T = Xd @ A.T
    Z = X @ W.T + s * (T @ B.T)
    return Xd, T, Z


def dropout_forward(X, W, A, B, s, mask, p, act="identity", W_up=None, A_up=None, B_up=None, mask_up=None):
    Xd, T, Z = _branch(X, W, A, B, s, mask, p)
    out = {"Xd": Xd, "T": T, "Z": Z}
    if act == "identity":
        out["Y"] = Z
    elif act == "silu":
        out["Y"] = silu(Z)
    elif act == "swiglu":
        Xd_up, T_up, Z_up = _branch(X, W_up, A_up, B_up, s, mask_up, p)
        out.update(Xd_up=Xd_up, T_up=T_up, Z_up=Z_up, Y=silu(Z) * Z_up)
    else:
        raise ValueError(act)
    return out


def _branch_backward(dZ, W, A, B, T, Xd, s, mask, p):
    U = dZ @ B
    dX = dZ @ W + (s * (U @ A)) * mask / (1.0 - p)
    return {"U": U, "dX": dX, "dA": s * (U.T @ Xd), "dB": s * (dZ.T @ T)}


def dropout_backward(dY, X, W, A, B, s, mask, p, act="identity", W_up=None, A_up=None, B_up=None, mask_up=None):
    fwd = dropout_forward(X, W, A, B, s, mask, p, act, W_up, A_up, B_up, mask_up)
    dZ, dZ_up = act_backward(dY, fwd, act)
    g = _branch_backward(dZ, W, A, B, fwd["T"], fwd["Xd"], s, mask, p)
    out = {"dX": g["dX"], "dA": g["dA"], "dB": g["dB"], "U": g["U"], "fwd": fwd}
    if act == "swiglu":
        gu = _branch_backward(dZ_up, W_up, A_up, B_up, fwd["T_up"], fwd["Xd_up"], s, mask_up, p)
        out["dX"] = g["dX"] + gu["dX"]
        out.update(dA_up=gu["dA"], dB_up=gu["dB"], U_up=gu["U"])
    return out
