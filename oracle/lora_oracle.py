"""Oracle for the fused LoRA-adapted linear layer: plain, slow, fp64, CPU.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Sources (web pages; cited by title and section):

* [P1] "Liger-Kernel内核级优化：GPU利用率飙升至90%以上"
  - section "为什么传统微调会“卡脖子”？": the LoRA forward y = Wx + B(Ax) and
    its unfused PyTorch form, four calls: ax = linear(x, A); bax = linear(ax, B);
    wx = linear(x, W); y = wx + bax.
  - section "内核融合：把“碎片化”变成“流水线”": the fused variant computes
    Wx + B(Ax) and applies SiLU as the last step (activation after the add).
  - section "系统架构与工作流程": the backward is fused too, with recompute.
* [P2] "Swift-All一文详解：如何用Liger-Kernel提升训练效率", section 2.2 (2)
  "SwiGLU 激活函数融合": Linear -> SwiGLU -> Linear fused.
* [P3] "Liger-Kernel加持！LlamaPro微调性能大幅提升的秘密": the merged form
  W + ΔW with ΔW the product of the two low-rank factors.
* [P4] "企业官网建设流程全解析" (a Liger inference article inside it), section
  "它适用于哪些模型": gate_proj / up_proj / down_proj with SwiGLU gating.

Readings where the pages are silent or inconsistent (each is restated where
it is used):

* Shapes: A is r x d_in and is applied first (x -> A x), B is d_out x r.  [P1]
  prints A in R^{d x r} yet writes Ax; [P3] swaps the roles.  The reading that
  makes ``linear(x, A)`` then ``linear(ax, B)`` typecheck is the one used.
* Scale: the LoRA branch is multiplied by s = alpha / r (the pages give alpha
  and r in their configs but no formula with the scale).
* No bias, no dropout (the four-call sequence has neither).
* SwiGLU: Y = SiLU(Z_gate) * Z_up, each of Z_gate / Z_up a LoRA linear with its
  own W, A, B (standard gate/up pairing; the pages give no formula).
* Backward: the chain rule of the forward above (the pages print no backward
  formula).  With dZ = dY * act'(Z) and U = dZ B:
  dX = dZ W + s U A,  dA = s U^T X,  dB = s dZ^T T  where T = X A^T.
* sigma(z) = 1 / (1 + exp(-z)),  SiLU(z) = z sigma(z).

All arithmetic is float64 on the exact values of the bf16 inputs.  Outputs are
not rounded.  Matrix products use numpy's matmul as a library primitive;
nothing is blocked, fused or reordered beyond the formulas above.
"""
from __future__ import annotations

import numpy as np

ACTS = ("identity", "silu", "swiglu")


# ---------------------------------------------------------------------------
# input decoding
# ---------------------------------------------------------------------------
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u32.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# activations  ([P1] "内核融合…": SiLU after the add; [P2] 2.2 (2), [P4]
# "它适用于哪些模型": SwiGLU gating of gate/up projections)
# ---------------------------------------------------------------------------
def sigmoid(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigma(z)."""
    return z * sigmoid(z)


def silu_grad(z: np.ndarray) -> np.ndarray:
    """d SiLU / dz = sigma(z) * (1 + z * (1 - sigma(z)))."""
    sg = sigmoid(z)
    return sg * (1.0 + z * (1.0 - sg))


# ---------------------------------------------------------------------------
# forward
# ---------------------------------------------------------------------------
def lora_linear_branch(X, W, A, B, s):
    """One LoRA linear without activation: the unfused sequence of [P1]
    section "为什么传统微调会“卡脖子”？" with the branch scaled by s.

    Returns (T, Z):  T = linear(X, A) = X A^T   (the rank-r intermediate "ax")
                     Z = linear(X, W) + s * linear(T, B) = X W^T + s T B^T
    """
    ax = X @ A.T            # ax  = F.linear(x, A)
    bax = ax @ B.T          # bax = F.linear(ax, B)
    wx = X @ W.T            # wx  = F.linear(x, W)
    Z = wx + s * bax        # y   = wx + bax   (scaled LoRA branch)
    return ax, Z


def lora_forward(X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
    """Forward of the LoRA-adapted linear, float64.

    act = identity : Y = Z
    act = silu     : Y = SiLU(Z)                    ([P1] "内核融合…")
    act = swiglu   : Y = SiLU(Z_gate) * Z_up         ([P2] 2.2 (2); [P4])
    Returns a dict with T, Z, Y (and T_up, Z_up for swiglu).
    """
    T, Z = lora_linear_branch(X, W, A, B, s)
    out = {"T": T, "Z": Z}
    if act == "identity":
        out["Y"] = Z
    elif act == "silu":
        out["Y"] = silu(Z)
    elif act == "swiglu":
        T_up, Z_up = lora_linear_branch(X, W_up, A_up, B_up, s)
        out["T_up"] = T_up
        out["Z_up"] = Z_up
        out["Y"] = silu(Z) * Z_up
    else:
        raise ValueError(act)
    return out


# ---------------------------------------------------------------------------
# backward (chain rule of the forward; [P1] "系统架构与工作流程" says only that
# the backward is fused with recompute — the formulas are derived, not printed)
# ---------------------------------------------------------------------------
def act_backward(dY, fwd, act):
    """dZ = dY * act'(Z).  For swiglu returns (dZ_gate, dZ_up)."""
    if act == "identity":
        return dY, None
    if act == "silu":
        return dY * silu_grad(fwd["Z"]), None
    if act == "swiglu":
        zg, zu = fwd["Z"], fwd["Z_up"]
        return dY * zu * silu_grad(zg), dY * silu(zg)
    raise ValueError(act)


def lora_linear_branch_backward(dZ, X, W, A, B, T, s):
    """Gradients of Z = X W^T + s (X A^T) B^T with W frozen.

    U  = dZ B                 (M x r)
    dX = dZ W + s U A         (M x d_in)
    dA = s U^T X              (r x d_in)
    dB = s dZ^T T             (d_out x r)
    """
    U = dZ @ B
    dX = dZ @ W + s * (U @ A)
    dA = s * (U.T @ X)
    dB = s * (dZ.T @ T)
    return {"U": U, "dX": dX, "dA": dA, "dB": dB}


def lora_backward(dY, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
    """Backward of ``lora_forward`` (recomputes the forward, float64).

    Returns dX, dA, dB (and dA_up, dB_up for swiglu) plus dZ / U intermediates.
    """
    fwd = lora_forward(X, W, A, B, s, act, W_up, A_up, B_up)
    dZ, dZ_up = act_backward(dY, fwd, act)
    g = lora_linear_branch_backward(dZ, X, W, A, B, fwd["T"], s)
    out = {"dZ": dZ, "U": g["U"], "dX": g["dX"], "dA": g["dA"], "dB": g["dB"], "fwd": fwd}
    if act == "swiglu":
        gu = lora_linear_branch_backward(dZ_up, X, W_up, A_up, B_up, fwd["T_up"], s)
        out["dZ_up"] = dZ_up
        out["U_up"] = gu["U"]
        out["dX"] = g["dX"] + gu["dX"]
        out["dA_up"] = gu["dA"]
        out["dB_up"] = gu["dB"]
    return out


# ---------------------------------------------------------------------------
# row-sampled evaluation for large shapes: rows of Y and dX depend only on the
# same rows of X and dY, so they can be computed one row set at a time.
# ---------------------------------------------------------------------------
def lora_forward_rows(rows, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
    """``lora_forward`` restricted to the given token rows."""
    return lora_forward(X[rows], W, A, B, s, act, W_up, A_up, B_up)


def lora_backward_rows(rows, dY, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
    """dX (and dZ, U) for the given token rows only."""
    return lora_backward(dY[rows], X[rows], W, A, B, s, act, W_up, A_up, B_up)


def lora_adapter_grads_identity(dY, X, A, B, s):
    """dA, dB for act = identity without touching W (cheap at any size):
    T = X A^T, U = dY B, dA = s U^T X, dB = s dY^T T."""
    T = X @ A.T
    U = dY @ B
    return {"T": T, "U": U, "dA": s * (U.T @ X), "dB": s * (dY.T @ T)}


# ---------------------------------------------------------------------------
# comparison against the stated tolerance
# ---------------------------------------------------------------------------
ATOL = 1e-2
RTOL = 1e-2
NORM_TOL = 5e-3


def compare(got, ref, atol=ATOL, rtol=RTOL, norm_tol=NORM_TOL):
    """Per element |got-ref| <= atol + rtol*|ref| and ||got-ref||/||ref|| <= norm_tol.

    Returns a dict with ok, worst excess, normwise error and the count of
    failing elements.
    """
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if got.shape != ref.shape:
        raise ValueError(f"shape mismatch {got.shape} vs {ref.shape}")
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    nfail = int(np.count_nonzero(~(err <= bound)))
    rn = float(np.linalg.norm(ref))
    norm_err = float(np.linalg.norm(got - ref) / rn) if rn > 0 else float(np.linalg.norm(got - ref))
    worst = float(np.max(err / bound)) if err.size else 0.0
    return {"ok": nfail == 0 and norm_err <= norm_tol, "nfail": nfail,
            "worst_ratio": worst, "norm_err": norm_err, "max_abs_err": float(err.max()) if err.size else 0.0}
