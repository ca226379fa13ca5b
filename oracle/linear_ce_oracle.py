"""Oracle for the output projection fused with the cross-entropy loss: plain,
slow, fp64, CPU.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Source: [P2] "Swift-All一文详解：如何用Liger-Kernel提升训练效率", section 2.2 (3)
"CrossEntropy Loss 与最后一层 Logits 计算融合": the loss is computed together
with the last layer's logits, in a numerically stable form, and its gradient
is taken straight from the previous layer's output without materialising the
full probability distribution.  That describes how a kernel evaluates the
quantity; the quantity itself is the usual one, written out here in full:

    z_m     = h_m W^T                              logits of token m (V classes)
    l_m     = logsumexp(z_m) - z_m[y_m]            its cross-entropy
    loss    = (1 / N) sum over valid m of l_m      N = the number of valid tokens
    dz_m    = (softmax(z_m) - onehot(y_m)) / N     (zero for ignored tokens)
    dh_m    = dz_m W

Readings (the pages leave these open):
* Reduction: the mean over the tokens whose label is valid (the usual
  language-model loss).  A label below 0 marks a token to ignore (padding);
  with no valid token the loss and every gradient are 0.
* W (the output projection, V x d) is frozen like the adapted layers' base
  weights, so only dh is returned.  No bias.
* logsumexp is evaluated with the row maximum subtracted first (the stable
  form the page asks for); in exact arithmetic this is the definition.
"""
from __future__ import annotations

import numpy as np


def logsumexp_rows(Z):
    """log(sum_j exp(Z[m, j])) per row, with the row maximum taken out first."""
    mx = np.max(Z, axis=1)
    return mx + np.log(np.sum(np.exp(Z - mx[:, None]), axis=1))


def linear_ce_forward(H, W, labels):
    """Returns {"logits", "lse", "loss_tok", "loss", "valid", "n_valid"}.
    H [M x d], W [V x d], labels int [M] (below 0: ignored)."""
    labels = np.asarray(labels)
    Z = H @ W.T
    lse = logsumexp_rows(Z)
    valid = labels >= 0
    picked = np.where(valid, Z[np.arange(len(labels)), np.where(valid, labels, 0)], 0.0)
    loss_tok = np.where(valid, lse - picked, 0.0)
    n_valid = int(np.count_nonzero(valid))
    loss = float(np.sum(loss_tok) / n_valid) if n_valid else 0.0
    return {"logits": Z, "lse": lse, "loss_tok": loss_tok, "loss": loss, "valid": valid, "n_valid": n_valid}


def linear_ce_backward(H, W, labels, dloss=1.0):
    """Gradient of dloss * loss with respect to H (W frozen): {"dlogits", "dH", "fwd"}."""
    f = linear_ce_forward(H, W, labels)
    M, V = f["logits"].shape
    if f["n_valid"] == 0:
        return {"dlogits": np.zeros((M, V)), "dH": np.zeros_like(H), "fwd": f}
    P = np.exp(f["logits"] - f["lse"][:, None])
    onehot = np.zeros((M, V))
    rows = np.nonzero(f["valid"])[0]
    onehot[rows, np.asarray(labels)[rows]] = 1.0
    dZ = (P - onehot) * (dloss / f["n_valid"])
    dZ[~f["valid"]] = 0.0
    return {"dlogits": dZ, "dH": dZ @ W, "fwd": f}
