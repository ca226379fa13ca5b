"""Oracle for the 4-bit frozen base weight ("w4g64"): plain, slow, fp64, CPU.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

Source: the pages name QLoRA fine-tuning, whose frozen base weight is stored
at 4 bits, among the settings the fused LoRA kernels serve ([P1]
"Liger-Kernel内核级优化：GPU利用率飙升至90%以上", opening section; [P2]
"Swift-All一文详解：如何用Liger-Kernel提升训练效率", section 2.3
"性能对比实测数据", whose table lists a QLoRA run), but they define no storage
format for the quantised weight.  The format below is this library's own,
stated in full, and it is the definition the oracle follows:

* W is d_out x d_in, d_in a multiple of 64.
* Codes q[n, k] in 0..15, two per byte, row-major: byte j of row n holds
  q[n, 2j] in its low nibble and q[n, 2j + 1] in its high nibble
  (Wq: uint8 [d_out x d_in/2]).
* One scale per output row and group of 64 consecutive input features,
  stored group-major as bf16 (Ws: [d_in/64 x d_out], Ws[g, n] scales
  W[n, 64 g : 64 g + 64]).
* The weight value is the bf16 rounding (round to nearest, ties to even) of
  scale * (q - 8); the product is exact in fp32 (8-bit scale significand times
  an integer of magnitude <= 8), so the rounding is the only step.
* The layer is then the bf16 LoRA layer on that W: Y = act(X W^T + s (X A^T) B^T).
"""
from __future__ import annotations

import numpy as np

from .lora_oracle import bf16_to_f64, lora_backward, lora_forward

GROUP = 64


def w4_codes(Wq: np.ndarray) -> np.ndarray:
    """The 4-bit codes of a packed weight: int array [d_out x d_in]."""
    b = np.asarray(Wq, dtype=np.uint8)
    q = np.empty((b.shape[0], 2 * b.shape[1]), dtype=np.int64)
    q[:, 0::2] = b & 0x0F           # low nibble: even input feature
    q[:, 1::2] = b >> 4             # high nibble: odd input feature
    return q


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values that are exact in float32 to the nearest bf16
    (ties to even), returned as float64."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)   # exact for the products here
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def w4_dequant(Wq: np.ndarray, Ws_bits: np.ndarray) -> np.ndarray:
    """W[n, k] = bf16(Ws[k // 64, n] * (q[n, k] - 8)), as float64 [d_out x d_in]."""
    q = w4_codes(Wq)
    d_out, d_in = q.shape
    scale = bf16_to_f64(Ws_bits)                              # [d_in/64 x d_out]
    assert scale.shape == (d_in // GROUP, d_out)
    per_elem = np.repeat(scale.T, GROUP, axis=1)              # [d_out x d_in]
    return round_to_bf16(per_elem * (q - 8).astype(np.float64))


def w4_tile(Wq: np.ndarray) -> np.ndarray:
    """The tiled code layout of the few-token kernel: tiles of 128 rows x 64
    features (4096 bytes each, row i of a tile at byte 32 i), ordered by
    128-row slice then by 64-feature block; rows past d_out are zero.
    Returns a flat uint8 array."""
    b = np.asarray(Wq, dtype=np.uint8)
    d_out, half = b.shape
    slices, nkb = (d_out + 127) // 128, half // 32
    padded = np.zeros((slices * 128, half), dtype=np.uint8)
    padded[:d_out] = b
    t = padded.reshape(slices, 128, nkb, 32).transpose(0, 2, 1, 3)   # [slice][kblock][row][32 bytes]
    return np.ascontiguousarray(t).reshape(-1)


def w4_forward(X, Wq, Ws_bits, A, B, s, act="identity", Wq_up=None, Ws_up_bits=None, A_up=None, B_up=None):
    """The LoRA forward with the dequantised base weight(s)."""
    W = w4_dequant(Wq, Ws_bits)
    W_up = w4_dequant(Wq_up, Ws_up_bits) if Wq_up is not None else None
    return lora_forward(X, W, A, B, s, act, W_up, A_up, B_up)


def w4_backward(dY, X, Wq, Ws_bits, A, B, s, act="identity", Wq_up=None, Ws_up_bits=None, A_up=None, B_up=None):
    """The LoRA backward with the dequantised base weight(s) (W frozen)."""
    W = w4_dequant(Wq, Ws_bits)
    W_up = w4_dequant(Wq_up, Ws_up_bits) if Wq_up is not None else None
    return lora_backward(dY, X, W, A, B, s, act, W_up, A_up, B_up)
