"""Seeded synthetic inputs for the fused LoRA-adapted linear layer.

This module is shared by the oracle (``oracle/``), the tests and ``bench.py``.
It draws random tensors and encodes them as bfloat16 bit patterns; it holds
none of the layer's arithmetic (no products, no activation, no gradient).

Workloads (sizes are the Llama-3-8B projection shapes; no weights or datasets
are used, every tensor is drawn here):

* X  ~ N(0, 1)            tokens x d_in
* W  ~ N(0, 1/d_in)       d_out x d_in   (frozen base weight)
* A  ~ U(-1/sqrt(d_in), +1/sqrt(d_in))   r x d_in      (maps d_in -> r)
* B  ~ N(0, 0.02^2)       d_out x r                    (maps r -> d_out)
* dY ~ N(0, 1)            tokens x d_out (upstream gradient)
* 4-bit base weight (the library's "w4g64" format): codes uniform in 0..15,
  packed two per byte (Wq: uint8 d_out x d_in/2, drawn as uniform bytes), and
  one scale per row and group of 64 input features (Ws: bf16 d_in/64 x d_out)
  ~ U(0.5, 1.5) / (4.6 sqrt(d_in)), so that the weight has roughly the spread
  of W above (the codes minus 8 have a standard deviation of about 4.6).
* dropout masks on the adapter input: each element of X kept with probability
  1 - p, packed eight per byte (bit j of byte b, least significant first, is
  element 8 b + j): uint8 tokens x d_in/8.
* output projection + cross-entropy: hidden states H ~ N(0, 1) (tokens x d),
  the frozen output projection W_out ~ N(0, 1/d) (V x d), so that the logits
  H W_out^T are about N(0, 1); labels int32 uniform in [0, V), a given
  fraction of them (5 % by default) replaced by -100 (tokens to ignore, as
  padding would be).
* attention-input block (RMSNorm, then the q, k, v projections, q and k
  rotated): the norm's weight g ~ U(0.5, 1.5) (bf16, d_in); each projection j
  has its own W, A, B, dY drawn as above from the seed (seed, j); token
  positions int32, uniform in [0, n_pos) for the tests, or m mod seq_len (a
  batch of whole sequences) for the benchmark; rotary tables float32
  [n_pos x head_dim/2] holding the cosine and sine of p * 10000^(-2i/head_dim),
  the RoFormer frequencies, as a model precomputes them.

Each tensor has its own stream: numpy's PCG64 seeded with (seed, tensor id).
Values are drawn in float64, rounded to float32 (round-to-nearest-even) and
then to bfloat16 (round-to-nearest-even); both sides of every comparison read
the same bf16 bits, so this double rounding only defines the inputs.
"""
from __future__ import annotations

import numpy as np

# Tensor ids for the per-tensor random streams.
_TENSOR_IDS = {
    "X": 1, "W": 2, "A": 3, "B": 4, "dY": 5,
    "W_up": 6, "A_up": 7, "B_up": 8,
    "Wq": 9, "Ws": 10, "Wq_up": 11, "Ws_up": 12,
    "mask": 13, "mask_up": 14,
    "g": 15, "pos": 16,
    "H": 17, "W_out": 18, "labels": 19, "ignore": 20,
}

ACTS = ("identity", "silu", "swiglu")

# The workloads.  ``act`` names the activation applied after the add;
# ``swiglu`` pairs a gate projection with an up projection.
CONFIGS = {
    "tiny": dict(M=64, d_in=256, d_out=256, r=8, alpha=16.0, act="identity"),
    "q_proj": dict(M=16384, d_in=4096, d_out=4096, r=8, alpha=16.0, act="identity"),
    "v_proj": dict(M=16384, d_in=4096, d_out=1024, r=64, alpha=16.0, act="identity"),
    "mlp_gate_up": dict(M=8192, d_in=4096, d_out=14336, r=64, alpha=16.0, act="swiglu"),
    "mlp_down": dict(M=8192, d_in=14336, d_out=4096, r=64, alpha=16.0, act="identity"),
    "small_m": dict(M=16, d_in=4096, d_out=4096, r=8, alpha=16.0, act="identity"),
    "small_m_ragged": dict(M=1000, d_in=4096, d_out=4096, r=8, alpha=16.0, act="identity"),
    # the few-token workload with the base weight in the 4-bit "w4g64" format
    "small_m_w4": dict(M=16, d_in=4096, d_out=4096, r=8, alpha=16.0, act="identity", weight="w4"),
    # q_proj with dropout p = 0.1 on the adapter input (the mask is drawn here)
    "q_proj_dropout": dict(M=16384, d_in=4096, d_out=4096, r=8, alpha=16.0, act="identity", dropout=0.1),
    # the Llama-3-8B output projection (vocabulary 128256) fused with the
    # cross-entropy loss, 8192 tokens (M = tokens, d_in = hidden, d_out = V)
    "lm_head_ce": dict(M=8192, d_in=4096, d_out=128256, r=0, alpha=0.0, act="ce"),
    # RMSNorm -> q (4096), k (1024), v (1024) LoRA projections, q and k rotated
    # (32 query and 8 key/value heads of 128); 4 sequences of 4096 tokens
    "qkv_rmsnorm_rope": dict(M=16384, d_in=4096, d_out=4096, r=8, alpha=16.0, act="identity",
                             d_kv=1024, head_dim=128, seq_len=4096, eps=1e-6),
}


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Encode float64 values as bfloat16 bit patterns (uint16).

    float64 -> float32 by numpy's RNE cast, then float32 -> bf16 by RNE on the
    upper 16 bits.  Inputs here are finite and far from overflow.
    """
    f = np.ascontiguousarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns to float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TENSOR_IDS[name]])))


def draw(name: str, shape, seed: int, d_in: int) -> np.ndarray:
    """Draw one tensor of the recipe above as bf16 bits."""
    g = _rng(seed, name)
    base = name.replace("_up", "")
    if base in ("X", "dY"):
        v = g.standard_normal(shape)
    elif base == "W":
        v = g.standard_normal(shape) * (1.0 / np.sqrt(d_in))
    elif base == "A":
        lim = 1.0 / np.sqrt(d_in)
        v = g.uniform(-lim, lim, size=shape)
    elif base == "B":
        v = g.standard_normal(shape) * 0.02
    else:  # pragma: no cover
        raise KeyError(name)
    return f64_to_bf16_bits(v)


def draw_w4(name: str, d_out: int, d_in: int, seed: int):
    """A 4-bit weight of the recipe above: (Wq uint8 [d_out x d_in/2], Ws bf16 bits [d_in/64 x d_out]).
    ``name`` is "W" or "W_up"."""
    suffix = name[1:]                       # "" or "_up"
    gq = _rng(seed, "Wq" + suffix)
    Wq = gq.integers(0, 256, size=(d_out, d_in // 2), dtype=np.uint8)
    gs = _rng(seed, "Ws" + suffix)
    Ws = f64_to_bf16_bits(gs.uniform(0.5, 1.5, size=(d_in // 64, d_out)) / (4.6 * np.sqrt(d_in)))
    return Wq, Ws


def draw_ce(M: int, d: int, V: int, seed: int, ignore_frac: float = 0.05, h_scale: float = 1.0):
    """Inputs of the output projection + cross-entropy: (H bf16 bits [M x d],
    W_out bf16 bits [V x d], labels int32 [M]); ``h_scale`` widens the logits."""
    H = f64_to_bf16_bits(_rng(seed, "H").standard_normal((M, d)) * h_scale)
    W = f64_to_bf16_bits(_rng(seed, "W_out").standard_normal((V, d)) / np.sqrt(d))
    labels = _rng(seed, "labels").integers(0, V, size=M).astype(np.int32)
    labels[_rng(seed, "ignore").random(M) < ignore_frac] = -100
    return H, W, labels


def draw_mask(name: str, M: int, d_in: int, p_drop: float, seed: int) -> np.ndarray:
    """A packed dropout mask of the recipe above; ``name`` is "mask" or "mask_up"."""
    keep = _rng(seed, name).random((M, d_in)) >= p_drop
    return np.packbits(keep.astype(np.uint8), axis=1, bitorder="little")


def draw_norm_weight(d: int, seed: int) -> np.ndarray:
    """The RMSNorm weight g [d] of the recipe above, as bf16 bits."""
    return f64_to_bf16_bits(_rng(seed, "g").uniform(0.5, 1.5, size=d))


def draw_positions(M: int, n_pos: int, seed: int) -> np.ndarray:
    """Token positions uniform in [0, n_pos), int32 [M]."""
    return _rng(seed, "pos").integers(0, n_pos, size=M).astype(np.int32)


def sequence_positions(M: int, seq_len: int) -> np.ndarray:
    """Positions of a batch of whole sequences: m mod seq_len, int32 [M]."""
    return (np.arange(M, dtype=np.int64) % seq_len).astype(np.int32)


def rotary_tables(n_pos: int, head_dim: int, base: float = 10000.0):
    """(cos, sin) float32 [n_pos x head_dim/2] of the angles p * base^(-2i/head_dim)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * base ** (-2.0 * i / head_dim)[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def make_inputs(M: int, d_in: int, d_out: int, r: int, act: str = "identity",
                seed: int = 0, with_grad: bool = True) -> dict:
    """All inputs of one fwd(+bwd) call as bf16 bit arrays (uint16, row-major)."""
    out = {
        "X": draw("X", (M, d_in), seed, d_in),
        "W": draw("W", (d_out, d_in), seed, d_in),
        "A": draw("A", (r, d_in), seed, d_in),
        "B": draw("B", (d_out, r), seed, d_in),
    }
    if act == "swiglu":
        out["W_up"] = draw("W_up", (d_out, d_in), seed, d_in)
        out["A_up"] = draw("A_up", (r, d_in), seed, d_in)
        out["B_up"] = draw("B_up", (d_out, r), seed, d_in)
    if with_grad:
        out["dY"] = draw("dY", (M, d_out), seed, d_in)
    return out


def config_inputs(name: str, seed: int = 0, with_grad: bool = True, M: int | None = None) -> dict:
    """Inputs for a named workload; ``M`` overrides the token count."""
    c = CONFIGS[name]
    return make_inputs(M if M is not None else c["M"], c["d_in"], c["d_out"], c["r"],
                       c["act"], seed=seed, with_grad=with_grad)
