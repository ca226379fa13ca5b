"""Python binding of the B200 fused LoRA-adapted linear layer (C ABI in
``include/lora_linear.h``).

The functions named like the C entry points (``lora_linear_fwd`` ...) take raw
device pointers (ints) and return the C status code; they only marshal
arguments.  ``forward`` / ``backward`` / ``LoRALinearFunction`` wrap them for
torch tensors (torch provides device memory and the stream).  Every step of the
computation runs in the library's CUDA kernels; there is no fallback: if the
library cannot be loaded, the first call raises ImportError.

The attention-input block (RMSNorm, then the q, k, v projections, q and k
rotated) is a sequence of calls on one stream:

    lora_linear_rmsnorm_fwd(X, g, M, d, eps, Xn, rstd, s)
    lora_linear_fwd_rope(desc_q, rope, Xn, Wq, Aq, Bq, Yq, Tq, ws, n, s)   # q, rotated
    lora_linear_fwd_rope(desc_k, rope, Xn, Wk, Ak, Bk, Yk, Tk, ws, n, s)   # k, rotated
    lora_linear_fwd(desc_v, Xn, Wv, Av, Bv, None, None, None, Yv, Tv, None, ws, n, s)
    lora_linear_bwd_rope(desc_q, rope, dYq, Xn, Wq, Aq, Bq, Tq, dXn, 0, dAq, dBq, ws, n, s)
    lora_linear_bwd_rope(desc_k, rope, dYk, Xn, Wk, Ak, Bk, Tk, dXn, 1, dAk, dBk, ws, n, s)
    lora_linear_bwd_rope(desc_v, None, dYv, Xn, Wv, Av, Bv, Tv, dXn, 1, dAv, dBv, ws, n, s)
    lora_linear_rmsnorm_bwd(X, g, rstd, dXn, M, d, dX, s)

with rope = make_rope_desc(pos, cos, sin, n_pos, head_dim) and dXn an fp32
[M x d] buffer that the q call writes and the k and v calls add to.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblora_linear.so")

ACT_IDENTITY, ACT_SILU, ACT_SWIGLU = 0, 1, 2
ACT_CODES = {"identity": ACT_IDENTITY, "silu": ACT_SILU, "swiglu": ACT_SWIGLU}

STATUS_NAMES = {
    0: "LORA_OK", 1: "LORA_ERR_INVALID_ARG", 2: "LORA_ERR_ALIGNMENT", 3: "LORA_ERR_UNSUPPORTED",
    4: "LORA_ERR_ARCH", 5: "LORA_ERR_WORKSPACE", 6: "LORA_ERR_CUDA", 7: "LORA_ERR_DEVICE_STATUS",
}

# Every symbol include/lora_linear.h declares.
EXPORTED = ("lora_linear_workspace_size", "lora_linear_workspace_init", "lora_linear_device_status",
            "lora_linear_fwd", "lora_linear_bwd", "lora_status_string", "lora_linear_abi_version",
            "lora_linear_launch_count", "lora_linear_fwd_noalloc", "lora_linear_noalloc_status",
            "lora_linear_timing_enable",
            "lora_linear_timing_read", "lora_linear_selftest_wait_timeout",
            "lora_linear_workspace_size_w4", "lora_linear_dequant_w4", "lora_linear_fwd_w4", "lora_linear_bwd_w4",
            "lora_linear_workspace_size_dropout", "lora_linear_fwd_dropout", "lora_linear_bwd_dropout",
            "lora_linear_w4_tiled_bytes", "lora_linear_w4_tile", "lora_linear_fwd_w4_tiled",
            "lora_linear_rmsnorm_fwd", "lora_linear_rmsnorm_bwd", "lora_linear_workspace_size_rope",
            "lora_linear_fwd_rope", "lora_linear_bwd_rope", "lora_linear_ce_workspace_size",
            "lora_linear_ce_fwd", "lora_linear_ce_bwd", "lora_linear_ce_fwd_bwd")


class LoraLinearDesc(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("d_in", ctypes.c_int64), ("d_out", ctypes.c_int64),
                ("r", ctypes.c_int64), ("s", ctypes.c_float), ("act", ctypes.c_int32)]


class LoraRopeDesc(ctypes.Structure):
    """Rotary tables: pos (int32 [M]), cos / sin (fp32 [n_pos x head_dim/2]) device pointers."""
    _fields_ = [("pos", ctypes.c_void_p), ("cos", ctypes.c_void_p), ("sin", ctypes.c_void_p),
                ("n_pos", ctypes.c_int64), ("head_dim", ctypes.c_int32)]


class LoraCeDesc(ctypes.Structure):
    """Output projection + cross-entropy: M tokens, hidden size d, vocabulary V."""
    _fields_ = [("M", ctypes.c_int64), ("d", ctypes.c_int64), ("V", ctypes.c_int64)]


class LoraError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m lora_linear_fine_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, i32, u32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)
    dp = ctypes.POINTER(LoraLinearDesc)
    lib.lora_linear_workspace_size.argtypes = [dp, i32]
    lib.lora_linear_workspace_size.restype = sz
    lib.lora_linear_workspace_init.argtypes = [vp, sz, vp]
    lib.lora_linear_workspace_init.restype = i32
    lib.lora_linear_device_status.argtypes = [vp, vp, u32p]
    lib.lora_linear_device_status.restype = i32
    lib.lora_linear_fwd.argtypes = [dp] + [vp] * 10 + [vp, sz, vp]
    lib.lora_linear_fwd.restype = i32
    lib.lora_linear_bwd.argtypes = [dp] + [vp] * 15 + [vp, sz, vp]
    lib.lora_linear_bwd.restype = i32
    lib.lora_status_string.argtypes = [i32]
    lib.lora_status_string.restype = ctypes.c_char_p
    lib.lora_linear_abi_version.argtypes = []
    lib.lora_linear_abi_version.restype = i32
    lib.lora_linear_launch_count.argtypes = []
    lib.lora_linear_launch_count.restype = ctypes.c_uint64
    lib.lora_linear_fwd_noalloc.argtypes = [dp] + [vp] * 10 + [vp]
    lib.lora_linear_fwd_noalloc.restype = i32
    lib.lora_linear_noalloc_status.argtypes = [vp, u32p]
    lib.lora_linear_noalloc_status.restype = i32
    lib.lora_linear_timing_enable.argtypes = [i32]
    lib.lora_linear_timing_enable.restype = i32
    dblp, u64p = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64)
    lib.lora_linear_timing_read.argtypes = [dblp, u64p, dblp, u64p]
    lib.lora_linear_timing_read.restype = i32
    lib.lora_linear_selftest_wait_timeout.argtypes = [vp, sz, i32, vp]
    lib.lora_linear_selftest_wait_timeout.restype = i32
    lib.lora_linear_workspace_size_w4.argtypes = [dp, i32]
    lib.lora_linear_workspace_size_w4.restype = sz
    lib.lora_linear_dequant_w4.argtypes = [vp, vp, ctypes.c_int64, ctypes.c_int64, vp, vp]
    lib.lora_linear_dequant_w4.restype = i32
    lib.lora_linear_fwd_w4.argtypes = [dp] + [vp] * 12 + [vp, sz, vp]
    lib.lora_linear_fwd_w4.restype = i32
    lib.lora_linear_bwd_w4.argtypes = [dp] + [vp] * 17 + [vp, sz, vp]
    lib.lora_linear_bwd_w4.restype = i32
    i64 = ctypes.c_int64
    lib.lora_linear_w4_tiled_bytes.argtypes = [i64, i64]
    lib.lora_linear_w4_tiled_bytes.restype = sz
    lib.lora_linear_w4_tile.argtypes = [vp, i64, i64, vp, vp]
    lib.lora_linear_w4_tile.restype = i32
    lib.lora_linear_fwd_w4_tiled.argtypes = [dp] + [vp] * 8 + [vp, sz, vp]
    lib.lora_linear_fwd_w4_tiled.restype = i32
    f32 = ctypes.c_float
    lib.lora_linear_workspace_size_dropout.argtypes = [dp, i32]
    lib.lora_linear_workspace_size_dropout.restype = sz
    lib.lora_linear_fwd_dropout.argtypes = [dp] + [vp] * 9 + [f32] + [vp] * 3 + [vp, sz, vp]
    lib.lora_linear_fwd_dropout.restype = i32
    lib.lora_linear_bwd_dropout.argtypes = [dp] + [vp] * 10 + [f32] + [vp] * 7 + [vp, sz, vp]
    lib.lora_linear_bwd_dropout.restype = i32
    rp = ctypes.POINTER(LoraRopeDesc)
    lib.lora_linear_rmsnorm_fwd.argtypes = [vp, vp, i64, i64, f32, vp, vp, vp]
    lib.lora_linear_rmsnorm_fwd.restype = i32
    lib.lora_linear_rmsnorm_bwd.argtypes = [vp, vp, vp, vp, i64, i64, vp, vp]
    lib.lora_linear_rmsnorm_bwd.restype = i32
    lib.lora_linear_workspace_size_rope.argtypes = [dp, i32]
    lib.lora_linear_workspace_size_rope.restype = sz
    lib.lora_linear_fwd_rope.argtypes = [dp, rp] + [vp] * 6 + [vp, sz, vp]
    lib.lora_linear_fwd_rope.restype = i32
    lib.lora_linear_bwd_rope.argtypes = [dp, rp] + [vp] * 7 + [i32, vp, vp] + [vp, sz, vp]
    lib.lora_linear_bwd_rope.restype = i32
    cp = ctypes.POINTER(LoraCeDesc)
    lib.lora_linear_ce_workspace_size.argtypes = [cp, i32]
    lib.lora_linear_ce_workspace_size.restype = sz
    lib.lora_linear_ce_fwd.argtypes = [cp] + [vp] * 5 + [vp, sz, vp]
    lib.lora_linear_ce_fwd.restype = i32
    lib.lora_linear_ce_bwd.argtypes = [cp] + [vp] * 6 + [vp, sz, vp]
    lib.lora_linear_ce_bwd.restype = i32
    lib.lora_linear_ce_fwd_bwd.argtypes = [cp] + [vp] * 7 + [vp, sz, vp]
    lib.lora_linear_ce_fwd_bwd.restype = i32
    return lib


class _LazyLib:
    """Loads the shared library on first use (so the build script can import
    this package before the library exists); a missing library raises."""

    _h = None

    def __getattr__(self, name):
        if _LazyLib._h is None:
            _LazyLib._h = _load()
        return getattr(_LazyLib._h, name)


_lib = _LazyLib()


# ---------------------------------------------------------------------------
# 1:1 wrappers of the C entry points (pointers are ints or None)
# ---------------------------------------------------------------------------
def make_desc(M, d_in, d_out, r, s, act) -> LoraLinearDesc:
    if isinstance(act, str):
        act = ACT_CODES[act]
    return LoraLinearDesc(int(M), int(d_in), int(d_out), int(r), float(s), int(act))


def lora_linear_workspace_size(desc: LoraLinearDesc, for_backward: int) -> int:
    return int(_lib.lora_linear_workspace_size(ctypes.byref(desc), int(for_backward)))


def lora_linear_workspace_init(workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_workspace_init(workspace, workspace_bytes, stream))


def lora_linear_selftest_wait_timeout(workspace, workspace_bytes, limit_log2, stream) -> int:
    return int(_lib.lora_linear_selftest_wait_timeout(workspace, workspace_bytes, int(limit_log2), stream))


def lora_linear_device_status(workspace, stream):
    out = ctypes.c_uint32(0)
    st = int(_lib.lora_linear_device_status(workspace, stream, ctypes.byref(out)))
    return st, int(out.value)


def lora_linear_fwd(desc, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save, workspace, workspace_bytes,
                    stream) -> int:
    return int(_lib.lora_linear_fwd(ctypes.byref(desc), X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save,
                                    workspace, workspace_bytes, stream))


def lora_linear_bwd(desc, dY, X, W, A, B, W_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up, dB_up,
                    workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_bwd(ctypes.byref(desc), dY, X, W, A, B, W_up, A_up, B_up, T_save, Z_save,
                                    dX, dA, dB, dA_up, dB_up, workspace, workspace_bytes, stream))


def lora_linear_fwd_noalloc(desc, X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save, stream) -> int:
    """The forward for callers that cannot allocate device memory: its scratch
    is a fixed 16 MiB device array inside the library (see the C header)."""
    return int(_lib.lora_linear_fwd_noalloc(ctypes.byref(desc), X, W, A, B, W_up, A_up, B_up, Y, T_save, Z_save,
                                            stream))


def lora_linear_noalloc_status(stream):
    """(status code, status word) of the no-alloc forward's scratch array on the
    current device; synchronises ``stream``."""
    out = ctypes.c_uint32(0)
    st = int(_lib.lora_linear_noalloc_status(stream, ctypes.byref(out)))
    return st, int(out.value)


NOALLOC_SCRATCH_BYTES = 16 << 20


# 4-bit frozen base weight ("w4g64": codes two per byte, low nibble first; one
# bf16 scale per row and 64 input features, group-major; W = bf16(scale * (code - 8)))
def lora_linear_workspace_size_w4(desc: LoraLinearDesc, for_backward: int) -> int:
    return int(_lib.lora_linear_workspace_size_w4(ctypes.byref(desc), int(for_backward)))


def lora_linear_dequant_w4(Wq, Ws, d_out, d_in, W, stream) -> int:
    return int(_lib.lora_linear_dequant_w4(Wq, Ws, int(d_out), int(d_in), W, stream))


def lora_linear_fwd_w4(desc, X, Wq, Ws, A, B, Wq_up, Ws_up, A_up, B_up, Y, T_save, Z_save, workspace,
                       workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_fwd_w4(ctypes.byref(desc), X, Wq, Ws, A, B, Wq_up, Ws_up, A_up, B_up, Y, T_save,
                                       Z_save, workspace, workspace_bytes, stream))


def lora_linear_w4_tiled_bytes(d_out, d_in) -> int:
    return int(_lib.lora_linear_w4_tiled_bytes(int(d_out), int(d_in)))


def lora_linear_w4_tile(Wq, d_out, d_in, Wt, stream) -> int:
    return int(_lib.lora_linear_w4_tile(Wq, int(d_out), int(d_in), Wt, stream))


def lora_linear_fwd_w4_tiled(desc, X, Wt, Ws, A, B, Y, T_save, Z_save, workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_fwd_w4_tiled(ctypes.byref(desc), X, Wt, Ws, A, B, Y, T_save, Z_save, workspace,
                                             workspace_bytes, stream))


def lora_linear_bwd_w4(desc, dY, X, Wq, Ws, A, B, Wq_up, Ws_up, A_up, B_up, T_save, Z_save, dX, dA, dB, dA_up,
                       dB_up, workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_bwd_w4(ctypes.byref(desc), dY, X, Wq, Ws, A, B, Wq_up, Ws_up, A_up, B_up, T_save,
                                       Z_save, dX, dA, dB, dA_up, dB_up, workspace, workspace_bytes, stream))


# RMSNorm prologue and rotary-embedding epilogue of the attention-input projections
def make_rope_desc(pos, cos, sin, n_pos, head_dim) -> LoraRopeDesc:
    return LoraRopeDesc(pos, cos, sin, int(n_pos), int(head_dim))


def lora_linear_rmsnorm_fwd(X, g, M, d, eps, Xn, rstd, stream) -> int:
    return int(_lib.lora_linear_rmsnorm_fwd(X, g, int(M), int(d), float(eps), Xn, rstd, stream))


def lora_linear_rmsnorm_bwd(X, g, rstd, dXn, M, d, dX, stream) -> int:
    """dXn: the fp32 sum of the projections' input gradients."""
    return int(_lib.lora_linear_rmsnorm_bwd(X, g, rstd, dXn, int(M), int(d), dX, stream))


def lora_linear_workspace_size_rope(desc: LoraLinearDesc, for_backward: int) -> int:
    return int(_lib.lora_linear_workspace_size_rope(ctypes.byref(desc), int(for_backward)))


def lora_linear_fwd_rope(desc, rope, X, W, A, B, Y, T_save, workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_fwd_rope(ctypes.byref(desc), ctypes.byref(rope), X, W, A, B, Y, T_save, workspace,
                                         workspace_bytes, stream))


def lora_linear_bwd_rope(desc, rope, dY, X, W, A, B, T_save, dXn, accumulate, dA, dB, workspace, workspace_bytes,
                         stream) -> int:
    """rope None: the projection is not rotated (v).  dXn: fp32, written
    (accumulate 0) or added to (accumulate 1)."""
    return int(_lib.lora_linear_bwd_rope(ctypes.byref(desc), None if rope is None else ctypes.byref(rope), dY, X, W,
                                         A, B, T_save, dXn, int(accumulate), dA, dB, workspace, workspace_bytes,
                                         stream))


# Output projection fused with the cross-entropy loss.
def make_ce_desc(M, d, V) -> LoraCeDesc:
    return LoraCeDesc(int(M), int(d), int(V))


def lora_linear_ce_workspace_size(desc, for_backward) -> int:
    return int(_lib.lora_linear_ce_workspace_size(ctypes.byref(desc), int(for_backward)))


def lora_linear_ce_fwd(desc, H, W, labels, loss, lse, workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_ce_fwd(ctypes.byref(desc), H, W, labels, loss, lse, workspace, workspace_bytes,
                                       stream))


def lora_linear_ce_bwd(desc, H, W, labels, lse, dloss, dH, workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_ce_bwd(ctypes.byref(desc), H, W, labels, lse, dloss, dH, workspace, workspace_bytes,
                                       stream))


def lora_linear_ce_fwd_bwd(desc, H, W, labels, dloss, loss, lse, dH, workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_ce_fwd_bwd(ctypes.byref(desc), H, W, labels, dloss, loss, lse, dH, workspace,
                                           workspace_bytes, stream))


def linear_cross_entropy(H, W, labels, workspace=None, stream=None):
    """(loss, lse): the mean cross-entropy of the logits H W^T against int32
    labels (below 0: ignored), for bf16 H [M x d] and W [V x d] on the current
    device.  lse [M] fp32 is the backward's input."""
    import torch
    M, d = H.shape
    V = W.shape[0]
    desc = make_ce_desc(M, d, V)
    ws = (workspace or Workspace(lora_linear_ce_workspace_size(desc, 0), H.device, stream)).ensure(
        lora_linear_ce_workspace_size(desc, 0), stream)
    loss = torch.empty((), dtype=torch.float32, device=H.device)
    lse = torch.empty(M, dtype=torch.float32, device=H.device)
    _check(lora_linear_ce_fwd(desc, _ptr(H), W.data_ptr(), _ptr(labels), loss.data_ptr(), _ptr(lse),
                              ws.buf.data_ptr(), ws.nbytes, _stream_handle(stream)), "lora_linear_ce_fwd")
    return loss, lse


def linear_cross_entropy_backward(H, W, labels, lse, dloss, workspace=None, stream=None):
    """dH (bf16 [M x d]) = dloss * d(loss)/dH; dloss a 0-d fp32 device tensor."""
    import torch
    M, d = H.shape
    V = W.shape[0]
    desc = make_ce_desc(M, d, V)
    ws = (workspace or Workspace(lora_linear_ce_workspace_size(desc, 1), H.device, stream)).ensure(
        lora_linear_ce_workspace_size(desc, 1), stream)
    dH = torch.empty((M, d), dtype=torch.bfloat16, device=H.device)
    _check(lora_linear_ce_bwd(desc, _ptr(H), W.data_ptr(), _ptr(labels), _ptr(lse), dloss.data_ptr(), _ptr(dH),
                              ws.buf.data_ptr(), ws.nbytes, _stream_handle(stream)), "lora_linear_ce_bwd")
    return dH


def lora_linear_timing_enable(enable: int) -> int:
    return int(_lib.lora_linear_timing_enable(int(enable)))


def lora_linear_timing_read():
    """(status, fwd_gemm_ms, fwd_launches, bwd_gemm_ms, bwd_launches) since the last read."""
    fm, bm = ctypes.c_double(0), ctypes.c_double(0)
    fl, bl = ctypes.c_uint64(0), ctypes.c_uint64(0)
    st = int(_lib.lora_linear_timing_read(ctypes.byref(fm), ctypes.byref(fl), ctypes.byref(bm), ctypes.byref(bl)))
    return st, fm.value, int(fl.value), bm.value, int(bl.value)


def status_string(status: int) -> str:
    s = _lib.lora_status_string(int(status))
    return s.decode() if s else "?"


def lora_linear_abi_version() -> int:
    return int(_lib.lora_linear_abi_version())


def lora_linear_launch_count() -> int:
    return int(_lib.lora_linear_launch_count())


# ---------------------------------------------------------------------------
# torch-tensor convenience layer (device memory + stream only)
# ---------------------------------------------------------------------------
def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream_handle(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(st: int, what: str):
    if st != 0:
        raise LoraError(st, what)


class Workspace:
    """A device workspace (torch uint8 tensor) whose status word is zeroed once."""

    def __init__(self, nbytes: int, device=None, stream=None):
        import torch
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        _check(lora_linear_workspace_init(self.buf.data_ptr(), self.nbytes, _stream_handle(stream)),
               "lora_linear_workspace_init")

    def ensure(self, nbytes: int, stream=None):
        if nbytes > self.nbytes:
            self.__init__(nbytes, self.buf.device, stream)
        return self

    def status(self, stream=None):
        st, word = lora_linear_device_status(self.buf.data_ptr(), _stream_handle(stream))
        return word


def forward(X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None, save=True, workspace=None,
            stream=None):
    """Y (and the saved T, Z for the backward) for bf16 tensors on the current device."""
    import torch
    M, d_in = X.shape
    d_out = W.shape[0]
    r = 0 if A is None else A.shape[0]
    act_code = ACT_CODES[act] if isinstance(act, str) else act
    desc = make_desc(M, d_in, d_out, r, s, act_code)
    np_ = 2 if act_code == ACT_SWIGLU else 1
    Y = torch.empty((M, d_out), dtype=torch.bfloat16, device=X.device)
    T = torch.empty((np_, M, r), dtype=torch.float32, device=X.device) if (save and r > 0) else None
    Z = (torch.empty((np_, M, d_out), dtype=torch.float32, device=X.device)
         if (save and act_code != ACT_IDENTITY) else None)
    need = lora_linear_workspace_size(desc, 0)
    ws = (workspace or Workspace(need, X.device, stream)).ensure(need, stream)
    _check(lora_linear_fwd(desc, _ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(W_up), _ptr(A_up), _ptr(B_up),
                           _ptr(Y), _ptr(T), _ptr(Z), ws.buf.data_ptr(), ws.nbytes, _stream_handle(stream)),
           "lora_linear_fwd")
    return Y, T, Z


def backward(dY, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None, T_save=None, Z_save=None,
             workspace=None, stream=None):
    """dX, dA, dB (and dA_up, dB_up for swiglu)."""
    import torch
    M, d_in = X.shape
    d_out = W.shape[0]
    r = 0 if A is None else A.shape[0]
    act_code = ACT_CODES[act] if isinstance(act, str) else act
    desc = make_desc(M, d_in, d_out, r, s, act_code)
    dX = torch.empty((M, d_in), dtype=torch.bfloat16, device=X.device)
    dA = torch.empty((r, d_in), dtype=torch.float32, device=X.device) if r > 0 else None
    dB = torch.empty((d_out, r), dtype=torch.float32, device=X.device) if r > 0 else None
    sw = act_code == ACT_SWIGLU
    dA_up = torch.empty_like(dA) if (sw and r > 0) else None
    dB_up = torch.empty_like(dB) if (sw and r > 0) else None
    need = lora_linear_workspace_size(desc, 1)
    ws = (workspace or Workspace(need, X.device, stream)).ensure(need, stream)
    _check(lora_linear_bwd(desc, _ptr(dY), _ptr(X), _ptr(W), _ptr(A), _ptr(B), _ptr(W_up), _ptr(A_up),
                           _ptr(B_up), _ptr(T_save), _ptr(Z_save), _ptr(dX), _ptr(dA), _ptr(dB), _ptr(dA_up),
                           _ptr(dB_up), ws.buf.data_ptr(), ws.nbytes, _stream_handle(stream)),
           "lora_linear_bwd")
    return dX, dA, dB, dA_up, dB_up


def _make_autograd():
    import torch

    class LoRALinearFunction(torch.autograd.Function):
        """y = act(x W^T + s (x A^T) B^T) with W frozen; grads for x, A, B.

        A and B are bf16 parameters; their gradients come back from the kernels
        in fp32 and are cast to the parameter dtype by autograd's contract."""

        @staticmethod
        def forward(ctx, X, W, A, B, s, act):
            Y, T, Z = forward(X, W, A, B, s, act)
            ctx.save_for_backward(X, W, A, B, T, Z)
            ctx.s, ctx.act = s, act
            return Y

        @staticmethod
        def backward(ctx, dY):
            X, W, A, B, T, Z = ctx.saved_tensors
            dX, dA, dB, _, _ = backward(dY.contiguous(), X, W, A, B, ctx.s, ctx.act, T_save=T, Z_save=Z)
            return dX, None, dA.to(A.dtype), dB.to(B.dtype), None, None

    return LoRALinearFunction


try:  # torch is optional for the 1:1 C wrappers
    LoRALinearFunction = _make_autograd()
except Exception:  # pragma: no cover
    LoRALinearFunction = None


# dropout on the adapter branch's input (mask: [M x d_in/8] bytes, bit j of byte b keeps element 8b + j)
def lora_linear_workspace_size_dropout(desc: LoraLinearDesc, for_backward: int) -> int:
    return int(_lib.lora_linear_workspace_size_dropout(ctypes.byref(desc), int(for_backward)))


def lora_linear_fwd_dropout(desc, X, W, A, B, W_up, A_up, B_up, mask, mask_up, p_drop, Y, T_save, Z_save,
                            workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_fwd_dropout(ctypes.byref(desc), X, W, A, B, W_up, A_up, B_up, mask, mask_up,
                                            float(p_drop), Y, T_save, Z_save, workspace, workspace_bytes, stream))


def lora_linear_bwd_dropout(desc, dY, X, W, A, B, W_up, A_up, B_up, mask, mask_up, p_drop, T_save, Z_save, dX, dA,
                            dB, dA_up, dB_up, workspace, workspace_bytes, stream) -> int:
    return int(_lib.lora_linear_bwd_dropout(ctypes.byref(desc), dY, X, W, A, B, W_up, A_up, B_up, mask, mask_up,
                                            float(p_drop), T_save, Z_save, dX, dA, dB, dA_up, dB_up, workspace,
                                            workspace_bytes, stream))


def linear_cross_entropy_fwd_bwd(H, W, labels, dloss, workspace=None, stream=None):
    """(loss, lse, dH) in one call, for a loss that is the step's final scalar
    (dloss: its upstream factor, a 0-d fp32 device tensor): the same results
    as linear_cross_entropy followed by linear_cross_entropy_backward, without
    recomputing the logits."""
    import torch
    M, d = H.shape
    V = W.shape[0]
    desc = make_ce_desc(M, d, V)
    ws = (workspace or Workspace(lora_linear_ce_workspace_size(desc, 2), H.device, stream)).ensure(
        lora_linear_ce_workspace_size(desc, 2), stream)
    loss = torch.empty((), dtype=torch.float32, device=H.device)
    lse = torch.empty(M, dtype=torch.float32, device=H.device)
    dH = torch.empty((M, d), dtype=torch.bfloat16, device=H.device)
    _check(lora_linear_ce_fwd_bwd(desc, _ptr(H), W.data_ptr(), _ptr(labels), dloss.data_ptr(), loss.data_ptr(),
                                  _ptr(lse), _ptr(dH), ws.buf.data_ptr(), ws.nbytes, _stream_handle(stream)),
           "lora_linear_ce_fwd_bwd")
    return loss, lse, dH
