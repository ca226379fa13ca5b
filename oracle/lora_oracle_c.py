"""Python face of the plain C fp64 oracle (oracle/lora_oracle_c.c).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import or call
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

This file only marshals arguments: it converts inputs to contiguous float64
arrays, allocates the outputs and calls the C functions, which hold every
step of the arithmetic.  The function names and the returned dictionaries
match ``oracle/lora_oracle.py`` (the numpy statement of the same layer), so
the same pins (tests/oracle_pins.py) apply to both.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build_oracle

_ACT = {"identity": 0, "silu": 1, "swiglu": 2}


def _in(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class COracle:
    """The C oracle bound to one compiled library (the default one, or a copy
    built from a modified source by the planted-mistake tests)."""

    def __init__(self, path):
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.oracle_threads.restype = ctypes.c_int
        for name in ("oracle_sigmoid", "oracle_silu", "oracle_silu_grad"):
            getattr(L, name).argtypes = [P, P, I64]
            getattr(L, name).restype = None
        L.oracle_bf16_to_f64.argtypes = [P, P, I64]
        L.oracle_bf16_to_f64.restype = None
        L.oracle_lora_forward.argtypes = [I64, I64, I64, I64, ctypes.c_double, ctypes.c_int] + [P] * 12
        L.oracle_lora_forward.restype = ctypes.c_int
        L.oracle_lora_backward.argtypes = [I64, I64, I64, I64, ctypes.c_double, ctypes.c_int] + [P] * 22
        L.oracle_lora_backward.restype = ctypes.c_int
        L.oracle_adapter_grads_identity.argtypes = [I64, I64, I64, I64, ctypes.c_double] + [P] * 8
        L.oracle_adapter_grads_identity.restype = ctypes.c_int
        self.L = L

    def threads(self) -> int:
        return int(self.L.oracle_threads())

    def _elementwise(self, fn, z):
        z = _in(z)
        out = np.empty_like(z)
        fn(_p(z), _p(out), z.size)
        return out

    def bf16_to_f64(self, bits):
        b = np.ascontiguousarray(bits, dtype=np.uint16)
        out = np.empty(b.shape, dtype=np.float64)
        self.L.oracle_bf16_to_f64(_p(b), _p(out), b.size)
        return out

    def sigmoid(self, z):
        return self._elementwise(self.L.oracle_sigmoid, z)

    def silu(self, z):
        return self._elementwise(self.L.oracle_silu, z)

    def silu_grad(self, z):
        return self._elementwise(self.L.oracle_silu_grad, z)

    @staticmethod
    def _operands(X, W, A, B, act, A_up, B_up):
        M, d_in = X.shape
        d_out = W.shape[0]
        r = A.shape[0] if A is not None else 0
        if A is None:
            A, B = np.zeros((0, d_in)), np.zeros((d_out, 0))
        if act == "swiglu" and A_up is None:
            A_up, B_up = np.zeros((0, d_in)), np.zeros((d_out, 0))
        return M, d_in, d_out, r, A, B, A_up, B_up

    def lora_forward(self, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
        X, W, A, B, W_up, A_up, B_up = map(_in, (X, W, A, B, W_up, A_up, B_up))
        M, d_in, d_out, r, A, B, A_up, B_up = self._operands(X, W, A, B, act, A_up, B_up)
        sw = act == "swiglu"
        T, Z, Y = np.empty((M, r)), np.empty((M, d_out)), np.empty((M, d_out))
        T_up = np.empty((M, r)) if sw else None
        Z_up = np.empty((M, d_out)) if sw else None
        rc = self.L.oracle_lora_forward(M, d_in, d_out, r, float(s), _ACT[act], _p(X), _p(W), _p(A), _p(B),
                                        _p(W_up), _p(A_up), _p(B_up), _p(T), _p(Z), _p(Y), _p(T_up), _p(Z_up))
        if rc != 0:
            raise MemoryError(f"oracle_lora_forward returned {rc}")
        out = {"T": T, "Z": Z, "Y": Y}
        if sw:
            out["T_up"], out["Z_up"] = T_up, Z_up
        return out

    def lora_backward(self, dY, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
        dY, X, W, A, B, W_up, A_up, B_up = map(_in, (dY, X, W, A, B, W_up, A_up, B_up))
        M, d_in, d_out, r, A, B, A_up, B_up = self._operands(X, W, A, B, act, A_up, B_up)
        sw = act == "swiglu"
        T, Z, Y = np.empty((M, r)), np.empty((M, d_out)), np.empty((M, d_out))
        T_up = np.empty((M, r)) if sw else None
        Z_up = np.empty((M, d_out)) if sw else None
        dZ, U, dX = np.empty((M, d_out)), np.empty((M, r)), np.empty((M, d_in))
        dA, dB = np.empty((r, d_in)), np.empty((d_out, r))
        dZ_up = np.empty((M, d_out)) if sw else None
        U_up = np.empty((M, r)) if sw else None
        dA_up = np.empty((r, d_in)) if sw else None
        dB_up = np.empty((d_out, r)) if sw else None
        rc = self.L.oracle_lora_backward(M, d_in, d_out, r, float(s), _ACT[act], _p(dY), _p(X), _p(W), _p(A),
                                         _p(B), _p(W_up), _p(A_up), _p(B_up), _p(T), _p(Z), _p(Y), _p(T_up),
                                         _p(Z_up), _p(dZ), _p(dZ_up), _p(U), _p(U_up), _p(dX), _p(dA), _p(dB),
                                         _p(dA_up), _p(dB_up))
        if rc != 0:
            raise MemoryError(f"oracle_lora_backward returned {rc}")
        fwd = {"T": T, "Z": Z, "Y": Y}
        out = {"dZ": dZ, "U": U, "dX": dX, "dA": dA, "dB": dB, "fwd": fwd}
        if sw:
            fwd.update(T_up=T_up, Z_up=Z_up)
            out.update(dZ_up=dZ_up, U_up=U_up, dA_up=dA_up, dB_up=dB_up)
        return out

    def lora_forward_rows(self, rows, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
        """``lora_forward`` restricted to the given token rows (rows are independent)."""
        return self.lora_forward(np.asarray(X)[rows], W, A, B, s, act, W_up, A_up, B_up)

    def lora_backward_rows(self, rows, dY, X, W, A, B, s, act="identity", W_up=None, A_up=None, B_up=None):
        """dX (and dZ, U) for the given token rows only."""
        return self.lora_backward(np.asarray(dY)[rows], np.asarray(X)[rows], W, A, B, s, act, W_up, A_up, B_up)

    def lora_adapter_grads_identity(self, dY, X, A, B, s):
        dY, X, A, B = map(_in, (dY, X, A, B))
        M, d_in = X.shape
        d_out, r = B.shape
        T, U = np.empty((M, r)), np.empty((M, r))
        dA, dB = np.empty((r, d_in)), np.empty((d_out, r))
        self.L.oracle_adapter_grads_identity(M, d_in, d_out, r, float(s), _p(dY), _p(X), _p(A), _p(B), _p(T),
                                             _p(U), _p(dA), _p(dB))
        return {"T": T, "U": U, "dA": dA, "dB": dB}


_default = None


def default() -> COracle:
    """The oracle built from oracle/lora_oracle_c.c (compiled on first use)."""
    global _default
    if _default is None:
        _default = COracle(build_oracle.build())
    return _default


def threads():
    return default().threads()


def bf16_to_f64(bits):
    return default().bf16_to_f64(bits)


def sigmoid(z):
    return default().sigmoid(z)


def silu(z):
    return default().silu(z)


def silu_grad(z):
    return default().silu_grad(z)


def lora_forward(*a, **k):
    return default().lora_forward(*a, **k)


def lora_backward(*a, **k):
    return default().lora_backward(*a, **k)


def lora_forward_rows(*a, **k):
    return default().lora_forward_rows(*a, **k)


def lora_backward_rows(*a, **k):
    return default().lora_backward_rows(*a, **k)


def lora_adapter_grads_identity(*a, **k):
    return default().lora_adapter_grads_identity(*a, **k)


def __getattr__(name):
    # the comparison helpers are not arithmetic of the layer: share them
    if name in ("compare", "ATOL", "RTOL", "NORM_TOL", "ACTS"):
        from . import lora_oracle
        return getattr(lora_oracle, name)
    raise AttributeError(name)
