"""fp64 CPU oracle for fused linear cross-entropy -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The GPU library never imports it, and
it imports nothing from the GPU library.

``flce`` computes, in fp64, the plain definition of the loss the pages
discuss (PyTorch PR #126348's linear + cross-entropy steps, with the softmax
rebuilt in backward from the logits and the per-row log-sum-exp; torchtune
issue #1228's mean NLL against labels; Liger-Kernel issue #227's Gemma2 logit
softcap).  ``ce`` computes the same loss and its gradient with respect to
the logits for a caller that already holds them (PR #126348's own case: the
row max and sum in the forward, the softmax rebuilt from the logits in the
backward).  The arithmetic lives in ``flce_oracle.c``; this module only
marshals numpy arrays to it.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None

BF16, FP32, FP64 = 0, 1, 2
_ERRORS = {1: "invalid argument", 2: "label outside [0, V) that is not ignore_index",
           3: "out of host memory"}


class OracleLabelError(ValueError):
    """A label is outside [0, V) and is not ignore_index."""


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.flce_oracle.restype = ctypes.c_int
        lib.flce_oracle.argtypes = [i64, i64, i64, ctypes.c_int, p, p, p, i64, ctypes.c_double,
                                    i64, ctypes.c_double, p, p, p, p, p, p]
        lib.flce_oracle_count_valid.restype = i64
        lib.flce_oracle_count_valid.argtypes = [p, i64, i64]
        lib.flce_oracle_threads.restype = ctypes.c_int
        lib.flce_oracle_threads.argtypes = []
        lib.flce_oracle_ce.restype = ctypes.c_int
        lib.flce_oracle_ce.argtypes = [i64, i64, ctypes.c_int, p, i64, p, i64, ctypes.c_double,
                                       i64, ctypes.c_double, p, p, p, p, p]
        _LIB = lib
    return _LIB


def threads() -> int:
    """OpenMP threads the oracle runs with."""
    return int(_lib().flce_oracle_threads())


def _as_input(a, dtype):
    """Return (contiguous array, oracle dtype code).

    dtype: "bf16" means `a` holds raw bf16 bit patterns (uint16 or int16);
    otherwise float32 / float64 arrays are passed as they are.
    """
    if dtype == "bf16":
        a = np.ascontiguousarray(a).view(np.uint16)
        return a, BF16
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, FP32
    if a.dtype == np.float64:
        return a, FP64
    raise TypeError("oracle inputs must be float32, float64 or bf16 bits, got %s" % a.dtype)


def count_valid(labels, ignore_index=-100) -> int:
    labels = np.ascontiguousarray(labels, dtype=np.int64)
    return int(_lib().flce_oracle_count_valid(labels.ctypes.data, labels.shape[0], ignore_index))


def flce(X, W, labels, ignore_index=-100, softcap=0.0, dloss=1.0, n_valid=None, grads=True,
         dtype=None, want_dW=True):
    """Forward and (optionally) backward of FLCE in fp64.

    X: [BT, H], W: [V, H] (float32 / float64, or raw bf16 bits with
    dtype="bf16"); labels: int64 [BT].  softcap <= 0 or non-finite is off.
    n_valid: divisor of the mean (None: count from `labels`).
    Returns a dict with lse, target, n_valid, loss and, if grads, dX and
    (unless want_dW is False) dW.
    """
    Xa, dx = _as_input(X, dtype)
    Wa, dw = _as_input(W, dtype)
    if dx != dw:
        raise TypeError("X and W must have the same dtype")
    if Xa.ndim != 2 or Wa.ndim != 2 or Xa.shape[1] != Wa.shape[1]:
        raise ValueError("X must be [BT, H] and W [V, H]")
    BT, H = Xa.shape
    V = Wa.shape[0]
    lab = np.ascontiguousarray(labels, dtype=np.int64)
    if lab.shape != (BT,):
        raise ValueError("labels must be [BT]")
    lse = np.empty(BT, np.float64)
    target = np.empty(BT, np.float64)
    nv = ctypes.c_int64(0)
    loss = ctypes.c_double(0.0)
    dX = np.empty((BT, H), np.float64) if grads else None
    dW = np.empty((V, H), np.float64) if grads and want_dW else None
    rc = _lib().flce_oracle(
        BT, H, V, dx, Xa.ctypes.data if BT else None, Wa.ctypes.data,
        lab.ctypes.data if BT else None, int(ignore_index), float(softcap),
        -1 if n_valid is None else int(n_valid), float(dloss),
        lse.ctypes.data, target.ctypes.data, ctypes.addressof(nv), ctypes.addressof(loss),
        dX.ctypes.data if grads else None, dW.ctypes.data if dW is not None else None)
    if rc == 2:
        raise OracleLabelError(_ERRORS[2])
    if rc != 0:
        raise RuntimeError("oracle failed: %s" % _ERRORS.get(rc, rc))
    out = {"lse": lse, "target": target, "n_valid": int(nv.value), "loss": float(loss.value)}
    if grads:
        out["dX"] = dX
        if dW is not None:
            out["dW"] = dW
    return out


def ce(Z, labels, ignore_index=-100, softcap=0.0, dloss=1.0, n_valid=None, grads=True,
       dtype=None, V=None):
    """Cross-entropy in fp64 from logits the caller already holds (PyTorch
    PR #126348's case: row max and sum in the forward, the softmax rebuilt
    from the logits and the row statistics in the backward).

    Z: [BT, ld] (float32 / float64, or raw bf16 bits with dtype="bf16"); the
    logits of row i are Z[i, :V] (V defaults to ld, so extra columns model a
    row stride).  labels: int64 [BT].  Returns a dict with lse, target,
    n_valid, loss and, if grads, dZ [BT, V].
    """
    Za, code = _as_input(Z, dtype)
    if Za.ndim != 2:
        raise ValueError("Z must be [BT, ld]")
    BT, ld = Za.shape
    V = ld if V is None else int(V)
    lab = np.ascontiguousarray(labels, dtype=np.int64)
    if lab.shape != (BT,):
        raise ValueError("labels must be [BT]")
    lse = np.empty(BT, np.float64)
    target = np.empty(BT, np.float64)
    nv = ctypes.c_int64(0)
    loss = ctypes.c_double(0.0)
    dZ = np.empty((BT, V), np.float64) if grads else None
    rc = _lib().flce_oracle_ce(
        BT, V, code, Za.ctypes.data if BT else None, ld, lab.ctypes.data if BT else None,
        int(ignore_index), float(softcap), -1 if n_valid is None else int(n_valid),
        float(dloss), lse.ctypes.data, target.ctypes.data, ctypes.addressof(nv),
        ctypes.addressof(loss), dZ.ctypes.data if grads else None)
    if rc == 2:
        raise OracleLabelError(_ERRORS[2])
    if rc != 0:
        raise RuntimeError("oracle failed: %s" % _ERRORS.get(rc, rc))
    out = {"lse": lse, "target": target, "n_valid": int(nv.value), "loss": float(loss.value)}
    if grads:
        out["dZ"] = dZ
    return out


__all__ = ["flce", "ce", "count_valid", "threads", "OracleLabelError"]
