"""ctypes binding of the FLCE C ABI (include/flce.h).

The functions here carry the C names and only marshal arguments: torch
tensors become device pointers, the problem becomes an ``flce_problem_t``
(or ``flce_ce_problem_t``), and a non-OK status becomes an ``FlceError``.
Before a pointer is taken, each tensor is checked against the problem it is
passed with (shape, element type, row stride, device), and a mismatch
raises ``ValueError``: the C ABI sees only addresses and sizes, so a tensor
whose layout differs from the problem's would otherwise be read wrongly.  Every step of the computation
runs in the CUDA kernels of ``_build/libflce.so``; if that library is missing
the first call raises instead of computing anything another way.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "libflce.so")

FLCE_BF16, FLCE_FP32 = 0, 1
FLCE_OP_FORWARD, FLCE_OP_BACKWARD, FLCE_OP_FUSED = 0, 1, 2

STATUS_NAMES = {
    0: "FLCE_OK", 1: "FLCE_ERR_INVALID_ARG", 2: "FLCE_ERR_UNSUPPORTED",
    3: "FLCE_ERR_MISALIGNED", 4: "FLCE_ERR_WORKSPACE_TOO_SMALL",
    5: "FLCE_ERR_LABEL_OUT_OF_RANGE", 6: "FLCE_ERR_TIMEOUT", 7: "FLCE_ERR_CUDA",
}

# Every symbol include/flce.h declares.
EXPORTS = ("flce_workspace_size", "flce_forward", "flce_backward", "flce_fused",
           "flce_get_device_status", "flce_status_string", "flce_set_wait_limit_ns",
           "flce_last_launch_count", "flce_profile_start", "flce_profile_stop",
           "flce_kernel_name", "flce_fused_noalloc", "flce_set_schedule",
           "flce_selftest_wait_timeout", "flce_count_valid", "flce_fused_global",
           "flce_ce_workspace_size", "flce_ce_forward", "flce_ce_backward",
           "flce_selftest_approx", "flce_set_workspace_limit", "flce_ce_fused",
           "flce_vp_workspace_size", "flce_vp_forward", "flce_vp_combine", "flce_vp_backward",
           "flce_fused_global_sliced", "flce_dw_slice_rows")
FLCE_SCHEDULE_AUTO, FLCE_SCHEDULE_RECOMPUTE, FLCE_SCHEDULE_FUSED_FORWARD = 0, 1, 2


class FlceError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, STATUS_NAMES.get(status, status),
                                          flce_status_string(status)))


class flce_problem_t(ctypes.Structure):
    _fields_ = [("BT", ctypes.c_int64), ("H", ctypes.c_int64), ("V", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("shift_seq_len", ctypes.c_int32),
                ("ignore_index", ctypes.c_int64), ("softcap", ctypes.c_float),
                ("dw_fp32", ctypes.c_int32), ("ldx", ctypes.c_int64), ("ldw", ctypes.c_int64),
                ("lddx", ctypes.c_int64), ("lddw", ctypes.c_int64)]


class flce_ce_problem_t(ctypes.Structure):
    _fields_ = [("BT", ctypes.c_int64), ("V", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("shift_seq_len", ctypes.c_int32), ("ignore_index", ctypes.c_int64),
                ("softcap", ctypes.c_float), ("reserved1", ctypes.c_int32),
                ("ld", ctypes.c_int64), ("ld_grad", ctypes.c_int64)]


_LIB = None


def lib():
    """Load libflce.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("FLCE CUDA library not built: %s is missing "
                               "(run linear_cross_entropy_tiles_b200/build.py)" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, p = ctypes.POINTER(flce_problem_t), ctypes.c_void_p
        L.flce_workspace_size.restype = ctypes.c_size_t
        L.flce_workspace_size.argtypes = [P, ctypes.c_int]
        L.flce_forward.restype = ctypes.c_int
        L.flce_forward.argtypes = [P, p, p, p, p, p, p, ctypes.c_size_t, p]
        L.flce_backward.restype = ctypes.c_int
        L.flce_backward.argtypes = [P, p, p, p, p, p, p, p, p, ctypes.c_size_t, p]
        L.flce_fused.restype = ctypes.c_int
        L.flce_fused.argtypes = [P, p, p, p, ctypes.c_float, p, p, p, p, ctypes.c_size_t, p]
        L.flce_get_device_status.restype = ctypes.c_int
        L.flce_get_device_status.argtypes = [p, p, ctypes.POINTER(ctypes.c_int32),
                                             ctypes.POINTER(ctypes.c_int64)]
        L.flce_status_string.restype = ctypes.c_char_p
        L.flce_status_string.argtypes = [ctypes.c_int]
        L.flce_set_wait_limit_ns.restype = ctypes.c_uint64
        L.flce_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.flce_last_launch_count.restype = ctypes.c_int32
        L.flce_last_launch_count.argtypes = []
        L.flce_profile_start.restype = ctypes.c_int
        L.flce_profile_start.argtypes = [ctypes.c_int32]
        L.flce_profile_stop.restype = ctypes.c_int32
        L.flce_profile_stop.argtypes = [ctypes.POINTER(ctypes.c_float),
                                        ctypes.POINTER(ctypes.c_int32), ctypes.c_int32]
        L.flce_kernel_name.restype = ctypes.c_char_p
        L.flce_kernel_name.argtypes = [ctypes.c_int32]
        L.flce_selftest_wait_timeout.restype = ctypes.c_int
        L.flce_selftest_wait_timeout.argtypes = [p, ctypes.c_uint64, p]
        L.flce_set_schedule.restype = ctypes.c_int32
        L.flce_set_schedule.argtypes = [ctypes.c_int32]
        L.flce_fused_noalloc.restype = ctypes.c_int
        L.flce_fused_noalloc.argtypes = [P, p, p, p, ctypes.c_float, p, p, p, p]
        L.flce_count_valid.restype = ctypes.c_int
        L.flce_count_valid.argtypes = [P, p, p, p]
        L.flce_fused_global.restype = ctypes.c_int
        L.flce_fused_global.argtypes = [P, p, p, p, p, ctypes.c_float, p, p, p, p,
                                        ctypes.c_size_t, p]
        L.flce_fused_global_sliced.restype = ctypes.c_int
        L.flce_fused_global_sliced.argtypes = [P, p, p, p, p, ctypes.c_float, p, p, p, p,
                                               ctypes.c_size_t, ctypes.c_int32,
                                               ctypes.POINTER(ctypes.c_void_p), p]
        L.flce_dw_slice_rows.restype = ctypes.c_int64
        L.flce_dw_slice_rows.argtypes = [ctypes.c_int64, ctypes.c_int32]
        L.flce_set_workspace_limit.restype = ctypes.c_uint64
        L.flce_set_workspace_limit.argtypes = [ctypes.c_uint64]
        L.flce_selftest_approx.restype = ctypes.c_int
        L.flce_selftest_approx.argtypes = [p, ctypes.c_int64, p, p]
        i64 = ctypes.c_int64
        L.flce_vp_workspace_size.restype = ctypes.c_size_t
        L.flce_vp_workspace_size.argtypes = [P, ctypes.c_int]
        L.flce_vp_forward.restype = ctypes.c_int
        L.flce_vp_forward.argtypes = [P, i64, i64, p, p, p, p, p, ctypes.c_size_t, p]
        L.flce_vp_combine.restype = ctypes.c_int
        L.flce_vp_combine.argtypes = [P, ctypes.c_int32, p, p, p, p, p, ctypes.c_size_t, p]
        L.flce_vp_backward.restype = ctypes.c_int
        L.flce_vp_backward.argtypes = [P, i64, i64, p, p, p, p, p, p, p, p, ctypes.c_size_t, p]
        C = ctypes.POINTER(flce_ce_problem_t)
        L.flce_ce_workspace_size.restype = ctypes.c_size_t
        L.flce_ce_workspace_size.argtypes = [C, ctypes.c_int]
        L.flce_ce_forward.restype = ctypes.c_int
        L.flce_ce_forward.argtypes = [C, p, p, p, p, p, ctypes.c_size_t, p]
        L.flce_ce_fused.restype = ctypes.c_int
        L.flce_ce_fused.argtypes = [C, p, p, ctypes.c_float, p, p, p, p, ctypes.c_size_t, p]
        L.flce_ce_backward.restype = ctypes.c_int
        L.flce_ce_backward.argtypes = [C, p, p, p, p, p, p, ctypes.c_size_t, p]
        _LIB = L
    return _LIB


_DTYPES = {torch.bfloat16: FLCE_BF16, torch.float32: FLCE_FP32}


def _dtype_code(dtype):
    return _DTYPES.get(dtype, 99) if isinstance(dtype, torch.dtype) else int(dtype)


def make_problem(BT, H, V, dtype=FLCE_BF16, ignore_index=-100, softcap=0.0,
                 shift_seq_len=0, ldx=0, ldw=0, lddx=0, lddw=0, dw_fp32=0) -> flce_problem_t:
    """An flce_problem_t; the row strides ld* are in elements, 0 = H;
    dw_fp32 = 1 asks for an fp32 dW whatever the input type."""
    return flce_problem_t(int(BT), int(H), int(V), _dtype_code(dtype), int(shift_seq_len),
                          int(ignore_index), float(softcap), int(dw_fp32), int(ldx), int(ldw),
                          int(lddx), int(lddw))


def make_ce_problem(BT, V, dtype=FLCE_BF16, ignore_index=-100, softcap=0.0, shift_seq_len=0,
                    ld=0, ld_grad=0) -> flce_ce_problem_t:
    """An flce_ce_problem_t; ld, ld_grad are row strides in elements, 0 = V."""
    return flce_ce_problem_t(int(BT), int(V), _dtype_code(dtype), int(shift_seq_len),
                             int(ignore_index), float(softcap), 0, int(ld), int(ld_grad))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr() if t.numel() > 0 else None


def _row_stride(t):
    """Elements between rows of a 2-D tensor whose rows are unit-stride."""
    if t.dim() != 2:
        raise ValueError("expected a 2-D tensor, got shape %s" % (tuple(t.shape),))
    if t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError("rows must be unit-stride (got strides %s)" % (t.stride(),))
    return t.stride(0) if t.shape[0] > 1 else t.shape[1]


def _check_matrix(name, t, rows, cols, dtype_code, ld, device):
    """Raise unless tensor t is a rows x cols matrix of the problem's dtype
    whose rows lie ld elements apart (0 = cols), on `device`."""
    if not isinstance(t, torch.Tensor):
        return device  # a raw address: the caller vouches for it
    if tuple(t.shape) != (rows, cols):
        raise ValueError("%s: shape %s, the problem says (%d, %d)"
                         % (name, tuple(t.shape), rows, cols))
    if _DTYPES.get(t.dtype) != dtype_code:
        raise ValueError("%s: dtype %s does not match the problem's" % (name, t.dtype))
    if rows > 1 and cols > 0 and _row_stride(t) != (ld or cols):
        raise ValueError("%s: row stride %d, the problem says %d"
                         % (name, _row_stride(t), ld or cols))
    if t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError("%s: rows must be unit-stride" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (got %s)" % (name, t.device))
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, other arguments on %s" % (name, t.device, device))
    return t.device


def _check_vector(name, t, n, dtype, device):
    if not isinstance(t, torch.Tensor):
        return device
    if t.dtype != dtype or t.numel() != n or (n > 1 and not t.is_contiguous()):
        raise ValueError("%s: need a dense %s tensor of %d elements, got %s %s"
                         % (name, dtype, n, t.dtype, tuple(t.shape)))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (got %s)" % (name, t.device))
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, other arguments on %s" % (name, t.device, device))
    return t.device


def _check_flce(p, X=None, W=None, labels=None, dX=None, dW=None, lse=None, extra=()):
    """Tensors passed with an flce_problem_t must be laid out as it says."""
    dev = None
    dev = _check_matrix("X", X, p.BT, p.H, p.dtype, p.ldx, dev)
    dev = _check_matrix("W", W, p.V, p.H, p.dtype, p.ldw, dev)
    dev = _check_matrix("dX", dX, p.BT, p.H, p.dtype, p.lddx, dev)
    dev = _check_matrix("dW", dW, p.V, p.H, FLCE_FP32 if p.dw_fp32 else p.dtype, p.lddw, dev)
    dev = _check_vector("labels", labels, p.BT, torch.int64, dev)
    dev = _check_vector("lse", lse, p.BT, torch.float32, dev)
    for name, t, n, dt in extra:
        dev = _check_vector(name, t, n, dt, dev)


def _check_ce(p, logits=None, labels=None, lse=None, dlogits=None, extra=()):
    dev = None
    dev = _check_matrix("logits", logits, p.BT, p.V, p.dtype, p.ld, dev)
    dev = _check_matrix("dlogits", dlogits, p.BT, p.V, p.dtype, p.ld_grad, dev)
    dev = _check_vector("labels", labels, p.BT, torch.int64, dev)
    dev = _check_vector("lse", lse, p.BT, torch.float32, dev)
    for name, t, n, dt in extra:
        dev = _check_vector(name, t, n, dt, dev)


def _nbytes(ws):
    return ws.numel() * ws.element_size()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status, where):
    if status != 0:
        raise FlceError(status, where)


def flce_status_string(status: int) -> str:
    return lib().flce_status_string(int(status)).decode()


def flce_workspace_size(problem: flce_problem_t, op: int) -> int:
    return int(lib().flce_workspace_size(ctypes.byref(problem), int(op)))


def flce_forward(problem, X, W, labels, loss, lse, ws, stream=None):
    _check_flce(problem, X=X, W=W, labels=labels, lse=lse,
                extra=[("loss", loss, 1, torch.float32)])
    _check(lib().flce_forward(ctypes.byref(problem), _ptr(X), _ptr(W), _ptr(labels), _ptr(loss),
                              _ptr(lse), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)), "flce_forward")


def flce_backward(problem, X, W, labels, lse, dloss, dX, dW, ws, stream=None):
    _check_flce(problem, X=X, W=W, labels=labels, lse=lse, dX=dX, dW=dW,
                extra=[("dloss", dloss, 1, torch.float32)])
    _check(lib().flce_backward(ctypes.byref(problem), _ptr(X), _ptr(W), _ptr(labels), _ptr(lse),
                               _ptr(dloss), _ptr(dX), _ptr(dW), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "flce_backward")


def flce_fused(problem, X, W, labels, dloss, loss, dX, dW, ws, stream=None):
    _check_flce(problem, X=X, W=W, labels=labels, dX=dX, dW=dW,
                extra=[("loss", loss, 1, torch.float32)])
    _check(lib().flce_fused(ctypes.byref(problem), _ptr(X), _ptr(W), _ptr(labels), float(dloss),
                            _ptr(loss), _ptr(dX), _ptr(dW), _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream)), "flce_fused")


def flce_count_valid(problem, labels, n_valid, stream=None):
    """n_valid (device int64 [1]) = number of rows whose (shifted) label is
    not the problem's ignore_index."""
    _check_flce(problem, labels=labels, extra=[("n_valid", n_valid, 1, torch.int64)])
    _check(lib().flce_count_valid(ctypes.byref(problem), _ptr(labels), _ptr(n_valid),
                                  _stream(stream)), "flce_count_valid")


def flce_fused_global(problem, X, W, labels, n_valid_global, dloss, loss, dX, dW, ws,
                      stream=None):
    """flce_fused with the mean's divisor taken from n_valid_global (device int64 [1])."""
    _check_flce(problem, X=X, W=W, labels=labels, dX=dX, dW=dW,
                extra=[("loss", loss, 1, torch.float32),
                       ("n_valid_global", n_valid_global, 1, torch.int64)])
    _check(lib().flce_fused_global(ctypes.byref(problem), _ptr(X), _ptr(W), _ptr(labels),
                                   _ptr(n_valid_global), float(dloss), _ptr(loss), _ptr(dX),
                                   _ptr(dW), _ptr(ws), ws.numel() * ws.element_size(),
                                   _stream(stream)), "flce_fused_global")


def _event_handle(ev, stream):
    """The cudaEvent_t of a torch.cuda.Event (an int passes through).  torch
    creates an event's CUDA object on its first record, so an event never
    recorded is recorded once on `stream` first (the call records it again)."""
    if isinstance(ev, int):
        return ev
    if not ev.cuda_event:
        ev.record(stream if stream is not None else torch.cuda.current_stream())
    return ev.cuda_event


def flce_fused_global_sliced(problem, X, W, labels, n_valid_global, dloss, loss, dX, dW, ws,
                             events, stream=None):
    """flce_fused_global (flce_fused when n_valid_global is None) recording
    events[s] once vocabulary slice s of dW (dw_slice_bounds) is final."""
    extra = [("loss", loss, 1, torch.float32)]
    if n_valid_global is not None:
        extra.append(("n_valid_global", n_valid_global, 1, torch.int64))
    _check_flce(problem, X=X, W=W, labels=labels, dX=dX, dW=dW, extra=extra)
    if not events:
        raise ValueError("flce_fused_global_sliced needs at least one event")
    handles = (ctypes.c_void_p * len(events))(*[_event_handle(e, stream) for e in events])
    _check(lib().flce_fused_global_sliced(ctypes.byref(problem), _ptr(X), _ptr(W), _ptr(labels),
                                          _ptr(n_valid_global), float(dloss), _ptr(loss),
                                          _ptr(dX), _ptr(dW), _ptr(ws),
                                          ws.numel() * ws.element_size(), len(events), handles,
                                          _stream(stream)), "flce_fused_global_sliced")


def flce_dw_slice_rows(V: int, n_slices: int) -> int:
    return int(lib().flce_dw_slice_rows(int(V), int(n_slices)))


def dw_slice_bounds(V: int, n_slices: int):
    """[(first row, end row)] of the n_slices vocabulary slices of dW that
    flce_fused_global_sliced hands over (trailing slices may be empty)."""
    r = flce_dw_slice_rows(V, n_slices)
    if r <= 0:
        raise ValueError("need V > 0 and 1 <= n_slices <= 64")
    return [(min(V, s * r), min(V, (s + 1) * r)) for s in range(n_slices)]


def flce_fused_noalloc(problem, X, W, labels, dloss, loss, dX, dW, stream=None):
    """flce_fused with the library's fixed scratch array instead of a workspace."""
    _check_flce(problem, X=X, W=W, labels=labels, dX=dX, dW=dW,
                extra=[("loss", loss, 1, torch.float32)])
    _check(lib().flce_fused_noalloc(ctypes.byref(problem), _ptr(X), _ptr(W), _ptr(labels),
                                    float(dloss), _ptr(loss), _ptr(dX), _ptr(dW),
                                    _stream(stream)), "flce_fused_noalloc")


def flce_ce_workspace_size(problem: flce_ce_problem_t, op: int) -> int:
    return int(lib().flce_ce_workspace_size(ctypes.byref(problem), int(op)))


def flce_ce_forward(problem, logits, labels, loss, lse, ws, stream=None):
    """loss and lse from logits the caller holds (one read of them)."""
    _check_ce(problem, logits=logits, labels=labels, lse=lse,
              extra=[("loss", loss, 1, torch.float32)])
    _check(lib().flce_ce_forward(ctypes.byref(problem), _ptr(logits), _ptr(labels), _ptr(loss),
                                 _ptr(lse), _ptr(ws), _nbytes(ws), _stream(stream)),
           "flce_ce_forward")


def flce_ce_backward(problem, logits, labels, lse, dloss, dlogits, ws, stream=None):
    """dlogits from the logits and the forward's lse; dlogits may be logits."""
    _check_ce(problem, logits=logits, labels=labels, lse=lse, dlogits=dlogits,
              extra=[("dloss", dloss, 1, torch.float32)])
    _check(lib().flce_ce_backward(ctypes.byref(problem), _ptr(logits), _ptr(labels), _ptr(lse),
                                  _ptr(dloss), _ptr(dlogits), _ptr(ws), _nbytes(ws),
                                  _stream(stream)), "flce_ce_backward")


def flce_ce_fused(problem, logits, labels, dloss, loss, lse, dlogits, ws, stream=None):
    """loss, lse (or None) and dlogits in one read of the logits."""
    _check_ce(problem, logits=logits, labels=labels, lse=lse, dlogits=dlogits,
              extra=[("loss", loss, 1, torch.float32)])
    _check(lib().flce_ce_fused(ctypes.byref(problem), _ptr(logits), _ptr(labels), float(dloss),
                               _ptr(loss), _ptr(lse), _ptr(dlogits), _ptr(ws), _nbytes(ws),
                               _stream(stream)), "flce_ce_fused")


def flce_vp_workspace_size(problem: flce_problem_t, op: int) -> int:
    return int(lib().flce_vp_workspace_size(ctypes.byref(problem), int(op)))


def flce_vp_forward(problem, v_offset, v_total, X, W, labels, stats, ws, stream=None):
    """stats [BT, 3] fp32: this rank's per-row (max, sum-exp, label logit) over
    its vocabulary slice [v_offset, v_offset + problem.V)."""
    _check_flce(problem, X=X, W=W, labels=labels,
                extra=[("stats", stats, 3 * problem.BT, torch.float32)])
    _check(lib().flce_vp_forward(ctypes.byref(problem), int(v_offset), int(v_total), _ptr(X),
                                 _ptr(W), _ptr(labels), _ptr(stats), _ptr(ws), _nbytes(ws),
                                 _stream(stream)), "flce_vp_forward")


def flce_vp_combine(problem, n_ranks, stats_all, labels, loss, lse, ws, stream=None):
    """lse and loss from all ranks' stats [n_ranks, BT, 3]; problem.V is the
    whole vocabulary."""
    _check_flce(problem, labels=labels, lse=lse,
                extra=[("stats_all", stats_all, 3 * n_ranks * problem.BT, torch.float32),
                       ("loss", loss, 1, torch.float32)])
    _check(lib().flce_vp_combine(ctypes.byref(problem), int(n_ranks), _ptr(stats_all),
                                 _ptr(labels), _ptr(loss), _ptr(lse), _ptr(ws), _nbytes(ws),
                                 _stream(stream)), "flce_vp_combine")


def flce_vp_backward(problem, v_offset, v_total, X, W, labels, lse, dloss, dX, dW, ws,
                     stream=None):
    """This rank's fp32 share of dX and its rows of dW from the global lse."""
    _check_flce(problem, X=X, W=W, labels=labels, lse=lse, dW=dW,
                extra=[("dloss", dloss, 1, torch.float32)])
    if isinstance(dX, torch.Tensor):
        _check_matrix("dX", dX, problem.BT, problem.H, FLCE_FP32, problem.lddx, None)
    _check(lib().flce_vp_backward(ctypes.byref(problem), int(v_offset), int(v_total), _ptr(X),
                                  _ptr(W), _ptr(labels), _ptr(lse), _ptr(dloss), _ptr(dX),
                                  _ptr(dW), _ptr(ws), _nbytes(ws), _stream(stream)),
           "flce_vp_backward")


def flce_get_device_status(ws, stream=None):
    st = ctypes.c_int32(0)
    nv = ctypes.c_int64(0)
    _check(lib().flce_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(st),
                                        ctypes.byref(nv)), "flce_get_device_status")
    return int(st.value), int(nv.value)


def flce_selftest_wait_timeout(ws, limit_ns: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test kernel (records FLCE_ERR_TIMEOUT in ws)."""
    _check(lib().flce_selftest_wait_timeout(_ptr(ws), int(limit_ns), _stream(stream)),
           "flce_selftest_wait_timeout")


def flce_selftest_approx(x: torch.Tensor) -> torch.Tensor:
    """[n, 4] fp32: the epilogues' tanh, CUDA's tanhf, the epilogues' exp2,
    CUDA's exp2f, evaluated on the device at the fp32 CUDA tensor x."""
    x = x.contiguous()
    if x.dtype != torch.float32 or not x.is_cuda:
        raise ValueError("x must be a float32 CUDA tensor")
    out = torch.empty(x.numel(), 4, dtype=torch.float32, device=x.device)
    _check(lib().flce_selftest_approx(_ptr(x), x.numel(), _ptr(out), _stream(None)),
           "flce_selftest_approx")
    return out


def flce_set_schedule(schedule: int) -> int:
    """Set the process-wide flce_fused schedule; returns the previous one."""
    prev = int(lib().flce_set_schedule(int(schedule)))
    if prev < 0:
        raise FlceError(1, "flce_set_schedule")
    return prev


def flce_set_workspace_limit(nbytes: int) -> int:
    """Cap the workspace the automatic flce_fused schedule plans (0 = none);
    returns the previous cap."""
    return int(lib().flce_set_workspace_limit(int(nbytes)))


def flce_set_wait_limit_ns(ns: int) -> int:
    return int(lib().flce_set_wait_limit_ns(int(ns)))


def flce_last_launch_count() -> int:
    return int(lib().flce_last_launch_count())


def flce_profile_start(n: int) -> None:
    _check(lib().flce_profile_start(int(n)), "flce_profile_start")


def flce_profile_stop(max_out: int = 1 << 16):
    """Return [(kernel name, milliseconds)] for the launches recorded."""
    ms = (ctypes.c_float * max_out)()
    kinds = (ctypes.c_int32 * max_out)()
    n = lib().flce_profile_stop(ms, kinds, max_out)
    if n < 0:
        raise FlceError(7, "flce_profile_stop")
    return [(flce_kernel_name(kinds[i]), float(ms[i])) for i in range(n)]


def flce_kernel_name(kind: int) -> str:
    return lib().flce_kernel_name(int(kind)).decode()


# ----------------------- convenience (allocates outputs) ----------------------

def _problem_of(X, W, ignore_index, softcap, shift_seq_len=0, dX=None, dW=None):
    """The problem of tensors X [BT, H] and W [V, H], their row strides
    included (rows must be unit-stride; dX, dW likewise when given)."""
    if X.dim() != 2 or W.dim() != 2 or X.shape[1] != W.shape[1]:
        raise ValueError("X must be [BT, H] and W [V, H], got %s and %s"
                         % (tuple(X.shape), tuple(W.shape)))
    if X.dtype != W.dtype or X.dtype not in _DTYPES:
        raise ValueError("X and W must both be bfloat16 or both float32 (got %s, %s)"
                         % (X.dtype, W.dtype))
    return make_problem(X.shape[0], X.shape[1], W.shape[0], X.dtype, ignore_index, softcap,
                        shift_seq_len, ldx=_row_stride(X), ldw=_row_stride(W),
                        lddx=_row_stride(dX) if dX is not None else 0,
                        lddw=_row_stride(dW) if dW is not None else 0,
                        dw_fp32=int(dW is not None and dW.dtype == torch.float32))


def _ws_for(n, device, where):
    if n == 0:
        raise FlceError(1, where)
    return torch.empty(n, dtype=torch.uint8, device=device)


def workspace(problem, op, device) -> torch.Tensor:
    return _ws_for(flce_workspace_size(problem, op), device, "flce_workspace_size")


def ce_workspace(problem, op, device) -> torch.Tensor:
    return _ws_for(flce_ce_workspace_size(problem, op), device, "flce_ce_workspace_size")


def forward(X, W, labels, ignore_index=-100, softcap=0.0, ws=None, stream=None,
            shift_seq_len=0):
    """Return (loss [1] fp32, lse [BT] fp32) computed by flce_forward."""
    p = _problem_of(X, W, ignore_index, softcap, shift_seq_len)
    ws = workspace(p, FLCE_OP_FORWARD, X.device) if ws is None else ws
    loss = torch.empty(1, dtype=torch.float32, device=X.device)
    lse = torch.empty(X.shape[0], dtype=torch.float32, device=X.device)
    flce_forward(p, X, W, labels, loss, lse, ws, stream)
    return loss, lse


def backward(X, W, labels, lse, dloss, ignore_index=-100, softcap=0.0, ws=None, stream=None,
             shift_seq_len=0):
    """Return (dX, dW) computed by flce_backward; dloss is a device fp32 tensor."""
    dX = torch.empty(X.shape, dtype=X.dtype, device=X.device)
    dW = torch.empty(W.shape, dtype=W.dtype, device=W.device)
    p = _problem_of(X, W, ignore_index, softcap, shift_seq_len, dX, dW)
    ws = workspace(p, FLCE_OP_BACKWARD, X.device) if ws is None else ws
    flce_backward(p, X, W, labels, lse, dloss, dX, dW, ws, stream)
    return dX, dW


def fused(X, W, labels, ignore_index=-100, softcap=0.0, dloss=1.0, ws=None, stream=None,
          n_valid_global=None, shift_seq_len=0, dX=None, dW=None, dw_fp32=False,
          slice_events=None):
    """Return (loss [1] fp32, dX, dW) computed by flce_fused, or by
    flce_fused_global when n_valid_global (device int64 [1]) is given.
    shift_seq_len = T > 0: labels are token ids of BT/T sequences and the op
    shifts them itself (position t scored against id t+1).  X and W may be
    row-strided views (e.g. a column slice of a wider tensor); dX, dW, when
    given, receive the gradients (row-strided views allowed), else dense
    tensors are allocated.  An fp32 dW (given, or dw_fp32=True) is written
    in fp32 whatever the input type.  slice_events (torch.cuda.Event list):
    through flce_fused_global_sliced, event s recorded once slice s of dW
    (dw_slice_bounds(V, len(slice_events))) is final."""
    dX = torch.empty(X.shape, dtype=X.dtype, device=X.device) if dX is None else dX
    if dW is None:
        dW = torch.empty(W.shape, dtype=torch.float32 if dw_fp32 else W.dtype, device=W.device)
    p = _problem_of(X, W, ignore_index, softcap, shift_seq_len, dX, dW)
    ws = workspace(p, FLCE_OP_FUSED, X.device) if ws is None else ws
    loss = torch.empty(1, dtype=torch.float32, device=X.device)
    if slice_events:
        flce_fused_global_sliced(p, X, W, labels, n_valid_global, dloss, loss, dX, dW, ws,
                                 slice_events, stream)
    elif n_valid_global is None:
        flce_fused(p, X, W, labels, dloss, loss, dX, dW, ws, stream)
    else:
        flce_fused_global(p, X, W, labels, n_valid_global, dloss, loss, dX, dW, ws, stream)
    return loss, dX, dW


def count_valid(X, W, labels, ignore_index=-100, stream=None, shift_seq_len=0) -> torch.Tensor:
    """Return a device int64 [1] tensor with the number of rows of the
    problem (X, W, labels) whose label is not ignored."""
    p = _problem_of(X, W, ignore_index, 0.0, shift_seq_len)
    n = torch.empty(1, dtype=torch.int64, device=labels.device)
    flce_count_valid(p, labels, n, stream)
    return n


def _ce_problem_of(logits, ignore_index, softcap, shift_seq_len, dlogits=None):
    if logits.dim() != 2 or logits.dtype not in _DTYPES:
        raise ValueError("logits must be a 2-D bfloat16 or float32 tensor, got %s %s"
                         % (logits.dtype, tuple(logits.shape)))
    return make_ce_problem(logits.shape[0], logits.shape[1], logits.dtype, ignore_index, softcap,
                           shift_seq_len, ld=_row_stride(logits),
                           ld_grad=_row_stride(dlogits) if dlogits is not None else 0)


def ce_forward(logits, labels, ignore_index=-100, softcap=0.0, ws=None, stream=None,
               shift_seq_len=0):
    """Return (loss [1] fp32, lse [BT] fp32) computed by flce_ce_forward from
    logits [BT, V] (a row-strided view is fine)."""
    p = _ce_problem_of(logits, ignore_index, softcap, shift_seq_len)
    ws = ce_workspace(p, FLCE_OP_FORWARD, logits.device) if ws is None else ws
    loss = torch.empty(1, dtype=torch.float32, device=logits.device)
    lse = torch.empty(logits.shape[0], dtype=torch.float32, device=logits.device)
    flce_ce_forward(p, logits, labels, loss, lse, ws, stream)
    return loss, lse


def ce_backward(logits, labels, lse, dloss, ignore_index=-100, softcap=0.0, ws=None,
                stream=None, shift_seq_len=0, out=None):
    """Return dlogits computed by flce_ce_backward; dloss is a device fp32
    [1] tensor.  out: where to write it (pass logits itself to overwrite
    the logits in place), else a new dense tensor."""
    out = torch.empty(logits.shape, dtype=logits.dtype, device=logits.device) if out is None \
        else out
    p = _ce_problem_of(logits, ignore_index, softcap, shift_seq_len, out)
    ws = ce_workspace(p, FLCE_OP_BACKWARD, logits.device) if ws is None else ws
    flce_ce_backward(p, logits, labels, lse, dloss, out, ws, stream)
    return out


def ce_fused(logits, labels, ignore_index=-100, softcap=0.0, dloss=1.0, ws=None, stream=None,
             shift_seq_len=0, out=None, want_lse=True):
    """Return (loss [1] fp32, lse [BT] fp32 or None, dlogits) computed by
    flce_ce_fused; out as in ce_backward (logits itself: in place)."""
    out = torch.empty(logits.shape, dtype=logits.dtype, device=logits.device) if out is None \
        else out
    p = _ce_problem_of(logits, ignore_index, softcap, shift_seq_len, out)
    ws = ce_workspace(p, FLCE_OP_FUSED, logits.device) if ws is None else ws
    loss = torch.empty(1, dtype=torch.float32, device=logits.device)
    lse = torch.empty(logits.shape[0], dtype=torch.float32, device=logits.device) \
        if want_lse else None
    flce_ce_fused(p, logits, labels, dloss, loss, lse, out, ws, stream)
    return loss, lse, out
