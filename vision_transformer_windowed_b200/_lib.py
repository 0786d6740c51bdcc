"""ctypes binding of the C ABI declared in include/fswin.h (argument marshalling only).

There is no fallback: if the compiled library is missing or fails to load, every
call raises.  Nothing here computes any part of the attention.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None

FS_OK, FS_ERR_NULL, FS_ERR_SHAPE, FS_ERR_ALIGN, FS_ERR_WORKSPACE, FS_ERR_CUDA, FS_ERR_TIMEOUT, FS_ERR_ARCH = range(8)
STATUS_NAMES = ["FS_OK", "FS_ERR_NULL", "FS_ERR_SHAPE", "FS_ERR_ALIGN", "FS_ERR_WORKSPACE", "FS_ERR_CUDA",
                "FS_ERR_TIMEOUT", "FS_ERR_ARCH"]


class FswinError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


class Shape(ctypes.Structure):
    """fs_winattn_shape"""
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "W", "heads", "d", "M", "s")]


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True):
    """Load libfswin.so (building it first when it is missing and nvcc exists)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            if not build_if_missing:
                raise FileNotFoundError(f"CUDA library not built: {path}")
            _build.build()
        lib = ctypes.CDLL(path)
        vp, P, st = ctypes.c_void_p, ctypes.POINTER(Shape), ctypes.c_int
        lib.fs_winattn_check_shape.argtypes = [P]
        lib.fs_winattn_check_shape.restype = st
        lib.fs_winattn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        lib.fs_winattn_fwd.restype = st
        lib.fs_winattn_block_fwd.argtypes = [P] + [vp] * 7 + [vp]
        lib.fs_winattn_block_fwd.restype = st
        lib.fs_winattn_bwd_workspace_bytes.argtypes = [P]
        lib.fs_winattn_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.fs_winattn_bwd.argtypes = [P] + [vp] * 12 + [ctypes.c_size_t, vp]
        lib.fs_winattn_bwd.restype = st
        lib.fs_status_string.argtypes = [st]
        lib.fs_status_string.restype = ctypes.c_char_p
        lib.fs_device_status.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        lib.fs_device_status.restype = st
        lib.fs_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.fs_set_wait_limit_ns.restype = st
        lib.fs_selftest_bounded_wait.argtypes = [ctypes.c_uint64, vp]
        lib.fs_selftest_bounded_wait.restype = st
        lib.fs_set_phase_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
        lib.fs_set_phase_events.restype = st
        lib.fs_winattn_bwd_noalloc.argtypes = [P] + [vp] * 12
        lib.fs_winattn_bwd_noalloc.restype = st
        lib.fs_winattn_bwd_noalloc_max_bytes.argtypes = []
        lib.fs_winattn_bwd_noalloc_max_bytes.restype = ctypes.c_size_t
        lib.fs_winattn_fwd_train.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        lib.fs_winattn_fwd_train.restype = st
        lib.fs_winattn_bwd_train.argtypes = [P] + [vp] * 12 + [ctypes.c_size_t, vp]
        lib.fs_winattn_bwd_train.restype = st
        lib.fs_winattn_lrbias_fwd.argtypes = [P] + [vp] * 6 + [ctypes.c_int, vp, vp, vp]
        lib.fs_winattn_lrbias_fwd.restype = st
        lib.fs_winattn_lrbias_bwd_workspace_bytes.argtypes = [P]
        lib.fs_winattn_lrbias_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.fs_winattn_lrbias_bwd.argtypes = [P] + [vp] * 9 + [ctypes.c_int] + [vp] * 7 + [ctypes.c_size_t, vp]
        lib.fs_winattn_lrbias_bwd.restype = st
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().fs_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != FS_OK:
        raise FswinError(status, what)


def make_shape(B: int, H: int, W: int, heads: int, d: int, M: int, s: int) -> Shape:
    return Shape(B, H, W, heads, d, M, s)


def fs_winattn_check_shape(shape: Shape) -> int:
    return load().fs_winattn_check_shape(ctypes.byref(shape))


def fs_winattn_fwd(shape: Shape, q: int, k: int, v: int, theta: int, o: int, lse: int, stream: int) -> None:
    _check(load().fs_winattn_fwd(ctypes.byref(shape), q, k, v, theta, o, lse, stream), "fs_winattn_fwd")


def fs_winattn_block_fwd(shape: Shape, x: int, w_qkv: int, b_qkv: int, w_o: int, b_o: int, theta: int, y: int,
                         stream: int) -> None:
    _check(load().fs_winattn_block_fwd(ctypes.byref(shape), x, w_qkv, b_qkv, w_o, b_o, theta, y, stream),
           "fs_winattn_block_fwd")


def fs_winattn_bwd_workspace_bytes(shape: Shape) -> int:
    return int(load().fs_winattn_bwd_workspace_bytes(ctypes.byref(shape)))


def fs_winattn_bwd(shape: Shape, q: int, k: int, v: int, o: int, dout: int, lse: int, theta: int, dq: int, dk: int,
                   dv: int, dtheta: int, workspace: int, workspace_bytes: int, stream: int) -> None:
    _check(load().fs_winattn_bwd(ctypes.byref(shape), q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta, workspace,
                                 workspace_bytes, stream), "fs_winattn_bwd")


def fs_winattn_fwd_train(shape: Shape, q: int, k: int, v: int, theta: int, o: int, lse: int, workspace: int,
                         workspace_bytes: int, stream: int) -> None:
    _check(load().fs_winattn_fwd_train(ctypes.byref(shape), q, k, v, theta, o, lse, workspace, workspace_bytes,
                                       stream), "fs_winattn_fwd_train")


def fs_winattn_bwd_train(shape: Shape, q: int, k: int, v: int, o: int, dout: int, lse: int, theta: int, dq: int,
                         dk: int, dv: int, dtheta: int, workspace: int, workspace_bytes: int, stream: int) -> None:
    _check(load().fs_winattn_bwd_train(ctypes.byref(shape), q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta,
                                       workspace, workspace_bytes, stream), "fs_winattn_bwd_train")


def fs_winattn_bwd_noalloc(shape: Shape, q: int, k: int, v: int, o: int, dout: int, lse: int, theta: int, dq: int,
                           dk: int, dv: int, dtheta: int, stream: int) -> None:
    """Backward without a caller workspace: for callers that cannot allocate
    device memory at that point; uses the library's own fixed scratch array."""
    _check(load().fs_winattn_bwd_noalloc(ctypes.byref(shape), q, k, v, o, dout, lse, theta, dq, dk, dv, dtheta,
                                         stream), "fs_winattn_bwd_noalloc")


def fs_winattn_bwd_noalloc_max_bytes() -> int:
    return int(load().fs_winattn_bwd_noalloc_max_bytes())


def fs_winattn_lrbias_fwd(shape: Shape, q: int, k: int, v: int, theta: int, u: int, w: int, rank: int, o: int,
                          lse: int, stream: int) -> None:
    _check(load().fs_winattn_lrbias_fwd(ctypes.byref(shape), q, k, v, theta, u, w, int(rank), o, lse, stream),
           "fs_winattn_lrbias_fwd")


def fs_winattn_lrbias_bwd_workspace_bytes(shape: Shape) -> int:
    return int(load().fs_winattn_lrbias_bwd_workspace_bytes(ctypes.byref(shape)))


def fs_winattn_lrbias_bwd(shape: Shape, q: int, k: int, v: int, o: int, dout: int, lse: int, theta: int, u: int,
                          w: int, rank: int, dq: int, dk: int, dv: int, dtheta: int, du: int, dw: int,
                          workspace: int, workspace_bytes: int, stream: int) -> None:
    _check(load().fs_winattn_lrbias_bwd(ctypes.byref(shape), q, k, v, o, dout, lse, theta, u, w, int(rank), dq, dk,
                                        dv, dtheta, du, dw, workspace, workspace_bytes, stream),
           "fs_winattn_lrbias_bwd")


def fs_device_status() -> int:
    code = ctypes.c_uint(0)
    _check(load().fs_device_status(ctypes.byref(code)), "fs_device_status")
    return int(code.value)


def fs_set_wait_limit_ns(limit_ns: int) -> None:
    _check(load().fs_set_wait_limit_ns(int(limit_ns)), "fs_set_wait_limit_ns")


def fs_set_phase_events(event_handles) -> None:
    """event_handles: raw cudaEvent_t values (e.g. torch.cuda.Event().cuda_event), or [] to switch off."""
    n = len(event_handles)
    arr = (ctypes.c_void_p * max(n, 1))(*[int(e) for e in event_handles])
    _check(load().fs_set_phase_events(arr if n else None, n), "fs_set_phase_events")


def fs_selftest_bounded_wait(limit_ns: int, stream: int) -> None:
    _check(load().fs_selftest_bounded_wait(int(limit_ns), stream), "fs_selftest_bounded_wait")
