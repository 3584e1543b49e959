"""ctypes view of ``libna2d.so`` -- the C ABI declared in ``include/na2d.h``.

Marshalling only: structures, prototypes and the status type.  Every step of
the computation runs in the library's CUDA kernels; nothing here computes.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

LIB_PATH = Path(__file__).resolve().parent / "libna2d.so"

NA2D_F32, NA2D_F16, NA2D_BF16 = 0, 1, 2

STATUS_NAMES = {
    0: "NA2D_OK", 1: "NA2D_ERR_NULL", 2: "NA2D_ERR_DTYPE", 3: "NA2D_ERR_SHAPE", 4: "NA2D_ERR_KERNEL",
    5: "NA2D_ERR_DILATION", 6: "NA2D_ERR_ALIGN", 7: "NA2D_ERR_ALIAS", 8: "NA2D_ERR_CUDA", 9: "NA2D_ERR_INTERNAL",
}

# every symbol the header declares
EXPORTS = ("na2d_qk_rpb", "na2d_softmax", "na2d_av", "na2d_forward", "na2d_device_faults", "na2d_status_str",
           "na2d_version", "na2d_last_kernel", "na2d_backward_workspace_size", "na2d_backward",
           "na2d_backward_noalloc", "na2d_forward_ex", "na2d_backward_ex", "na2d_debug_set_wait_limit",
           "na2d_forward_host_workspace_size", "na2d_forward_host")


class Problem(ctypes.Structure):
    """``na2d_problem``: one problem description (scale fixed at 1/sqrt(D))."""
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("D", ctypes.c_int), ("k", ctypes.c_int), ("d", ctypes.c_int), ("dtype", ctypes.c_int)]


class Tensor(ctypes.Structure):
    """``na2d_tensor``: data pointer and element strides (b, head, y, x)."""
    _fields_ = [("data", ctypes.c_void_p), ("stride_b", ctypes.c_longlong), ("stride_h", ctypes.c_longlong),
                ("stride_y", ctypes.c_longlong), ("stride_x", ctypes.c_longlong)]


class Dropout(ctypes.Structure):
    """``na2d_dropout``: probability, Philox key and counter offset."""
    _fields_ = [("p", ctypes.c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_ulonglong)]


class Na2dError(RuntimeError):
    """A non-OK ``na2d_status`` returned by the library."""

    def __init__(self, status: int, what: str, message: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({message})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it has not been built: there is no
    fallback implementation."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m neighborhood_attention_na2d_b200.build`")
        L = ctypes.CDLL(str(LIB_PATH))
        P, vp, fp = ctypes.POINTER(Problem), ctypes.c_void_p, ctypes.c_void_p
        L.na2d_qk_rpb.argtypes = [P, vp, vp, vp, fp, vp]
        L.na2d_softmax.argtypes = [P, fp, vp]
        L.na2d_av.argtypes = [P, fp, vp, vp, vp]
        L.na2d_forward.argtypes = [P, vp, vp, vp, vp, vp, vp]
        for f in ("na2d_qk_rpb", "na2d_softmax", "na2d_av", "na2d_forward"):
            getattr(L, f).restype = ctypes.c_int
        L.na2d_device_faults.argtypes = [ctypes.POINTER(ctypes.c_uint), vp]
        L.na2d_device_faults.restype = ctypes.c_int
        L.na2d_status_str.argtypes = [ctypes.c_int]
        L.na2d_status_str.restype = ctypes.c_char_p
        L.na2d_version.argtypes = []
        L.na2d_version.restype = ctypes.c_int
        L.na2d_backward_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
        L.na2d_backward_workspace_size.restype = ctypes.c_int
        L.na2d_backward.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.na2d_backward.restype = ctypes.c_int
        L.na2d_backward_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.na2d_backward_noalloc.restype = ctypes.c_int
        TP, DP = ctypes.POINTER(Tensor), ctypes.POINTER(Dropout)
        L.na2d_forward_ex.argtypes = [P, TP, TP, TP, vp, TP, fp, DP, vp]
        L.na2d_forward_ex.restype = ctypes.c_int
        L.na2d_backward_ex.argtypes = [P, TP, TP, TP, vp, TP, TP, TP, TP, vp, DP, vp, ctypes.c_size_t, vp]
        L.na2d_backward_ex.restype = ctypes.c_int
        L.na2d_forward_host_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
        L.na2d_forward_host_workspace_size.restype = ctypes.c_int
        L.na2d_forward_host.argtypes = [P, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        L.na2d_forward_host.restype = ctypes.c_int
        L.na2d_debug_set_wait_limit.argtypes = [ctypes.c_longlong]
        L.na2d_debug_set_wait_limit.restype = None
        L.na2d_last_kernel.argtypes = []
        L.na2d_last_kernel.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().na2d_status_str(status).decode()


def check(status: int, what: str) -> None:
    if status != 0:
        raise Na2dError(status, what, status_str(status))


# Raw-pointer calls (integers are device addresses; stream is a cudaStream_t
# handle as an int, 0 for the legacy default stream).  They return the status.
def forward_ptr(p: Problem, q: int, k: int, v: int, rpb: int | None, out: int, stream: int = 0) -> int:
    return lib().na2d_forward(ctypes.byref(p), q, k, v, rpb, out, stream)


def qk_rpb_ptr(p: Problem, q: int, k: int, rpb: int | None, attn: int, stream: int = 0) -> int:
    return lib().na2d_qk_rpb(ctypes.byref(p), q, k, rpb, attn, stream)


def softmax_ptr(p: Problem, attn: int, stream: int = 0) -> int:
    return lib().na2d_softmax(ctypes.byref(p), attn, stream)


def av_ptr(p: Problem, attn: int, v: int, out: int, stream: int = 0) -> int:
    return lib().na2d_av(ctypes.byref(p), attn, v, out, stream)


def backward_workspace_size(p: Problem) -> int:
    n = ctypes.c_size_t(0)
    check(lib().na2d_backward_workspace_size(ctypes.byref(p), ctypes.byref(n)), "na2d_backward_workspace_size")
    return n.value


def backward_ptr(p: Problem, q: int, k: int, v: int, rpb: int | None, dout: int, dq: int, dk: int, dv: int,
                 drpb: int | None, workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return lib().na2d_backward(ctypes.byref(p), q, k, v, rpb, dout, dq, dk, dv, drpb, workspace, workspace_bytes,
                               stream)


def backward_noalloc_ptr(p: Problem, q: int, k: int, v: int, rpb: int | None, dout: int, dq: int, dk: int, dv: int,
                         drpb: int | None, stream: int = 0) -> int:
    """na2d_backward with the library's built-in scratch (no workspace)."""
    return lib().na2d_backward_noalloc(ctypes.byref(p), q, k, v, rpb, dout, dq, dk, dv, drpb, stream)


def device_faults(stream: int = 0) -> int:
    """Reads and clears the device's count of timed-out bounded waits."""
    c = ctypes.c_uint(0)
    check(lib().na2d_device_faults(ctypes.byref(c), stream), "na2d_device_faults")
    return c.value
