"""B200-native 2D (dilated) neighborhood attention -- Python binding of libna2d.

The four calls mirror the C ABI in ``include/na2d.h`` and take torch CUDA
tensors (torch provides device memory and streams only; the computation runs
in the library's sm_100a kernels):

    na2d_qk_rpb(q, k, rpb, kernel_size, dilation)        -> attn  [B,heads,H,W,k*k] fp32
    na2d_softmax(attn, kernel_size, dilation)            -> attn  (in place)
    na2d_av(attn, v, kernel_size, dilation)              -> out   [B,heads,H,W,D]
    na2d_forward(q, k, v, rpb, kernel_size, dilation)    -> out   (fused)

q, k, v are contiguous [B, heads, H, W, D] tensors in float32, float16 or
bfloat16 on one CUDA device; rpb is [heads, 2k-1, 2k-1] in the same dtype, or
None.  Calls are asynchronous on the current torch stream.  A non-OK status
from the library raises ``Na2dError``; there is no CPU fallback.
"""
from __future__ import annotations

from ._native import Na2dError, Problem, check, device_faults, lib, status_str  # noqa: F401

__all__ = ["na2d_qk_rpb", "na2d_softmax", "na2d_av", "na2d_forward", "na2d_status_str", "na2d_device_faults",
           "Na2dError", "make_problem"]


def _torch():
    import torch
    return torch


def _dtype_code(dtype) -> int:
    torch = _torch()
    codes = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
    if dtype not in codes:
        raise Na2dError(2, "dtype", f"{dtype} is not float32, float16 or bfloat16")
    return codes[dtype]


def make_problem(shape, kernel_size: int, dilation: int, dtype) -> Problem:
    B, heads, H, W, D = shape
    return Problem(B, heads, H, W, D, kernel_size, dilation, _dtype_code(dtype))


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise Na2dError(1, "device", "tensors must be CUDA tensors (there is no CPU path)")
    if not t.is_contiguous():
        raise Na2dError(3, "layout", "tensors must be contiguous")
    return t.data_ptr()


def _stream(t) -> int:
    return _torch().cuda.current_stream(t.device).cuda_stream


def na2d_status_str(status: int) -> str:
    return status_str(status)


def na2d_device_faults(device=None) -> int:
    """Count of device-side bounded waits that timed out since the last call
    (synchronises the current stream); zero unless the library has a bug."""
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return device_faults(torch.cuda.current_stream(dev).cuda_stream)


def na2d_forward(q, k, v, rpb, kernel_size: int, dilation: int = 1, out=None):
    """Fused forward: softmax(q.k/sqrt(D) + rpb) . v over each query's window."""
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    if out is None:
        out = _torch().empty_like(q)
    ptrs = (_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out))
    with _torch().cuda.device(q.device):
        check(lib().na2d_forward(p, *ptrs, _stream(q)), "na2d_forward")
    return out


def na2d_qk_rpb(q, k, rpb, kernel_size: int, dilation: int = 1, attn=None):
    """Scores (fp32): q.k/sqrt(D) + rpb for each query's k*k neighbours."""
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    if attn is None:
        attn = _torch().empty(tuple(q.shape[:4]) + (kernel_size * kernel_size,), dtype=_torch().float32,
                              device=q.device)
    ptrs = (_ptr(q), _ptr(k), _ptr(rpb), _ptr(attn))
    with _torch().cuda.device(q.device):
        check(lib().na2d_qk_rpb(p, *ptrs, _stream(q)), "na2d_qk_rpb")
    return attn


def na2d_softmax(attn, kernel_size: int, dilation: int = 1, D: int = 32, dtype=None):
    """In-place softmax over the last (k*k) axis of an fp32 score tensor."""
    B, heads, H, W, _ = attn.shape
    p = make_problem((B, heads, H, W, D), kernel_size, dilation, dtype or _torch().float32)
    ptr = _ptr(attn)
    with _torch().cuda.device(attn.device):
        check(lib().na2d_softmax(p, ptr, _stream(attn)), "na2d_softmax")
    return attn


def na2d_av(attn, v, kernel_size: int, dilation: int = 1, out=None):
    """Weighted sum of values: out = sum_n attn[..., n] * v[key_n]."""
    p = make_problem(v.shape, kernel_size, dilation, v.dtype)
    if out is None:
        out = _torch().empty_like(v)
    ptrs = (_ptr(attn), _ptr(v), _ptr(out))
    with _torch().cuda.device(v.device):
        check(lib().na2d_av(p, *ptrs, _stream(v)), "na2d_av")
    return out
