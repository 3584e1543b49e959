"""B200-native 2D (dilated) neighborhood attention -- Python binding of libna2d.

The four calls mirror the C ABI in ``include/na2d.h`` and take torch CUDA
tensors (torch provides device memory and streams only; the computation runs
in the library's sm_100a kernels):

    na2d_qk_rpb(q, k, rpb, kernel_size, dilation)        -> attn  [B,heads,H,W,k*k] fp32
    na2d_softmax(attn, kernel_size, dilation)            -> attn  (in place)
    na2d_av(attn, v, kernel_size, dilation)              -> out   [B,heads,H,W,D]
    na2d_forward(q, k, v, rpb, kernel_size, dilation)    -> out   (fused)
    na2d_backward(q, k, v, rpb, dout, kernel_size, dilation) -> (dq, dk, dv, drpb)
    na2d(q, k, v, rpb, kernel_size, dilation)            -> out   (autograd: backward via na2d_backward)
    na2d_forward_ex(q, k, v, rpb, kernel_size, dilation, return_attn=, dropout_p=, seed=)
                                                         -> out [, attn]  (strided views, weights, dropout)
    na2d_backward_ex(q, k, v, rpb, dout, ...)            -> (dq, dk, dv, drpb)  (strided views, dropout)
    na2d_qkv_packed(qkv, rpb, kernel_size, dilation, heads) -> out (B, H, W, heads*D), read in place

q, k, v are [B, heads, H, W, D] tensors (D in 16, 32, 64, 128) in float32,
float16 or bfloat16 on one CUDA device -- contiguous for the plain calls, any
strides with contiguous channels for the _ex calls; rpb is [heads, 2k-1, 2k-1]
in the same dtype, or None.  Maps shorter than k*d are zero-padded at the
bottom/right and cropped, as the DiNAT layer does.  Calls are asynchronous on
the current torch stream.  A non-OK status from the library raises
``Na2dError``; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes

from ._native import (Dropout, Na2dError, Problem, Tensor, backward_workspace_size, check, device_faults, lib,  # noqa: F401
                      status_str)

__all__ = ["na2d_qk_rpb", "na2d_softmax", "na2d_av", "na2d_forward", "na2d_status_str", "na2d_device_faults",
           "na2d_last_kernel", "na2d_backward", "na2d", "na2d_forward_ex", "na2d_backward_ex", "na2d_qkv_packed",
           "na2d_forward_host", "na2d_forward_host_workspace_size", "Na2dError", "make_problem"]

# status codes used for argument errors raised before the library is called
_ERR_NULL, _ERR_DTYPE, _ERR_SHAPE = 1, 2, 3


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
        raise Na2dError(_ERR_NULL, "device", "tensors must be CUDA tensors (there is no CPU path)")
    if not t.is_contiguous():
        raise Na2dError(_ERR_SHAPE, "layout", "tensors must be contiguous")
    return t.data_ptr()


def _like(name: str, t, ref, shape=None, dtype=None) -> None:
    """Checks on the host that tensor `t` has the given shape (default: ref's),
    dtype (default: ref's) and ref's device; the library receives raw pointers
    and could not detect a mismatch, so a short or foreign buffer is refused
    here, before any launch."""
    if t is None:
        raise Na2dError(_ERR_NULL, name, f"{name} is required")
    want_shape = tuple(ref.shape) if shape is None else tuple(shape)
    want_dtype = ref.dtype if dtype is None else dtype
    if t.dim() != len(want_shape) or tuple(t.shape) != want_shape:
        raise Na2dError(_ERR_SHAPE, name, f"{name} has shape {tuple(t.shape)}, expected {want_shape}")
    if t.dtype != want_dtype:
        raise Na2dError(_ERR_DTYPE, name, f"{name} is {t.dtype}, expected {want_dtype}")
    if t.device != ref.device:
        raise Na2dError(_ERR_NULL, name, f"{name} is on {t.device}, expected {ref.device}")


def _check_qkv(q, kernel_size: int) -> None:
    if q.dim() != 5:
        raise Na2dError(_ERR_SHAPE, "q", f"q must be [B, heads, H, W, D], got shape {tuple(q.shape)}")


def _check_rpb(rpb, q, kernel_size: int) -> None:
    if rpb is None:
        return
    nb = 2 * kernel_size - 1
    _like("rpb", rpb, q, shape=(q.shape[1], nb, nb))


def _attn_shape(x, kernel_size: int):
    return tuple(x.shape[:4]) + (kernel_size * kernel_size,)


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


def na2d_last_kernel() -> str | None:
    """Name of the kernel that this thread's last na2d_forward call launched
    (None if it launched nothing)."""
    r = lib().na2d_last_kernel()
    return r.decode() if r else None


def na2d_forward(q, k, v, rpb, kernel_size: int, dilation: int = 1, out=None):
    """Fused forward: softmax(q.k/sqrt(D) + rpb) . v over each query's window."""
    _check_qkv(q, kernel_size)
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    _like("k", k, q)
    _like("v", v, q)
    _check_rpb(rpb, q, kernel_size)
    if out is None:
        out = _torch().empty_like(q)
    _like("out", out, q)
    ptrs = (_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out))
    with _torch().cuda.device(q.device):
        check(lib().na2d_forward(p, *ptrs, _stream(q)), "na2d_forward")
    return out


def na2d_forward_host_workspace_size(shape, kernel_size: int, dilation: int = 1, dtype=None) -> int:
    """Bytes of device workspace na2d_forward_host needs for a [B, heads, H, W, D]
    problem of the given dtype."""
    p = make_problem(tuple(shape), kernel_size, dilation, dtype or _torch().float16)
    n = ctypes.c_size_t(0)
    check(lib().na2d_forward_host_workspace_size(p, ctypes.byref(n)), "na2d_forward_host_workspace_size")
    return n.value


def na2d_forward_host(q, k, v, rpb, kernel_size: int, dilation: int = 1, out=None, workspace=None, device=None):
    """na2d_forward on host (CPU) tensors: the library copies the batch to the
    GPU in chunks, runs the forward and copies the output back, overlapping
    the copies with the kernels.  q, k, v, rpb and out should be pinned
    (``pin_memory()``); out is allocated pinned when not given.  workspace: a
    CUDA uint8 tensor of at least na2d_forward_host_workspace_size() bytes,
    allocated here when not given.  Asynchronous: out holds the result once
    the device's current stream has passed this call."""
    torch = _torch()
    _check_qkv(q, kernel_size)
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    for name, t in (("q", q), ("k", k), ("v", v), ("rpb", rpb), ("out", out)):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise Na2dError(_ERR_NULL, name, f"{name} must be a contiguous host (CPU) tensor")
    _like("k", k, q)
    _like("v", v, q)
    _check_rpb(rpb, q, kernel_size)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    _like("out", out, q)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    need = na2d_forward_host_workspace_size(q.shape, kernel_size, dilation, q.dtype)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    if not workspace.is_cuda or workspace.device != dev or not workspace.is_contiguous():
        raise Na2dError(_ERR_NULL, "workspace", f"workspace must be a contiguous CUDA tensor on {dev}")
    nbytes = workspace.numel() * workspace.element_size()
    host = [None if t is None else t.data_ptr() for t in (q, k, v, rpb, out)]
    with torch.cuda.device(dev):
        st = torch.cuda.current_stream(dev).cuda_stream
        check(lib().na2d_forward_host(p, *host, workspace.data_ptr(), nbytes, st), "na2d_forward_host")
    return out


def na2d_qk_rpb(q, k, rpb, kernel_size: int, dilation: int = 1, attn=None):
    """Scores (fp32): q.k/sqrt(D) + rpb for each query's k*k neighbours."""
    _check_qkv(q, kernel_size)
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    _like("k", k, q)
    _check_rpb(rpb, q, kernel_size)
    if attn is None:
        attn = _torch().empty(_attn_shape(q, kernel_size), dtype=_torch().float32, device=q.device)
    _like("attn", attn, q, shape=_attn_shape(q, kernel_size), dtype=_torch().float32)
    ptrs = (_ptr(q), _ptr(k), _ptr(rpb), _ptr(attn))
    with _torch().cuda.device(q.device):
        check(lib().na2d_qk_rpb(p, *ptrs, _stream(q)), "na2d_qk_rpb")
    return attn


def na2d_softmax(attn, kernel_size: int, dilation: int = 1, D: int = 32, dtype=None):
    """In-place softmax over the last (k*k) axis of an fp32 score tensor."""
    if attn.dim() != 5 or attn.shape[4] != kernel_size * kernel_size:
        raise Na2dError(_ERR_SHAPE, "attn", f"attn must be [B, heads, H, W, {kernel_size * kernel_size}], "
                        f"got {tuple(attn.shape)}")
    if attn.dtype != _torch().float32:
        raise Na2dError(_ERR_DTYPE, "attn", f"attn must be float32, got {attn.dtype}")
    B, heads, H, W, _ = attn.shape
    p = make_problem((B, heads, H, W, D), kernel_size, dilation, dtype or _torch().float32)
    ptr = _ptr(attn)
    with _torch().cuda.device(attn.device):
        check(lib().na2d_softmax(p, ptr, _stream(attn)), "na2d_softmax")
    return attn


def na2d_av(attn, v, kernel_size: int, dilation: int = 1, out=None):
    """Weighted sum of values: out = sum_n attn[..., n] * v[key_n]."""
    _check_qkv(v, kernel_size)
    p = make_problem(v.shape, kernel_size, dilation, v.dtype)
    _like("attn", attn, v, shape=_attn_shape(v, kernel_size), dtype=_torch().float32)
    if out is None:
        out = _torch().empty_like(v)
    _like("out", out, v)
    ptrs = (_ptr(attn), _ptr(v), _ptr(out))
    with _torch().cuda.device(v.device):
        check(lib().na2d_av(p, *ptrs, _stream(v)), "na2d_av")
    return out


def na2d_backward(q, k, v, rpb, dout, kernel_size: int, dilation: int = 1, dq=None, dk=None, dv=None, drpb=None,
                  workspace=None):
    """Gradients (dq, dk, dv, drpb) of na2d_forward for the output gradient
    dout; drpb is None when rpb is None.  The fp32 workspace is allocated with
    torch unless given (a uint8 CUDA tensor of at least
    backward_workspace_size bytes)."""
    torch = _torch()
    _check_qkv(q, kernel_size)
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    for name, t in (("k", k), ("v", v), ("dout", dout)):
        _like(name, t, q)
    _check_rpb(rpb, q, kernel_size)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _like(name, t, q)
    if rpb is not None and drpb is None:
        drpb = torch.empty_like(rpb)
    if drpb is not None:
        _check_rpb(drpb, q, kernel_size)
    need = backward_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if workspace.device != q.device:
        raise Na2dError(_ERR_NULL, "workspace", f"workspace is on {workspace.device}, expected {q.device}")
    nbytes = workspace.numel() * workspace.element_size()
    ptrs = (_ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(drpb),
            _ptr(workspace))
    with torch.cuda.device(q.device):
        check(lib().na2d_backward(p, *ptrs, nbytes, _stream(q)), "na2d_backward")
    return dq, dk, dv, drpb


def _autograd_function():
    torch = _torch()

    class _NA2D(torch.autograd.Function):
        """Autograd wrapper: forward = na2d_forward, backward = na2d_backward
        (both in the library's kernels)."""

        @staticmethod
        def forward(ctx, q, k, v, rpb, kernel_size, dilation, dropout_p, seed):
            rpb = None if rpb is None else rpb.contiguous()
            ctx.save_for_backward(q, k, v, rpb)
            ctx.kd = (kernel_size, dilation)
            ctx.drop = (dropout_p, seed)
            if dropout_p:
                return na2d_forward_ex(q, k, v, rpb, kernel_size, dilation, dropout_p=dropout_p, seed=seed)
            q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
            return na2d_forward(q, k, v, rpb, kernel_size, dilation)

        @staticmethod
        def backward(ctx, dout):
            q, k, v, rpb = ctx.saved_tensors
            p, seed = ctx.drop
            if p or not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
                dq, dk, dv, drpb = na2d_backward_ex(q, k, v, rpb, dout, *ctx.kd, dropout_p=p, seed=seed)
            else:
                dq, dk, dv, drpb = na2d_backward(q, k, v, rpb, dout.contiguous(), *ctx.kd)
            return dq, dk, dv, drpb, None, None, None, None

    return _NA2D


_NA2D = None


def na2d(q, k, v, rpb, kernel_size: int, dilation: int = 1, dropout_p: float = 0.0, seed: int | None = None):
    """Differentiable neighborhood attention (forward and backward in the
    library's kernels), for training with torch autograd.  With dropout_p > 0
    the Philox seed is drawn from torch's CPU generator unless given; the
    backward reproduces the same mask."""
    global _NA2D
    if _NA2D is None:
        _NA2D = _autograd_function()
    if dropout_p and seed is None:
        seed = int(_torch().randint(0, 2 ** 62, (1,)).item())
    return _NA2D.apply(q, k, v, rpb, kernel_size, dilation, float(dropout_p), int(seed or 0))


# ---------------------------------------------------------------------------
# Strided views, attention weights, dropout.
def _view(name: str, t, ref_shape, dtype, device) -> Tensor:
    """An na2d_tensor for a [B, heads, H, W, D] torch tensor with contiguous
    channels (any other strides); shape, dtype and device are checked here."""
    if t is None:
        raise Na2dError(_ERR_NULL, name, f"{name} is required")
    if tuple(t.shape) != tuple(ref_shape):
        raise Na2dError(_ERR_SHAPE, name, f"{name} has shape {tuple(t.shape)}, expected {tuple(ref_shape)}")
    if t.dtype != dtype:
        raise Na2dError(_ERR_DTYPE, name, f"{name} is {t.dtype}, expected {dtype}")
    if not t.is_cuda or t.device != device:
        raise Na2dError(_ERR_NULL, name, f"{name} must be on {device}")
    if t.stride(4) != 1:
        raise Na2dError(_ERR_SHAPE, name, f"{name} must have contiguous channels (stride 1 on the last dim)")
    sb, sh, sy, sx, _ = t.stride()
    return Tensor(t.data_ptr(), sb, sh, sy, sx)


def _dropout(p: float, seed: int, offset: int):
    if not p:
        return None
    return Dropout(float(p), int(seed) & ((1 << 64) - 1), int(offset) & ((1 << 64) - 1))


def na2d_forward_ex(q, k, v, rpb, kernel_size: int, dilation: int = 1, out=None, return_attn: bool = False,
                    dropout_p: float = 0.0, seed: int = 0, offset: int = 0):
    """Forward on strided tensors (e.g. channels-last views), optionally
    returning the attention weights [B, heads, H, W, k*k] (fp32, after
    dropout) and applying attention dropout (Philox, seed/offset)."""
    import ctypes
    torch = _torch()
    _check_qkv(q, kernel_size)
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    _check_rpb(rpb, q, kernel_size)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=q.device)
    views = [_view(n, t, q.shape, q.dtype, q.device) for n, t in (("q", q), ("k", k), ("v", v), ("out", out))]
    attn = None
    if return_attn:
        attn = torch.empty(_attn_shape(q, kernel_size), dtype=torch.float32, device=q.device)
    dr = _dropout(dropout_p, seed, offset)
    with torch.cuda.device(q.device):
        check(lib().na2d_forward_ex(p, *[ctypes.byref(x) for x in views[:3]], _ptr(rpb), ctypes.byref(views[3]),
                                    None if attn is None else attn.data_ptr(),
                                    None if dr is None else ctypes.byref(dr), _stream(q)), "na2d_forward_ex")
    return (out, attn) if return_attn else out


def na2d_backward_ex(q, k, v, rpb, dout, kernel_size: int, dilation: int = 1, dq=None, dk=None, dv=None,
                     drpb=None, dropout_p: float = 0.0, seed: int = 0, offset: int = 0, workspace=None):
    """Backward on strided tensors with the forward's dropout mask (same
    dropout_p, seed, offset); returns (dq, dk, dv, drpb)."""
    import ctypes
    torch = _torch()
    _check_qkv(q, kernel_size)
    p = make_problem(q.shape, kernel_size, dilation, q.dtype)
    _check_rpb(rpb, q, kernel_size)
    dq = torch.empty(q.shape, dtype=q.dtype, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=q.dtype, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=q.dtype, device=q.device) if dv is None else dv
    if rpb is not None and drpb is None:
        drpb = torch.empty_like(rpb)
    if drpb is not None:
        _check_rpb(drpb, q, kernel_size)
    views = [_view(n, t, q.shape, q.dtype, q.device)
             for n, t in (("q", q), ("k", k), ("v", v), ("dout", dout), ("dq", dq), ("dk", dk), ("dv", dv))]
    need = backward_workspace_size(p)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dr = _dropout(dropout_p, seed, offset)
    with torch.cuda.device(q.device):
        check(lib().na2d_backward_ex(p, *[ctypes.byref(x) for x in views[:3]], _ptr(rpb), ctypes.byref(views[3]),
                                     *[ctypes.byref(x) for x in views[4:]], _ptr(drpb),
                                     None if dr is None else ctypes.byref(dr), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(q)), "na2d_backward_ex")
    return dq, dk, dv, drpb


def qkv_views(qkv, heads: int):
    """q, k, v as [B, heads, H, W, D] views of a channels-last fused
    projection output (B, H, W, 3 * heads * D), ordered (3, heads, D) along
    the channels.  No data moves."""
    B, H, W, C = qkv.shape
    if C % (3 * heads):
        raise Na2dError(_ERR_SHAPE, "qkv", f"channels {C} are not 3 * heads * D for heads={heads}")
    D = C // (3 * heads)
    x = qkv.view(B, H, W, 3, heads, D).permute(3, 0, 4, 1, 2, 5)
    return x[0], x[1], x[2]


def na2d_qkv_packed(qkv, rpb, kernel_size: int, dilation: int, heads: int, out=None):
    """Neighborhood attention read straight from a channels-last fused q/k/v
    projection (B, H, W, 3 * heads * D); writes and returns the channels-last
    output (B, H, W, heads * D) (no permute copies on either side)."""
    torch = _torch()
    q, k, v = qkv_views(qkv, heads)
    B, H, W, C = qkv.shape
    D = C // (3 * heads)
    if out is None:
        out = torch.empty(B, H, W, heads * D, dtype=qkv.dtype, device=qkv.device)
    if tuple(out.shape) != (B, H, W, heads * D) or not out.is_contiguous():
        raise Na2dError(_ERR_SHAPE, "out", f"out must be a contiguous ({B}, {H}, {W}, {heads * D}) tensor")
    ov = out.view(B, H, W, heads, D).permute(0, 3, 1, 2, 4)
    na2d_forward_ex(q, k, v, rpb, kernel_size, dilation, out=ov)
    return out
