"""fp64 CPU oracle for 2D (dilated) neighborhood attention -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its Python
binding) never imports it and shares no code with it.

The arithmetic lives in ``na2d_oracle.c`` (plain C, fp64, no tiling); this module
compiles it with gcc and marshals numpy arrays.  See that file's header for the
definition it follows:

* "Dilated Neighborhood Attention Transformer" (gitcode DiNAT article, section
  "DiNAT 的核心思想"): scores from ``natten2dqkrpb``, ``softmax(dim=-1)``, then
  ``natten2dav`` -- the three stages exported here as ``qk_rpb``, ``softmax``
  and ``av``, and composed in ``forward``.
* "Neighborhood Attention Transformer" (README mirror, figure caption): nearest
  neighbourhood, full self attention when the window covers the image, edges as
  special cases.  The exact clamp rule is the NATTEN rule of the problem
  statement (see ``axis_neighbors``).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, a brute-force search formulation, invariants and the pages' stage table;
``tests/test_oracle_mutants.py`` shows that plausible mistakes planted in a copy
of the C source fail those pins.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
SOURCE = _HERE / "na2d_oracle.c"
LIB_PATH = _HERE / "libna2d_oracle.so"

_DP = ctypes.POINTER(ctypes.c_double)


def compile_c(src: Path, out: Path) -> Path:
    """gcc -O2 a copy of the oracle source into a shared library."""
    tmp = out.with_name(out.name + f".tmp{os.getpid()}")
    cmd = ["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", str(tmp), str(src), "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> Path:
    """Compile the C oracle into ``oracle/libna2d_oracle.so``."""
    if force or not LIB_PATH.exists() or LIB_PATH.stat().st_mtime < SOURCE.stat().st_mtime:
        compile_c(SOURCE, LIB_PATH)
    return LIB_PATH


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return _DP()
    return a.ctypes.data_as(_DP)


def _shape(q: np.ndarray, kernel_size: int, dilation: int):
    if q.ndim != 5:
        raise ValueError("expected [B, heads, H, W, D]")
    B, heads, H, W, D = q.shape
    return B, heads, H, W, D, kernel_size, dilation


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid shape (some dilation group shorter than k?)")


class Oracle:
    """The oracle functions bound to one compiled copy of ``na2d_oracle.c``."""

    def __init__(self, lib_path: Path | str):
        lib = ctypes.CDLL(str(lib_path))
        i, ip = ctypes.c_int, ctypes.POINTER(ctypes.c_int)
        lib.oracle_axis_window.argtypes = [i, i, i, i, ip, ip, ip]
        lib.oracle_axis_neighbors.argtypes = [i, i, i, i, ip, ip]
        lib.oracle_na2d_qk_rpb.argtypes = [i] * 7 + [_DP, _DP, _DP, _DP, i]
        lib.oracle_na2d_softmax.argtypes = [i] * 7 + [_DP, i]
        lib.oracle_na2d_av.argtypes = [i] * 7 + [_DP, _DP, _DP, i]
        lib.oracle_na2d_forward.argtypes = [i] * 7 + [_DP, _DP, _DP, _DP, _DP, i]
        lib.oracle_na2d_backward.argtypes = [i] * 7 + [_DP] * 9 + [i]
        u64, f64 = ctypes.c_ulonglong, ctypes.c_double
        lib.oracle_na2d_forward_ex.argtypes = [i] * 7 + [_DP] * 6 + [f64, u64, u64, i, i]
        lib.oracle_na2d_backward_ex.argtypes = [i] * 7 + [_DP] * 9 + [f64, u64, u64, i, i]
        lib.oracle_philox4x32_10.argtypes = [ctypes.POINTER(ctypes.c_uint)] * 3
        lib.oracle_philox4x32_10.restype = None
        for f in ("oracle_axis_window", "oracle_axis_neighbors", "oracle_na2d_qk_rpb",
                  "oracle_na2d_softmax", "oracle_na2d_av", "oracle_na2d_forward", "oracle_na2d_backward",
                  "oracle_na2d_forward_ex", "oracle_na2d_backward_ex"):
            getattr(lib, f).restype = ctypes.c_int
        self._lib = lib

    # -- the window rule -------------------------------------------------
    def axis_window(self, L: int, k: int, d: int, i: int) -> tuple[int, int, int]:
        """(g, i', s') of coordinate i on an axis of length L (NATTEN clamp rule)."""
        g, ip, s = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        if self._lib.oracle_axis_window(L, k, d, i, ctypes.byref(g), ctypes.byref(ip), ctypes.byref(s)) != 0:
            raise ValueError(f"no window: L={L} k={k} d={d} i={i}")
        return g.value, ip.value, s.value

    def axis_neighbors(self, L: int, k: int, d: int, i: int) -> tuple[list[int], list[int]]:
        """Key coordinates g + d(s'+t) and bias indices s'+t-i'+k-1, t = 0..k-1."""
        keys = (ctypes.c_int * k)()
        bidx = (ctypes.c_int * k)()
        if self._lib.oracle_axis_neighbors(L, k, d, i, keys, bidx) != 0:
            raise ValueError(f"no window: L={L} k={k} d={d} i={i}")
        return list(keys), list(bidx)

    # -- the three stages and their composition -----------------------------
    def qk_rpb(self, q, k, rpb, kernel_size: int, dilation: int, nthreads: int | None = None) -> np.ndarray:
        """attn[b,h,i,j,ty*k+tx] = q.k / sqrt(D) + rpb[h, dy, dx]."""
        q, k = _f64(q), _f64(k)
        rpb = None if rpb is None else _f64(rpb)
        shp = _shape(q, kernel_size, dilation)
        attn = np.empty(q.shape[:4] + (kernel_size * kernel_size,), dtype=np.float64)
        _check(self._lib.oracle_na2d_qk_rpb(*shp, _ptr(q), _ptr(k), _ptr(rpb), _ptr(attn),
                                            nthreads or default_threads()), "qk_rpb")
        return attn

    def softmax(self, attn, kernel_size: int, dilation: int, D: int = 32, nthreads: int | None = None) -> np.ndarray:
        """Softmax over the last (k*k) dimension; returns a new array."""
        a = _f64(attn).copy()
        B, heads, H, W, _ = a.shape
        _check(self._lib.oracle_na2d_softmax(B, heads, H, W, D, kernel_size, dilation, _ptr(a),
                                             nthreads or default_threads()), "softmax")
        return a

    def av(self, attn, v, kernel_size: int, dilation: int, nthreads: int | None = None) -> np.ndarray:
        """out[b,h,i,j,:] = sum_n attn[b,h,i,j,n] * v[key_n]."""
        a, v = _f64(attn), _f64(v)
        shp = _shape(v, kernel_size, dilation)
        out = np.empty(v.shape, dtype=np.float64)
        _check(self._lib.oracle_na2d_av(*shp, _ptr(a), _ptr(v), _ptr(out),
                                        nthreads or default_threads()), "av")
        return out

    def forward(self, q, k, v, rpb, kernel_size: int, dilation: int, nthreads: int | None = None) -> np.ndarray:
        """out = softmax(q.k/sqrt(D) + rpb) . v over each query's k*k (dilated) window."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        rpb = None if rpb is None else _f64(rpb)
        shp = _shape(q, kernel_size, dilation)
        out = np.empty(q.shape, dtype=np.float64)
        _check(self._lib.oracle_na2d_forward(*shp, _ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(out),
                                             nthreads or default_threads()), "forward")
        return out

    def backward(self, q, k, v, rpb, dout, kernel_size: int, dilation: int, nthreads: int | None = None):
        """Gradients (dq, dk, dv, drpb) of the fused forward for the output
        gradient dout; drpb is returned even when rpb is None (the gradient
        with respect to a zero bias)."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        rpb = None if rpb is None else _f64(rpb)
        shp = _shape(q, kernel_size, dilation)
        dq, dk, dv = (np.empty(q.shape, dtype=np.float64) for _ in range(3))
        nb = 2 * kernel_size - 1
        drpb = np.empty((q.shape[1], nb, nb), dtype=np.float64)
        _check(self._lib.oracle_na2d_backward(*shp, _ptr(q), _ptr(k), _ptr(v), _ptr(rpb), _ptr(dout), _ptr(dq),
                                              _ptr(dk), _ptr(dv), _ptr(drpb), nthreads or default_threads()),
               "backward")
        return dq, dk, dv, drpb

    # -- dropout, returned weights --------------------------------------------
    def philox(self, ctr, key) -> list[int]:
        """Philox4x32-10 of a 4-word counter and 2-word key (SC 2011 definition)."""
        c = (ctypes.c_uint * 4)(*ctr)
        kk = (ctypes.c_uint * 2)(*key)
        o = (ctypes.c_uint * 4)()
        self._lib.oracle_philox4x32_10(c, kk, o)
        return list(o)

    def forward_ex(self, q, k, v, rpb, kernel_size: int, dilation: int, dropout_p: float = 0.0, seed: int = 0,
                   offset: int = 0, return_attn: bool = False):
        """Forward with attention dropout (Philox mask) and, optionally, the
        weights after dropout [B, heads, H, W, k*k].  Maps shorter than
        kernel_size * dilation are zero-padded and cropped as in
        forward_padded; weights are numbered over the real map."""
        H, W = q.shape[2], q.shape[3]
        Q, K, V = (self._pad(t, kernel_size, dilation) for t in (q, k, v))
        rpb = None if rpb is None else _f64(rpb)
        shp = _shape(Q, kernel_size, dilation)
        out = np.empty(Q.shape, dtype=np.float64)
        attn = np.empty(q.shape[:4] + (kernel_size * kernel_size,), dtype=np.float64) if return_attn else None
        _check(self._lib.oracle_na2d_forward_ex(*shp, _ptr(Q), _ptr(K), _ptr(V), _ptr(rpb), _ptr(out), _ptr(attn),
                                                float(np.float32(dropout_p)), seed, offset, H, W), "forward_ex")
        out = np.ascontiguousarray(out[:, :, :H, :W])
        return (out, attn) if return_attn else out

    def backward_ex(self, q, k, v, rpb, dout, kernel_size: int, dilation: int, dropout_p: float = 0.0,
                    seed: int = 0, offset: int = 0):
        """Gradients of forward_ex with the same dropout mask."""
        H, W = q.shape[2], q.shape[3]
        Q, K, V, G = (self._pad(t, kernel_size, dilation) for t in (q, k, v, dout))
        rpb = None if rpb is None else _f64(rpb)
        shp = _shape(Q, kernel_size, dilation)
        dq, dk, dv = (np.empty(Q.shape, dtype=np.float64) for _ in range(3))
        nb = 2 * kernel_size - 1
        drpb = np.empty((q.shape[1], nb, nb), dtype=np.float64)
        _check(self._lib.oracle_na2d_backward_ex(*shp, _ptr(Q), _ptr(K), _ptr(V), _ptr(rpb), _ptr(G), _ptr(dq),
                                                 _ptr(dk), _ptr(dv), _ptr(drpb), float(np.float32(dropout_p)), seed,
                                                 offset, H, W), "backward_ex")
        crop = lambda a: np.ascontiguousarray(a[:, :, :H, :W])   # noqa: E731
        return crop(dq), crop(dk), crop(dv), drpb

    @staticmethod
    def _pad(t, kernel_size: int, dilation: int):
        """Zero pixels at the bottom / right up to kernel_size * dilation."""
        H, W = t.shape[2], t.shape[3]
        pads = ((0, 0), (0, 0), (0, max(0, kernel_size * dilation - H)), (0, max(0, kernel_size * dilation - W)),
                (0, 0))
        return np.ascontiguousarray(np.pad(_f64(t), pads))

    # -- maps shorter than k * d ------------------------------------------------
    def forward_padded(self, q, k, v, rpb, kernel_size: int, dilation: int):
        """The layer's padding (HF DiNAT maybe_pad, gitcode DiNAT article's
        layer walkthrough): pad the map with zero pixels at the bottom/right
        up to kernel_size * dilation, attend, crop back to H x W."""
        H, W = q.shape[2], q.shape[3]
        pads = ((0, 0), (0, 0), (0, max(0, kernel_size * dilation - H)), (0, max(0, kernel_size * dilation - W)),
                (0, 0))
        Q, K, V = (np.pad(_f64(t), pads) for t in (q, k, v))
        return self.forward(Q, K, V, rpb, kernel_size, dilation)[:, :, :H, :W]

    def backward_padded(self, q, k, v, rpb, dout, kernel_size: int, dilation: int):
        """Gradients of forward_padded: the padded pixels' outputs are cropped
        (zero output gradient there) and their input gradients dropped."""
        H, W = q.shape[2], q.shape[3]
        pads = ((0, 0), (0, 0), (0, max(0, kernel_size * dilation - H)), (0, max(0, kernel_size * dilation - W)),
                (0, 0))
        Q, K, V, G = (np.pad(_f64(t), pads) for t in (q, k, v, dout))
        dq, dk, dv, drpb = self.backward(Q, K, V, rpb, G, kernel_size, dilation)
        return dq[:, :, :H, :W], dk[:, :, :H, :W], dv[:, :, :H, :W], drpb

    def forward_query(self, q, k, v, rpb, kernel_size: int, dilation: int,
                      b: int, h: int, i: int, j: int) -> np.ndarray:
        """One output row from the definition, with numpy on the window that
        ``axis_neighbors`` returns; used for sampled checks at full sizes."""
        H, W, D = q.shape[2], q.shape[3], q.shape[4]
        ky, by = self.axis_neighbors(H, kernel_size, dilation, i)
        kx, bx = self.axis_neighbors(W, kernel_size, dilation, j)
        qv = np.asarray(q[b, h, i, j], dtype=np.float64)
        keys = np.asarray(k[b, h][np.ix_(ky, kx)], dtype=np.float64).reshape(-1, D)
        vals = np.asarray(v[b, h][np.ix_(ky, kx)], dtype=np.float64).reshape(-1, D)
        s = keys @ qv / np.sqrt(D)
        if rpb is not None:
            s = s + np.asarray(rpb[h], dtype=np.float64)[np.ix_(by, bx)].reshape(-1)
        p = np.exp(s - s.max())
        p /= p.sum()
        return p @ vals


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from ``oracle/na2d_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def axis_window(L, k, d, i):
    return get().axis_window(L, k, d, i)


def axis_neighbors(L, k, d, i):
    return get().axis_neighbors(L, k, d, i)


def qk_rpb(q, k, rpb, kernel_size, dilation, nthreads=None):
    return get().qk_rpb(q, k, rpb, kernel_size, dilation, nthreads)


def softmax(attn, kernel_size, dilation, D=32, nthreads=None):
    return get().softmax(attn, kernel_size, dilation, D, nthreads)


def av(attn, v, kernel_size, dilation, nthreads=None):
    return get().av(attn, v, kernel_size, dilation, nthreads)


def forward(q, k, v, rpb, kernel_size, dilation, nthreads=None):
    return get().forward(q, k, v, rpb, kernel_size, dilation, nthreads)


def forward_query(q, k, v, rpb, kernel_size, dilation, b, h, i, j):
    return get().forward_query(q, k, v, rpb, kernel_size, dilation, b, h, i, j)


def backward(q, k, v, rpb, dout, kernel_size, dilation, nthreads=None):
    return get().backward(q, k, v, rpb, dout, kernel_size, dilation, nthreads)


def philox(ctr, key):
    return get().philox(ctr, key)


def forward_ex(q, k, v, rpb, kernel_size, dilation, dropout_p=0.0, seed=0, offset=0, return_attn=False):
    return get().forward_ex(q, k, v, rpb, kernel_size, dilation, dropout_p, seed, offset, return_attn)


def backward_ex(q, k, v, rpb, dout, kernel_size, dilation, dropout_p=0.0, seed=0, offset=0):
    return get().backward_ex(q, k, v, rpb, dout, kernel_size, dilation, dropout_p, seed, offset)


def forward_padded(q, k, v, rpb, kernel_size, dilation):
    return get().forward_padded(q, k, v, rpb, kernel_size, dilation)


def backward_padded(q, k, v, rpb, dout, kernel_size, dilation):
    return get().backward_padded(q, k, v, rpb, dout, kernel_size, dilation)
