"""The C-ABI library on the host (no GPU needed): it loads, exports exactly what
include/na2d.h declares, and rejects bad arguments before any CUDA call.

The argument checks pass fake, never-dereferenced addresses.  They run in a
child process with CUDA_VISIBLE_DEVICES set empty, so even a case that wrongly
passed the checks could not launch a kernel on a real device.
"""
import json
import os
import re
import subprocess
import sys
from pathlib import Path

import pytest

from neighborhood_attention_na2d_b200 import _native
from neighborhood_attention_na2d_b200.build import build

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "na2d.h"
FAKE = 0x10000          # 16-byte aligned, never dereferenced
FAKE2 = 0x200000

BAD_PROBLEMS = [
    (dict(k=6), 4), (dict(k=0), 4), (dict(k=15), 4), (dict(k=-3), 4),
    (dict(d=0), 5), (dict(d=-1), 5),
    (dict(H=0), 3), (dict(W=0), 3), (dict(B=-1), 3), (dict(heads=-2), 3),
    (dict(D=48), 3), (dict(D=256), 3), (dict(D=8), 3),
    (dict(dtype=7), 2),
    (dict(H=1 << 20, W=1 << 20, k=1), 3),  # plane too large
]


def prob(**kw):
    base = dict(B=2, heads=2, H=14, W=14, D=32, k=7, d=1, dtype=_native.NA2D_F16)
    base.update(kw)
    return _native.Problem(**base)


def _host_checks() -> dict:
    """Runs in the child process: every call must fail (or be empty) on the host."""
    r = {}
    for i, (kw, _) in enumerate(BAD_PROBLEMS):
        r[f"bad{i}"] = _native.forward_ptr(prob(**kw), FAKE, FAKE, FAKE, None, FAKE2)
    p = prob()
    L = _native.lib()
    r["null_problem"] = L.na2d_forward(None, FAKE, FAKE, FAKE, None, FAKE2, None)
    r["null_q"] = _native.forward_ptr(p, 0, FAKE, FAKE, None, FAKE2)
    r["null_out"] = _native.forward_ptr(p, FAKE, FAKE, FAKE, None, 0)
    r["null_qk_k"] = _native.qk_rpb_ptr(p, FAKE, 0, None, FAKE2)
    r["null_softmax"] = _native.softmax_ptr(p, 0)
    r["null_av_v"] = _native.av_ptr(p, FAKE, 0, FAKE2)
    r["align_q"] = _native.forward_ptr(p, FAKE + 8, FAKE, FAKE, None, FAKE2)
    r["align_rpb"] = _native.forward_ptr(p, FAKE, FAKE, FAKE, FAKE + 1, FAKE2)
    r["align_attn"] = _native.qk_rpb_ptr(p, FAKE, FAKE, None, FAKE2 + 4)
    r["align_softmax"] = _native.softmax_ptr(p, FAKE + 4)
    r["align_av"] = _native.av_ptr(p, FAKE + 4, FAKE, FAKE2)
    nbytes = 2 * 2 * 14 * 14 * 32 * 2
    r["alias_out_q"] = _native.forward_ptr(p, FAKE, FAKE2, FAKE2, None, FAKE)
    r["alias_partial"] = _native.forward_ptr(p, FAKE, FAKE, FAKE, None, FAKE + nbytes - 16)
    r["alias_av"] = _native.av_ptr(p, FAKE, FAKE2, FAKE2)
    r["empty_B"] = _native.forward_ptr(prob(B=0), 0, 0, 0, None, 0)
    r["empty_heads"] = _native.forward_ptr(prob(heads=0), 0, 0, 0, None, 0)
    r["empty_qk"] = _native.qk_rpb_ptr(prob(B=0), 0, 0, None, 0)
    r["empty_softmax"] = _native.softmax_ptr(prob(B=0), 0)
    r["empty_av"] = _native.av_ptr(prob(B=0), 0, 0, 0)
    r["faults_null"] = L.na2d_device_faults(None, None)
    ws = _native.backward_workspace_size(p)
    r["ws_bytes"] = ws
    r["ws_empty"] = _native.backward_workspace_size(prob(B=0))
    F = [FAKE + 0x100000 * i for i in range(1, 10)]   # disjoint, 16-byte aligned
    r["bwd_null_dout"] = _native.backward_ptr(p, F[0], F[1], F[2], None, 0, F[3], F[4], F[5], None, F[6], ws)
    r["bwd_null_ws"] = _native.backward_ptr(p, F[0], F[1], F[2], None, F[7], F[3], F[4], F[5], None, 0, ws)
    r["bwd_small_ws"] = _native.backward_ptr(p, F[0], F[1], F[2], None, F[7], F[3], F[4], F[5], None, F[6], ws - 4)
    r["bwd_align"] = _native.backward_ptr(p, F[0], F[1], F[2], None, F[7], F[3] + 8, F[4], F[5], None, F[6], ws)
    r["bwd_alias_in"] = _native.backward_ptr(p, F[0], F[1], F[2], None, F[7], F[0], F[4], F[5], None, F[6], ws)
    r["bwd_alias_out"] = _native.backward_ptr(p, F[0], F[1], F[2], None, F[7], F[3], F[3], F[5], None, F[6], ws)
    r["bwd_alias_ws"] = _native.backward_ptr(p, F[0], F[1], F[2], None, F[7], F[3], F[4], F[5], None, F[7], ws)
    r["bwd_bad_k"] = _native.backward_ptr(prob(k=4), F[0], F[1], F[2], None, F[7], F[3], F[4], F[5], None, F[6], ws)
    r["bwd_empty"] = _native.backward_ptr(prob(B=0), 0, 0, 0, None, 0, 0, 0, 0, None, 0, 0)
    # forward_ex: strided views, weights, dropout
    import ctypes
    def T(ptr, sb=2 * 14 * 14 * 32, sh=14 * 14 * 32, sy=14 * 32, sx=32):
        return _native.Tensor(ptr, sb, sh, sy, sx)
    def fx(q, k, v, out, attn=None, drop=None, pp=None):
        return L.na2d_forward_ex(ctypes.byref(pp or p), ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), None,
                                 ctypes.byref(out), attn, None if drop is None else ctypes.byref(drop), None)
    r["fx_null"] = fx(T(0), T(F[1]), T(F[2]), T(F[3]))
    r["fx_stride_align"] = fx(T(F[0], sx=36), T(F[1]), T(F[2]), T(F[3]))
    r["fx_neg_stride"] = fx(T(F[0], sy=-448), T(F[1]), T(F[2]), T(F[3]))
    r["fx_out_self_overlap"] = fx(T(F[0]), T(F[1]), T(F[2]), T(F[3], sx=16))
    r["fx_out_on_input"] = fx(T(F[0]), T(F[1]), T(F[2]), T(F[0]))
    r["fx_attn_on_input"] = fx(T(F[0]), T(F[1]), T(F[2]), T(F[3]), attn=F[1])
    r["fx_drop_p"] = fx(T(F[0]), T(F[1]), T(F[2]), T(F[3]), drop=_native.Dropout(1.0, 1, 0))
    r["fx_drop_neg"] = fx(T(F[0]), T(F[1]), T(F[2]), T(F[3]), drop=_native.Dropout(-0.1, 1, 0))
    r["fx_empty"] = fx(T(0), T(0), T(0), T(0), pp=prob(B=0))
    # one fused channels-last buffer: q, k, v views 2 * 32 elements apart per
    # head block, the output interleaved with them in a fourth slot is refused
    # only when it lands on an input block
    P3 = dict(sb=14 * 14 * 4 * 64, sh=32, sy=14 * 4 * 64, sx=4 * 64)
    base = F[0]
    r["fx_fused_ok"] = L.na2d_forward_ex(ctypes.byref(p), ctypes.byref(T(base, **P3)),
                                         ctypes.byref(T(base + 128, **P3)), ctypes.byref(T(base + 256, **P3)), None,
                                         ctypes.byref(T(base + 384, **P3)), None, None, None)
    r["fx_fused_clash"] = L.na2d_forward_ex(ctypes.byref(p), ctypes.byref(T(base, **P3)),
                                            ctypes.byref(T(base + 128, **P3)), ctypes.byref(T(base + 256, **P3)),
                                            None, ctypes.byref(T(base + 192, **P3)), None, None, None)
    # the host-buffer forward: workspace and alias checks before any copy
    ws = ctypes.c_size_t(0)
    L.na2d_forward_host_workspace_size(ctypes.byref(p), ctypes.byref(ws))
    r["fh_ws_size"] = ws.value
    big = 1 << 24
    r["fh_null_ws"] = L.na2d_forward_host(ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE2, None, big, None)
    r["fh_align_ws"] = L.na2d_forward_host(ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE2, FAKE + 8, big, None)
    r["fh_small_ws"] = L.na2d_forward_host(ctypes.byref(p), FAKE, FAKE, FAKE, None, FAKE2, FAKE, ws.value - 16,
                                           None)
    r["fh_alias"] = L.na2d_forward_host(ctypes.byref(p), FAKE, FAKE2, FAKE2, None, FAKE + 64, FAKE, big, None)
    r["fh_null_q"] = L.na2d_forward_host(ctypes.byref(p), None, FAKE, FAKE, None, FAKE2, FAKE, big, None)
    r["fh_bad_k"] = L.na2d_forward_host(ctypes.byref(prob(k=6)), FAKE, FAKE, FAKE, None, FAKE2, FAKE, big, None)
    r["fh_empty"] = L.na2d_forward_host(ctypes.byref(prob(B=0)), FAKE, FAKE, FAKE, None, FAKE2, None, 0, None)
    return r


@pytest.fixture(scope="module")
def host_results():
    build()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    code = ("import json, sys; sys.path[:0] = [%r, %r]; import test_abi_host as t; "
            "print(json.dumps(t._host_checks()))") % (str(ROOT), str(Path(__file__).parent))
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_fused_views_pass_the_host_checks(host_results):
    """Interleaved q / k / v / out views of one fused buffer pass every host
    check; with no device the call then fails only at the launch
    (NA2D_ERR_CUDA), never with an argument error."""
    assert host_results["fx_fused_ok"] == 8


def test_forward_host_workspace_size(host_results):
    """B=2 heads=2 14x14 D=32 f16: two chunks of one batch element, two slots of
    q, k, v and out (25,088 bytes each, already a multiple of 256) and the
    676-byte bias table rounded up to 768."""
    assert host_results["fh_ws_size"] == 8 * 2 * 14 * 14 * 32 * 2 + 768


@pytest.mark.parametrize("B", [1, 2, 7, 8, 9, 16, 33, 100])
def test_forward_host_workspace_size_chunks(B):
    """The host-buffer forward's workspace for a range of batches: at most 8
    chunks of ceil(B / min(B, 8)) batch elements, two slots of q, k, v and
    out (one slot for a single chunk), each rounded up to 256 bytes, then the
    bias table rounded up to 256 bytes.  Host-only: no CUDA call."""
    import ctypes
    build()
    heads, H, W, D, k = 3, 10, 9, 32, 5
    p = prob(B=B, heads=heads, H=H, W=W, D=D, k=k)
    n = ctypes.c_size_t(0)
    assert _native.lib().na2d_forward_host_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0
    cb = -(-B // min(B, 8))
    nchunk = -(-B // cb)
    slots = 2 if nchunk > 1 else 1
    r256 = lambda x: -(-x // 256) * 256
    per = r256(cb * heads * H * W * D * 2)
    assert nchunk <= 8
    assert n.value == 4 * slots * per + r256(heads * (2 * k - 1) ** 2 * 2)


def test_backward_workspace_size(host_results):
    """[lse, delta] fp32 per query and head plus the fp32 bias table."""
    assert host_results["ws_bytes"] == (2 * 2 * 2 * 14 * 14 + 2 * 13 * 13) * 4
    assert host_results["ws_empty"] == 0


def header_functions():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"NA2D_API\s+[\w\s\*]+?\b(na2d_\w+)\s*\(", text)))


def test_exports_match_header():
    build()
    lib = _native.lib()
    declared = header_functions()
    assert declared == sorted(_native.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", str(_native.LIB_PATH)], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted({ln.split()[-1] for ln in out.splitlines() if ln.split() and ln.split()[-1].startswith("na2d")})
    assert exported == declared          # nothing internal leaks, nothing is missing
    for name in declared:
        assert hasattr(lib, name)


def test_version_and_status_strings():
    build()
    assert _native.lib().na2d_version() == 200
    names = [_native.status_str(s) for s in range(10)]
    assert names[0] == "ok" and len(set(names)) == 10
    assert _native.status_str(99) == "unknown status"


@pytest.mark.parametrize("i", range(len(BAD_PROBLEMS)))
def test_forward_rejects_bad_problems(host_results, i):
    assert host_results[f"bad{i}"] == BAD_PROBLEMS[i][1], BAD_PROBLEMS[i][0]


@pytest.mark.parametrize("case,status", [
    ("null_problem", 1), ("null_q", 1), ("null_out", 1), ("null_qk_k", 1), ("null_softmax", 1), ("null_av_v", 1),
    ("align_q", 6), ("align_rpb", 6), ("align_attn", 6), ("align_softmax", 6), ("align_av", 6),
    ("alias_out_q", 7), ("alias_partial", 7), ("alias_av", 7),
    ("empty_B", 0), ("empty_heads", 0), ("empty_qk", 0), ("empty_softmax", 0), ("empty_av", 0), ("faults_null", 1),
    ("bwd_null_dout", 1), ("bwd_null_ws", 1), ("bwd_small_ws", 3), ("bwd_align", 6), ("bwd_alias_in", 7),
    ("bwd_alias_out", 7), ("bwd_alias_ws", 7), ("bwd_bad_k", 4), ("bwd_empty", 0),
    ("fx_null", 1), ("fx_stride_align", 6), ("fx_neg_stride", 6), ("fx_out_self_overlap", 7), ("fx_out_on_input", 7),
    ("fx_attn_on_input", 7), ("fx_drop_p", 3), ("fx_drop_neg", 3), ("fx_empty", 0), ("fx_fused_clash", 7),
    ("fh_null_ws", 1), ("fh_align_ws", 6), ("fh_small_ws", 3), ("fh_alias", 7), ("fh_null_q", 1), ("fh_bad_k", 4),
    ("fh_empty", 0),
])
def test_host_checks(host_results, case, status):
    assert host_results[case] == status


def test_binding_refuses_cpu_tensors():
    import torch
    import neighborhood_attention_na2d_b200 as na
    build()
    x = torch.zeros(1, 1, 7, 7, 32, dtype=torch.float16)
    with pytest.raises(na.Na2dError):
        na.na2d_forward(x, x, x, None, 7, 1, out=torch.empty_like(x))


# ---------------------------------------------------------------------------
# The Python binding checks every tensor against q before calling the library
# (which receives raw pointers and cannot detect a short or mistyped buffer).
# CPU tensors suffice: the checks run before any device work.
def _t(*shape, dtype=None):
    import torch
    return torch.zeros(*shape, dtype=dtype or torch.float16)


@pytest.mark.parametrize("case,status", [
    ("short_k", 3), ("short_v", 3), ("k_dtype", 2), ("out_short", 3), ("out_dtype", 2),
    ("rpb_small", 3), ("rpb_dtype", 2), ("rpb_heads", 3), ("q_4d", 3),
])
def test_binding_forward_mismatch(case, status):
    import torch
    import neighborhood_attention_na2d_b200 as na
    q = _t(1, 2, 14, 14, 32)
    k, v, out, rpb = _t(1, 2, 14, 14, 32), _t(1, 2, 14, 14, 32), _t(1, 2, 14, 14, 32), _t(2, 13, 13)
    if case == "short_k":
        k = _t(1, 2, 14, 13, 32)
    elif case == "short_v":
        v = _t(1, 1, 14, 14, 32)
    elif case == "k_dtype":
        k = _t(1, 2, 14, 14, 32, dtype=torch.bfloat16)
    elif case == "out_short":
        out = _t(1, 2, 14, 14, 16)
    elif case == "out_dtype":
        out = _t(1, 2, 14, 14, 32, dtype=torch.float32)
    elif case == "rpb_small":
        rpb = _t(2, 11, 11)
    elif case == "rpb_dtype":
        rpb = _t(2, 13, 13, dtype=torch.float32)
    elif case == "rpb_heads":
        rpb = _t(3, 13, 13)
    elif case == "q_4d":
        q = _t(2, 14, 14, 32)
    with pytest.raises(na.Na2dError) as e:
        na.na2d_forward(q, k, v, rpb, 7, 1, out=out)
    assert e.value.status == status


@pytest.mark.parametrize("case,status", [("attn_short", 3), ("attn_dtype", 2), ("av_out", 3), ("sm_shape", 3),
                                         ("sm_dtype", 2), ("qk_k", 3)])
def test_binding_split_mismatch(case, status):
    import torch
    import neighborhood_attention_na2d_b200 as na
    q = _t(1, 2, 14, 14, 32)
    attn = torch.zeros(1, 2, 14, 14, 49)
    with pytest.raises(na.Na2dError) as e:
        if case == "attn_short":
            na.na2d_av(torch.zeros(1, 2, 14, 14, 25), q, 7, 1)
        elif case == "attn_dtype":
            na.na2d_av(attn.half(), q, 7, 1)
        elif case == "av_out":
            na.na2d_av(attn, q, 7, 1, out=_t(1, 2, 14, 14, 8))
        elif case == "sm_shape":
            na.na2d_softmax(torch.zeros(1, 2, 14, 14, 48), 7, 1)
        elif case == "sm_dtype":
            na.na2d_softmax(attn.double(), 7, 1)
        elif case == "qk_k":
            na.na2d_qk_rpb(q, _t(1, 2, 13, 14, 32), None, 7, 1)
    assert e.value.status == status
