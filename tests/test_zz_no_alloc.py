"""na2d_backward_noalloc, called through the C ABI.

Some callers of this library cannot allocate device memory while they run:
code whose host framework owns every device allocation and allows none
during execution, or a loop that cannot accept the device-wide
synchronisation a cudaMalloc / cudaFree may cause.  For them the library has
na2d_backward_noalloc, which uses a fixed 16 MiB scratch array built into the
library instead of a workspace from the caller.

This file checks that it returns what na2d_backward (the workspace entry
point) returns, within the backward tests' tolerance, on two calls in a row
on different problems (so the second call cannot lean on what the first left
in the shared array), and that a problem too large for the array is refused
before any launch.  It is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import neighborhood_attention_na2d_b200 as na
from neighborhood_attention_na2d_b200 import _native
from neighborhood_attention_na2d_b200.build import build
from neighborhood_attention_na2d_b200.inputs import DTYPES, Shape, make_inputs

pytestmark = pytest.mark.gpu

# the backward tests' tolerance: |a - b| <= atol + rtol * |b|
ATOL = {"f32": 1e-5, "f16": 5e-3, "bf16": 2e-2}
RTOL = {"f32": 1e-5, "f16": 2.0 ** -10, "bf16": 2.0 ** -7}


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build()
    torch.cuda.init()


def _dout(shape, seed):
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return torch.randn((shape.B, shape.heads, shape.H, shape.W, shape.D), generator=gen).to(DTYPES[shape.dtype])


def _noalloc(shape, q, k, v, rpb, dout):
    """Outputs are the caller's buffers (allocated here, by the test); the
    entry point itself allocates nothing."""
    dq, dk, dv, drpb = (torch.full_like(t, float("nan")) for t in (q, q, q, rpb))
    p = na.make_problem(q.shape, shape.k, shape.d, q.dtype)
    st = _native.backward_noalloc_ptr(p, q.data_ptr(), k.data_ptr(), v.data_ptr(), rpb.data_ptr(), dout.data_ptr(),
                                      dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), drpb.data_ptr(),
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0, _native.status_str(st)
    return dq, dk, dv, drpb


def test_noalloc_matches_workspace_entry_point_twice():
    shapes = [Shape(2, 2, 14, 15, 32, 7, 1, "bf16", 901), Shape(1, 3, 16, 16, 32, 5, 2, "f16", 902)]
    for shape in shapes:                       # two calls in a row, different problems
        q, k, v, rpb = (t.cuda() for t in make_inputs(shape))
        dout = _dout(shape, shape.seed + 1).cuda()
        got = _noalloc(shape, q, k, v, rpb, dout)
        want = na.na2d_backward(q, k, v, rpb, dout, shape.k, shape.d)
        torch.cuda.synchronize()
        for name, g, w in zip(("dq", "dk", "dv", "drpb"), got, want):
            g, w = g.double().cpu().numpy(), w.double().cpu().numpy()
            excess = np.abs(g - w) - (ATOL[shape.dtype] + RTOL[shape.dtype] * np.abs(w))
            assert excess.max() <= 0, f"{shape.describe()} {name}: worst excess {excess.max():.3g}"


def test_noalloc_refuses_problems_beyond_its_scratch():
    """8 bytes per query and head: 64 x 16 x 64 x 64 needs 32 MiB > 16 MiB.
    The addresses are never dereferenced: the size check refuses the call
    before any launch."""
    p = _native.Problem(64, 16, 64, 64, 32, 7, 1, _native.NA2D_BF16)
    F = [0x10000000 + 0x4000000 * i for i in range(8)]   # disjoint, aligned, never read
    st = _native.backward_noalloc_ptr(p, F[0], F[1], F[2], None, F[3], F[4], F[5], F[6], None, 0)
    assert st == 3
