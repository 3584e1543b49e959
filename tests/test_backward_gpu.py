"""GPU parity of the backward (na2d_backward, through the C ABI) against the
fp64 oracle's backward on the same seeded inputs.

Tolerance, per element: |got - want| <= atol + rtol * |want|, with the
forward's absolute bounds as atol (1e-5 fp32, 5e-3 fp16, 2e-2 bf16) and rtol
covering the final rounding of large gradients to the dtype (half an ulp is
2^-9 relative for bf16, 2^-12 for fp16; the bias gradient sums up to
B*H*W terms, so its magnitude grows with the batch): rtol = 1e-5 (fp32),
2^-10 (fp16), 2^-7 (bf16).  All arithmetic on the GPU is fp32.
"""
import numpy as np
import pytest
import torch

import neighborhood_attention_na2d_b200 as na
import oracle
from neighborhood_attention_na2d_b200.build import build
from neighborhood_attention_na2d_b200.inputs import Shape, all_shapes, make_inputs

pytestmark = pytest.mark.gpu

ATOL = {"f32": 1e-5, "f16": 5e-3, "bf16": 2e-2}
RTOL = {"f32": 1e-5, "f16": 2.0 ** -10, "bf16": 2.0 ** -7}


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build()
    torch.cuda.init()


def f64(t):
    return None if t is None else t.double().numpy()


def make_dout(shape: Shape, seed: int):
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    from neighborhood_attention_na2d_b200.inputs import DTYPES
    return torch.randn((shape.B, shape.heads, shape.H, shape.W, shape.D), generator=gen).to(DTYPES[shape.dtype])


def check(name, got, want, dtype):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    bound = ATOL[dtype] + RTOL[dtype] * np.abs(want)
    excess = np.abs(got - want) - bound
    assert excess.max() <= 0, f"{name}: worst excess {excess.max():.3g} at {np.unravel_index(excess.argmax(), excess.shape)}"


def run(shape: Shape, with_rpb=True):
    q, k, v, rpb = make_inputs(shape)
    if not with_rpb:
        rpb = None
    dout = make_dout(shape, shape.seed + 77)
    dev = [None if t is None else t.cuda() for t in (q, k, v, rpb, dout)]
    dq, dk, dv, drpb = na.na2d_backward(*dev, shape.k, shape.d, drpb=None if with_rpb else
                                        torch.empty(shape.heads, 2 * shape.k - 1, 2 * shape.k - 1,
                                                    dtype=q.dtype, device="cuda"))
    torch.cuda.synchronize()
    want = oracle.backward(f64(q), f64(k), f64(v), f64(rpb), f64(dout), shape.k, shape.d)
    for name, g, w in zip(("dq", "dk", "dv", "drpb"), (dq, dk, dv, drpb), want):
        check(f"{shape.describe()} {name}", g, w, shape.dtype)


SMALL = [Shape(1, 2, 9, 11, 32, 3, 1, "f32", 801), Shape(2, 1, 13, 12, 32, 5, 2, "f16", 802),
         Shape(1, 3, 14, 14, 32, 7, 1, "bf16", 803), Shape(1, 2, 15, 17, 32, 7, 2, "f16", 804),
         Shape(2, 2, 14, 14, 32, 7, 2, "bf16", 805), Shape(1, 1, 13, 13, 32, 13, 1, "f32", 806),
         Shape(1, 2, 27, 26, 32, 13, 2, "bf16", 807), Shape(1, 2, 7, 8, 32, 1, 1, "f16", 808)]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.describe())
@pytest.mark.parametrize("with_rpb", [True, False], ids=["rpb", "no_rpb"])
def test_backward_small(shape, with_rpb):
    """Ragged maps, clamped edges, dilation, k from 1 to 13, every dtype."""
    run(shape, with_rpb)


@pytest.mark.parametrize("name,shape", all_shapes(), ids=[f"{n}:{s.describe()}" for n, s in all_shapes()])
def test_backward_workloads(name, shape):
    """Every workload shape at full size, every gradient element."""
    run(shape)


def test_autograd_matches_oracle():
    """torch autograd through na.na2d (forward and backward in the library)."""
    shape = Shape(2, 2, 16, 15, 32, 7, 1, "f16", 809)
    q, k, v, rpb = make_inputs(shape)
    dout = make_dout(shape, 5)
    leaves = [t.cuda().requires_grad_(True) for t in (q, k, v, rpb)]
    out = na.na2d(*leaves, shape.k, shape.d)
    out.backward(dout.cuda())
    want = oracle.backward(f64(q), f64(k), f64(v), f64(rpb), f64(dout), shape.k, shape.d)
    for name, t, w in zip(("dq", "dk", "dv", "drpb"), leaves, want):
        check(name, t.grad, w, shape.dtype)


def test_backward_rejects_small_workspace_and_alias():
    shape = Shape(1, 2, 14, 14, 32, 7, 1, "f16", 810)
    q, k, v, rpb = (t.cuda() for t in make_inputs(shape))
    dout = torch.randn_like(q)
    need = na.backward_workspace_size(na.make_problem(q.shape, 7, 1, q.dtype))
    assert need == (2 * 2 * 14 * 14 + 2 * 13 * 13) * 4
    with pytest.raises(na.Na2dError) as e:
        na.na2d_backward(q, k, v, rpb, dout, 7, 1, workspace=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 3
    with pytest.raises(na.Na2dError) as e:
        na.na2d_backward(q, k, v, rpb, dout, 7, 1, dq=dout)
    assert e.value.status == 7
