"""GPU parity of the library beyond the plain forward, through the C ABI,
against the fp64 oracle on the same seeded inputs:

* head dims 16, 64 and 128 (the plain forward, the split path, the backward);
* maps shorter than kernel_size x dilation (zero padding, then crop: the
  oracle's forward_padded / backward_padded);
* channels-last tensors: q, k, v read in place from one fused projection
  output (B, H, W, 3 * heads * D), the output written channels-last;
* the attention weights returned after dropout, and attention dropout
  (Philox mask: the kept/dropped pattern must match the oracle's exactly),
  forward, backward and through torch autograd.

Tolerances: the forward's max abs error 1e-5 (fp32), 5e-3 (fp16), 2e-2
(bf16); gradients |got - want| <= atol + rtol |want| as in
test_backward_gpu.py; returned fp32 weights 1e-5 (fp32 arithmetic on inputs
rounded to the dtype, compared with the oracle on the same rounded inputs).
"""
import numpy as np
import pytest
import torch

import neighborhood_attention_na2d_b200 as na
import oracle
from neighborhood_attention_na2d_b200.build import build
from neighborhood_attention_na2d_b200.inputs import DTYPES, Shape, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 5e-3, "bf16": 2e-2}
RTOL = {"f32": 1e-5, "f16": 2.0 ** -10, "bf16": 2.0 ** -7}


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build()
    torch.cuda.init()


def f64(t):
    return None if t is None else t.double().cpu().numpy()


def randn(shape: Shape, seed: int, dims=None):
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    dims = dims or (shape.B, shape.heads, shape.H, shape.W, shape.D)
    return torch.randn(dims, generator=gen).to(DTYPES[shape.dtype])


def max_err(a, b):
    return float(np.abs(np.asarray(a) - np.asarray(b)).max()) if np.asarray(a).size else 0.0


def check_grad(name, got, want, dtype):
    got = f64(got)
    excess = np.abs(got - want) - (TOL[dtype] + RTOL[dtype] * np.abs(want))
    assert excess.max() <= 0, f"{name}: worst excess {excess.max():.3g}"


# ---------------------------------------------------------------------------
OTHER_D = [Shape(2, 2, 13, 11, 16, 7, 1, "f16", 1101), Shape(1, 3, 12, 15, 64, 5, 2, "bf16", 1102),
           Shape(1, 2, 9, 10, 128, 3, 1, "f32", 1103), Shape(2, 1, 14, 14, 64, 7, 2, "f16", 1104),
           Shape(1, 2, 8, 9, 128, 7, 1, "bf16", 1105), Shape(1, 1, 15, 13, 16, 13, 1, "f32", 1106)]


@pytest.mark.parametrize("shape", OTHER_D, ids=lambda s: s.describe())
def test_head_dims_forward_split_backward(shape):
    q, k, v, rpb = make_inputs(shape)
    qd, kd, vd, rd = (t.cuda() for t in (q, k, v, rpb))
    out = na.na2d_forward(qd, kd, vd, rd, shape.k, shape.d)
    torch.cuda.synchronize()
    assert na.na2d_last_kernel() == "fwd_simt_kernel"
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    assert max_err(f64(out), want) <= TOL[shape.dtype]
    # split path
    attn = na.na2d_qk_rpb(qd, kd, rd, shape.k, shape.d)
    na.na2d_softmax(attn, shape.k, shape.d, D=shape.D, dtype=q.dtype)
    o2 = na.na2d_av(attn, vd, shape.k, shape.d)
    torch.cuda.synchronize()
    assert max_err(f64(o2), want) <= TOL[shape.dtype]
    # backward
    g = randn(shape, shape.seed + 5)
    grads = na.na2d_backward(qd, kd, vd, rd, g.cuda(), shape.k, shape.d)
    torch.cuda.synchronize()
    wants = oracle.backward(f64(q), f64(k), f64(v), f64(rpb), f64(g), shape.k, shape.d)
    for name, a, b in zip(("dq", "dk", "dv", "drpb"), grads, wants):
        check_grad(name, a, b, shape.dtype)


PADDED = [Shape(1, 2, 5, 9, 32, 7, 1, "f16", 1201), Shape(2, 1, 10, 6, 32, 3, 4, "bf16", 1202),
          Shape(1, 2, 3, 3, 32, 13, 1, "f32", 1203), Shape(1, 3, 7, 7, 32, 7, 2, "bf16", 1204),
          Shape(1, 2, 20, 9, 64, 5, 3, "f16", 1205), Shape(1, 1, 1, 1, 16, 3, 1, "f32", 1206)]


@pytest.mark.parametrize("shape", PADDED, ids=lambda s: s.describe())
def test_padded_short_maps(shape):
    """H or W < k * d: zero padding at the bottom/right, then crop."""
    q, k, v, rpb = make_inputs(shape)
    qd, kd, vd, rd = (t.cuda() for t in (q, k, v, rpb))
    out = na.na2d_forward(qd, kd, vd, rd, shape.k, shape.d)
    torch.cuda.synchronize()
    want = oracle.forward_padded(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    assert max_err(f64(out), want) <= TOL[shape.dtype]
    attn = na.na2d_qk_rpb(qd, kd, rd, shape.k, shape.d)
    na.na2d_softmax(attn, shape.k, shape.d, D=shape.D, dtype=q.dtype)
    o2 = na.na2d_av(attn, vd, shape.k, shape.d)
    torch.cuda.synchronize()
    assert max_err(f64(o2), want) <= TOL[shape.dtype]
    g = randn(shape, shape.seed + 6)
    grads = na.na2d_backward(qd, kd, vd, rd, g.cuda(), shape.k, shape.d)
    torch.cuda.synchronize()
    wants = oracle.backward_padded(f64(q), f64(k), f64(v), f64(rpb), f64(g), shape.k, shape.d)
    for name, a, b in zip(("dq", "dk", "dv", "drpb"), grads, wants):
        check_grad(name, a, b, shape.dtype)


# ---------------------------------------------------------------------------
QKV = [(2, 14, 15, 2, 32, 7, 1, "f16"), (1, 28, 28, 4, 32, 7, 4, "bf16"), (2, 9, 11, 3, 64, 3, 2, "f32"),
       (1, 5, 6, 2, 16, 7, 1, "bf16")]


@pytest.mark.parametrize("B,H,W,heads,D,k,d,dtype", QKV)
def test_fused_qkv_channels_last(B, H, W, heads, D, k, d, dtype):
    """q, k, v read in place from a (B, H, W, 3 * heads * D) projection output;
    the output written channels-last (B, H, W, heads * D); and the backward
    on the same strided views."""
    shape = Shape(B, heads, H, W, D, k, d, dtype, 1300 + H)
    qkv = randn(shape, shape.seed, dims=(B, H, W, 3 * heads * D))
    rpb = (randn(shape, shape.seed + 1, dims=(heads, 2 * k - 1, 2 * k - 1)).float() * 0.02).to(qkv.dtype)
    qkvd, rd = qkv.cuda(), rpb.cuda()
    out = na.na2d_qkv_packed(qkvd, rd, k, d, heads)
    torch.cuda.synchronize()
    q, kk, v = (t.contiguous() for t in na.qkv_views(qkv, heads))
    fwd = oracle.forward_padded if min(H, W) < k * d else oracle.forward
    want = fwd(f64(q), f64(kk), f64(v), f64(rpb), k, d)                   # [B, heads, H, W, D]
    want_cl = want.transpose(0, 2, 3, 1, 4).reshape(B, H, W, heads * D)
    assert max_err(f64(out), want_cl) <= TOL[dtype]
    # backward on views: gradients land in a channels-last fused gradient buffer
    g = randn(shape, shape.seed + 2, dims=(B, H, W, heads * D))
    gview = g.cuda().view(B, H, W, heads, D).permute(0, 3, 1, 2, 4)
    dqkv = torch.full_like(qkvd, float("nan"))
    dq, dk, dv = na.qkv_views(dqkv, heads)
    qd, kd, vd = na.qkv_views(qkvd, heads)
    na.na2d_backward_ex(qd, kd, vd, rd, gview, k, d, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    bwd = oracle.backward_padded if min(H, W) < k * d else oracle.backward
    wants = bwd(f64(q), f64(kk), f64(v), f64(rpb), f64(gview.cpu()), k, d)
    for name, a, b in zip(("dq", "dk", "dv"), (dq, dk, dv), wants[:3]):
        check_grad(name, a, b, dtype)


# ---------------------------------------------------------------------------
DROP = [(Shape(2, 2, 14, 13, 32, 7, 1, "f16", 1401), 0.1, 12345, 0),
        (Shape(1, 3, 12, 12, 64, 5, 2, "bf16", 1402), 0.5, (7 << 40) + 3, 1 << 33),
        (Shape(1, 2, 9, 8, 32, 3, 3, "f32", 1403), 0.25, 1, 77),
        (Shape(1, 2, 5, 6, 16, 7, 1, "f32", 1404), 0.0, 5, 0)]


@pytest.mark.parametrize("shape,p,seed,offset", DROP, ids=lambda x: x.describe() if isinstance(x, Shape) else str(x))
def test_weights_and_dropout(shape, p, seed, offset):
    """The returned weights and the output with dropout; the kept/dropped
    pattern must equal the oracle's exactly; then the backward with the same
    mask."""
    q, k, v, rpb = make_inputs(shape)
    qd, kd, vd, rd = (t.cuda() for t in (q, k, v, rpb))
    out, attn = na.na2d_forward_ex(qd, kd, vd, rd, shape.k, shape.d, return_attn=True, dropout_p=p, seed=seed,
                                   offset=offset)
    torch.cuda.synchronize()
    assert na.na2d_last_kernel() == "fwd_simt_kernel"
    fwd = oracle.forward_ex
    want, wattn = fwd(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d, p, seed, offset, return_attn=True)
    got_attn = attn.double().cpu().numpy()
    assert np.array_equal(got_attn > 0, wattn > 0), "dropout mask differs from the oracle's"
    assert max_err(got_attn, wattn) <= 1e-5 / (1 - p)
    assert max_err(f64(out), want) <= TOL[shape.dtype]
    g = randn(shape, shape.seed + 7)
    grads = na.na2d_backward_ex(qd, kd, vd, rd, g.cuda(), shape.k, shape.d, dropout_p=p, seed=seed, offset=offset)
    torch.cuda.synchronize()
    wants = oracle.backward_ex(f64(q), f64(k), f64(v), f64(rpb), f64(g), shape.k, shape.d, p, seed, offset)
    for name, a, b in zip(("dq", "dk", "dv", "drpb"), grads, wants):
        check_grad(name, a, b, shape.dtype)


def test_autograd_with_dropout():
    shape = Shape(1, 2, 15, 14, 32, 7, 1, "bf16", 1501)
    q, k, v, rpb = make_inputs(shape)
    g = randn(shape, 3)
    leaves = [t.cuda().requires_grad_(True) for t in (q, k, v, rpb)]
    out = na.na2d(*leaves, shape.k, shape.d, dropout_p=0.2, seed=4242)
    out.backward(g.cuda())
    want = oracle.forward_ex(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d, 0.2, 4242, 0)
    assert max_err(f64(out.detach()), want) <= TOL[shape.dtype]
    wants = oracle.backward_ex(f64(q), f64(k), f64(v), f64(rpb), f64(g), shape.k, shape.d, 0.2, 4242, 0)
    for name, t, w in zip(("dq", "dk", "dv", "drpb"), leaves, wants):
        check_grad(name, t.grad, w, shape.dtype)


def test_forward_ex_contiguous_takes_the_fast_kernels():
    shape = Shape(2, 2, 16, 16, 32, 7, 1, "f16", 1601)
    q, k, v, rpb = (t.cuda() for t in make_inputs(shape))
    na.na2d_forward_ex(q, k, v, rpb, 7, 1)
    assert na.na2d_last_kernel() == "fwd_stream_kernel"


# ---------------------------------------------------------------------------
# (layout, W, the kernel that must run): at W <= 64 the streaming kernel takes
# all three layouts (rows copied as 16-byte pieces when they are strided);
# above 64 columns its column bands copy rows of densely packed images only,
# so these views take the generic kernel
STRIDED = [("fused_qkv", 20, "fwd_stream_kernel"), ("channels_last", 20, "fwd_stream_kernel"),
           ("padded_rows", 20, "fwd_stream_kernel"), ("padded_rows", 72, "fwd_simt_kernel"),
           ("fused_qkv", 72, "fwd_simt_kernel"), ("channels_last", 72, "fwd_simt_kernel")]


@pytest.mark.parametrize("layout,W,kernel", STRIDED)
def test_stream_kernel_strided_rows(layout, W, kernel):
    """The k = 7 sliding-window forward on q, k, v views whose rows are not
    contiguous: the three views of a fused (B, H, W, 3 heads D) buffer,
    channels-last (B, H, W, heads D) tensors, and [B, heads, H, W, D] slices
    of tensors with two spare pixels per row; the kernel that runs is the
    one the dispatch promises, and the output equals the oracle."""
    B, heads, H, D, k, d = 2, 2, 14, 32, 7, 1
    shape = Shape(B, heads, H, W, D, k, d, "f16", 1500 + W)
    q, kk, v, rpb = make_inputs(shape)
    if layout == "fused_qkv":
        qkv = torch.cat([t.permute(0, 2, 3, 1, 4).reshape(B, H, W, heads * D) for t in (q, kk, v)], dim=-1).cuda()
        qd, kd, vd = na.qkv_views(qkv, heads)
    elif layout == "channels_last":
        qd, kd, vd = (t.permute(0, 2, 3, 1, 4).contiguous().cuda().permute(0, 3, 1, 2, 4) for t in (q, kk, v))
    else:
        def padded(t):
            big = torch.zeros(B, heads, H, W + 2, D, dtype=t.dtype)
            big[:, :, :, :W] = t
            return big.cuda()[:, :, :, :W]
        qd, kd, vd = (padded(t) for t in (q, kk, v))
    out = torch.full((B, heads, H, W, D), float("nan"), dtype=q.dtype, device="cuda")
    na.na2d_forward_ex(qd, kd, vd, rpb.cuda(), k, d, out=out)
    torch.cuda.synchronize()
    assert na.na2d_last_kernel() == kernel
    want = oracle.forward(f64(q), f64(kk), f64(v), f64(rpb), k, d)
    assert max_err(f64(out), want) <= TOL["f16"]
