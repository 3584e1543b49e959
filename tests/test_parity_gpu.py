"""GPU parity: the CUDA library, called through its C ABI, against the fp64
oracle on the same seeded inputs.

Tolerances (max abs error, fp32 accumulation everywhere): 1e-5 for fp32,
5e-3 for fp16 and 2e-2 for bf16 -- the bounds the problem statement sets for
this operation.  Inputs are drawn in fp32 and rounded to the dtype first; the
oracle sees exactly those rounded values, upcast to fp64.
"""
import math
import random

import numpy as np
import pytest
import torch

import neighborhood_attention_na2d_b200 as na
import oracle
from neighborhood_attention_na2d_b200.build import build
from neighborhood_attention_na2d_b200.inputs import WORKLOADS, Shape, all_shapes, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 5e-3, "bf16": 2e-2}
PAD = 256   # guard-band elements around every output (keeps 16-byte alignment)
SENTINEL = -12345.0


@pytest.fixture(scope="module", autouse=True)
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build()
    torch.cuda.init()


def f64(t):
    return None if t is None else t.double().numpy()


def guarded_out(like: torch.Tensor):
    """An output tensor inside a larger buffer whose margins hold a sentinel."""
    n = like.numel()
    buf = torch.full((n + 2 * PAD,), SENTINEL, dtype=like.dtype, device="cuda")
    return buf, buf[PAD:PAD + n].view(like.shape)


def check_guards(buf):
    edge = torch.cat([buf[:PAD], buf[-PAD:]]).float()
    assert bool((edge == float(torch.tensor(SENTINEL, dtype=buf.dtype).float())).all()), "write outside the output"


def run_forward(shape: Shape, with_rpb=True, seed=None):
    q, k, v, rpb = make_inputs(shape, seed)
    if not with_rpb:
        rpb = None
    buf, out = guarded_out(q)
    na.na2d_forward(q.cuda(), k.cuda(), v.cuda(), None if rpb is None else rpb.cuda(), shape.k, shape.d, out=out)
    torch.cuda.synchronize()
    check_guards(buf)
    return (q, k, v, rpb), out.double().cpu().numpy()


def max_err(a, b):
    return float(np.abs(a - b).max()) if a.size else 0.0


# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,shape", all_shapes(), ids=[f"{n}:{s.describe()}" for n, s in all_shapes()])
def test_workload_parity(name, shape):
    """Every workload shape, every output element, against the oracle."""
    (q, k, v, rpb), got = run_forward(shape)
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    err = max_err(got, want)
    assert err <= TOL[shape.dtype], f"{shape.describe()}: max abs err {err}"


def _ragged_cases():
    rnd = random.Random(2024)
    cases = []
    for n in range(48):
        k = rnd.choice([1, 3, 5, 7, 7, 9, 11, 13])
        d = rnd.choice([1, 1, 2, 3, 4, 5, 8])
        while k * d > 40:
            d = max(1, d // 2)
        H = rnd.randint(k * d, k * d + 2 * d + 11)
        W = rnd.randint(k * d, k * d + 2 * d + 11)
        dtype = rnd.choice(["f16", "bf16", "bf16", "f32"])
        cases.append((Shape(rnd.choice([1, 2]), rnd.choice([1, 3]), H, W, 32, k, d, dtype, 5000 + n),
                      rnd.random() < 0.8))
    return cases


@pytest.mark.parametrize("shape,with_rpb", _ragged_cases(), ids=lambda x: x.describe() if isinstance(x, Shape) else str(x))
def test_ragged_shapes(shape, with_rpb):
    """Seeded sweep of ragged sizes (H, W not multiples of any tile), every
    supported k, dilations 1..8, all three dtypes, with and without bias."""
    (q, k, v, rpb), got = run_forward(shape, with_rpb)
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    err = max_err(got, want)
    assert err <= TOL[shape.dtype], f"{shape.describe()} rpb={with_rpb}: max abs err {err}"


def _stream_cases():
    """Shapes of the k = 7 streaming schedules: d = 1 row streaming (W from 14
    to 64, odd and short H, several images per CTA, CTA ranges that cross
    images) and dense 7 x 7 groups (H = W = 7d, odd group counts)."""
    cases = []
    n = 0
    for (B, heads, H, W) in [(1, 1, 8, 14), (2, 3, 9, 15), (1, 2, 13, 21), (3, 1, 14, 28), (1, 2, 29, 40),
                             (2, 1, 17, 49), (2, 2, 56, 56), (1, 3, 11, 57), (1, 1, 30, 63), (2, 3, 8, 64),
                             (4, 3, 56, 56), (9, 5, 14, 14)]:
        for dtype in ("f16", "bf16"):
            cases.append((Shape(B, heads, H, W, 32, 7, 1, dtype, 7000 + n), n % 3 != 2))
            n += 1
    for (B, heads, d) in [(1, 1, 1), (3, 3, 1), (1, 2, 2), (2, 1, 3), (1, 3, 5), (1, 1, 8), (3, 1, 8)]:
        for dtype in ("f16", "bf16"):
            cases.append((Shape(B, heads, 7 * d, 7 * d, 32, 7, d, dtype, 7000 + n), n % 3 != 2))
            n += 1
    # 64 heads (the largest bias table of the dense kernel), more units than
    # SMs with an odd group count, and more sliding-row images than SMs (the
    # pairs are then split evenly across images)
    cases.append((Shape(1, 64, 7, 7, 32, 7, 1, "bf16", 7100), True))
    cases.append((Shape(3, 101, 7, 7, 32, 7, 1, "f16", 7101), True))
    cases.append((Shape(75, 2, 14, 14, 32, 7, 1, "f16", 7102), True))
    # maps wider than 64 columns: column bands (a partial last band, three
    # and four bands, more band images than SMs)
    cases.append((Shape(1, 2, 12, 65, 32, 7, 1, "f16", 7103), True))
    cases.append((Shape(2, 1, 17, 100, 32, 7, 1, "bf16", 7104), True))
    cases.append((Shape(1, 1, 10, 128, 32, 7, 1, "f16", 7105), False))
    cases.append((Shape(1, 1, 9, 200, 32, 7, 1, "bf16", 7106), True))
    cases.append((Shape(60, 1, 8, 72, 32, 7, 1, "f16", 7107), True))
    return cases


@pytest.mark.parametrize("shape,with_rpb", _stream_cases(), ids=lambda x: x.describe() if isinstance(x, Shape) else str(x))
def test_stream_shapes(shape, with_rpb):
    """The streaming k = 7 kernel's schedules, every output element."""
    (q, k, v, rpb), got = run_forward(shape, with_rpb)
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    err = max_err(got, want)
    assert err <= TOL[shape.dtype], f"{shape.describe()} rpb={with_rpb}: max abs err {err}"


def _ugrp_cases():
    """Shapes of the tcgen05 kernel for dilation groups of k .. 16 pixels a
    side with k >= 9: every key-tile height (NKR 9 .. 14), square and
    non-square groups, widths below 16 (zero-filled columns), heights below 16
    (a short second strip), ranges of units that span two (batch, head)
    planes, and blocks with more units than ring stages."""
    rows = [
        (1, 1, 9, 9, 9, 1, "f16", True),        # NKR 9, one group
        (1, 2, 10, 12, 9, 1, "bf16", True),     # NKR 10 / 12 strips
        (2, 1, 33, 36, 9, 3, "f16", False),     # 11 x 12 groups
        (1, 3, 16, 16, 9, 1, "bf16", True),     # NKR 12
        (2, 2, 14, 11, 11, 1, "bf16", True),    # 14 x 11 groups, NKR 13
        (1, 2, 24, 22, 11, 2, "f16", True),     # 12 x 11 groups
        (1, 2, 13, 16, 13, 1, "f16", True),     # NKR 13
        (2, 3, 42, 39, 13, 3, "bf16", True),    # 14 x 13 groups, NKR 14
        (1, 2, 32, 32, 13, 2, "f16", False),    # 16 x 16 groups
        (2, 4, 64, 64, 13, 4, "bf16", True),    # 16 x 16 groups, 3 - 4 units per block
        (8, 8, 64, 64, 9, 4, "f16", True),      # about 7 units per block: the ring wraps twice
        (30, 10, 16, 16, 13, 1, "bf16", True),  # 300 planes of one group: blocks span two planes
        (20, 10, 24, 24, 11, 2, "f16", True),   # 800 units, 5 per block across plane boundaries
    ]
    return [(Shape(B, h, H, W, 32, k, d, dt, 7300 + i), rpb) for i, (B, h, H, W, k, d, dt, rpb) in enumerate(rows)]


@pytest.mark.parametrize("shape,with_rpb", _ugrp_cases(), ids=lambda x: x.describe() if isinstance(x, Shape) else str(x))
def test_ugrp_shapes(shape, with_rpb):
    """The tcgen05 kernel for groups of k .. 16 pixels, every output element."""
    (q, k, v, rpb), got = run_forward(shape, with_rpb)
    assert na.na2d_last_kernel() == "fwd_ugrp_kernel"
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    err = max_err(got, want)
    assert err <= TOL[shape.dtype], f"{shape.describe()} rpb={with_rpb}: max abs err {err}"


@pytest.mark.parametrize("k,d,L", [(3, 1, 3), (7, 1, 7), (13, 1, 13), (7, 2, 14), (13, 2, 26), (5, 8, 40), (13, 9, 117)])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_window_covers_group(k, d, L, dtype):
    """Edge case: every dilation group exactly k long, so every query attends to
    its whole group (dense attention per sub-grid); includes the largest k and
    a large dilation."""
    shape = Shape(2, 2, L, L, 32, k, d, dtype, 77)
    (q, kk, v, rpb), got = run_forward(shape)
    want = oracle.forward(f64(q), f64(kk), f64(v), f64(rpb), k, d)
    assert max_err(got, want) <= TOL[dtype]


def test_full_attention_matches_dense_torch():
    """k = H = W, d = 1, no bias: the GPU result is plain softmax attention,
    compared with a dense fp64 torch computation (not the oracle)."""
    for k, dtype in [(7, "f16"), (13, "bf16"), (7, "f32")]:
        shape = Shape(2, 3, k, k, 32, k, 1, dtype, 91)
        (q, kk, v, _), got = run_forward(shape, with_rpb=False)
        Q, K, V = (t.double().reshape(2, 3, k * k, 32) for t in (q, kk, v))
        P = torch.softmax(Q @ K.transpose(-1, -2) / math.sqrt(32), dim=-1)
        want = (P @ V).reshape(2, 3, k, k, 32).numpy()
        assert max_err(got, want) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("k,d,H,W", [(7, 1, 14, 17), (3, 3, 11, 13), (13, 1, 15, 13), (5, 2, 13, 10)])
def test_split_path(dtype, k, d, H, W):
    """na2d_qk_rpb -> na2d_softmax -> na2d_av, stage by stage against the oracle."""
    shape = Shape(2, 2, H, W, 32, k, d, dtype, 123)
    q, kk, v, rpb = make_inputs(shape)
    qd, kd, vd, rd = (t.cuda() for t in (q, kk, v, rpb))
    attn = na.na2d_qk_rpb(qd, kd, rd, k, d)
    torch.cuda.synchronize()
    ref_scores = oracle.qk_rpb(f64(q), f64(kk), f64(rpb), k, d)
    assert max_err(attn.double().cpu().numpy(), ref_scores) <= 1e-4
    gpu_scores = attn.double().cpu().numpy()
    na.na2d_softmax(attn, k, d)
    torch.cuda.synchronize()
    probs = attn.double().cpu().numpy()
    assert max_err(probs, oracle.softmax(gpu_scores, k, d)) <= 1e-6
    out = na.na2d_av(attn, vd, k, d)
    torch.cuda.synchronize()
    assert max_err(out.double().cpu().numpy(), oracle.av(probs, f64(v), k, d)) <= TOL[dtype]
    # the whole chain against the fused definition
    assert max_err(out.double().cpu().numpy(), oracle.forward(f64(q), f64(kk), f64(v), f64(rpb), k, d)) <= TOL[dtype]


def test_empty_batch():
    x = torch.empty(0, 2, 14, 14, 32, dtype=torch.float16, device="cuda")
    out = na.na2d_forward(x, x, x, None, 7, 1)
    assert out.shape == x.shape


def test_side_stream_and_determinism():
    shape = WORKLOADS["dinat_s1_bf16"].shapes[0]
    q, k, v, rpb = (t.cuda() for t in make_inputs(shape))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = na.na2d_forward(q, k, v, rpb, shape.k, shape.d)
        b = na.na2d_forward(q, k, v, rpb, shape.k, shape.d)
    s.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("shape,kernel", [
    (Shape(2, 2, 56, 56, 32, 7, 8, "bf16", 7401), "fwd_umma_kernel"),
    (Shape(1, 2, 32, 32, 32, 13, 2, "f16", 7402), "fwd_ugrp_kernel"),
    (Shape(2, 2, 28, 28, 32, 7, 1, "bf16", 7403), "fwd_stream_kernel"),
], ids=lambda x: x.describe() if isinstance(x, Shape) else x)
def test_output_only_16_byte_aligned(shape, kernel):
    """An output that starts 16 bytes past a 32-byte boundary takes the kernels'
    16-byte store path; every element still matches the oracle and nothing is
    written outside the output."""
    q, k, v, rpb = make_inputs(shape)
    n, pad = q.numel(), 8   # 8 16-bit elements: 16 bytes
    buf = torch.full((n + 2 * PAD,), SENTINEL, dtype=q.dtype, device="cuda")
    out = buf[PAD + pad:PAD + pad + n].view(q.shape)
    assert out.data_ptr() % 32 == 16
    na.na2d_forward(q.cuda(), k.cuda(), v.cuda(), rpb.cuda(), shape.k, shape.d, out=out)
    torch.cuda.synchronize()
    assert na.na2d_last_kernel() == kernel
    edge = torch.cat([buf[:PAD + pad], buf[PAD + pad + n:]]).float()
    assert bool((edge == float(torch.tensor(SENTINEL, dtype=buf.dtype).float())).all()), "write outside the output"
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    err = max_err(out.double().cpu().numpy(), want)
    assert err <= TOL[shape.dtype], f"{shape.describe()}: max abs err {err}"


@pytest.mark.parametrize("shape,pinned,with_rpb", [
    (Shape(5, 2, 28, 28, 32, 7, 1, "f16", 7501), True, True),     # 5 chunks of one batch element
    (Shape(9, 2, 56, 56, 32, 7, 8, "bf16", 7502), True, True),    # chunks of 2, the last one of 1
    (Shape(3, 2, 14, 14, 32, 5, 2, "f32", 7503), False, False),   # pageable buffers, no bias
    (Shape(1, 4, 32, 32, 32, 13, 2, "bf16", 7504), True, True),   # a single chunk
], ids=lambda x: x.describe() if isinstance(x, Shape) else str(x))
def test_forward_on_host_buffers(shape, pinned, with_rpb):
    """na2d_forward_host: host tensors in, host tensor out, the batch pipelined
    through the device in chunks; every element matches the oracle and the
    device-buffer forward of the same inputs."""
    q, k, v, rpb = make_inputs(shape)
    if not with_rpb:
        rpb = None
    host = [None if t is None else (t.pin_memory() if pinned else t.clone()) for t in (q, k, v, rpb)]
    out = torch.full(q.shape, SENTINEL, dtype=q.dtype)
    out = out.pin_memory() if pinned else out
    na.na2d_forward_host(*host, shape.k, shape.d, out=out)
    torch.cuda.current_stream().synchronize()
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    err = max_err(out.double().numpy(), want)
    assert err <= TOL[shape.dtype], f"{shape.describe()}: max abs err {err}"
    dev = na.na2d_forward(q.cuda(), k.cuda(), v.cuda(), None if rpb is None else rpb.cuda(), shape.k, shape.d)
    torch.cuda.synchronize()
    assert float((out.double() - dev.double().cpu()).abs().max()) <= TOL[shape.dtype]


def test_forward_on_host_buffers_back_to_back():
    """Calls queued back to back on one stream (the host does not wait in
    between) each see their own inputs and write their own outputs."""
    shape = Shape(6, 2, 28, 28, 32, 7, 1, "f16", 7510)
    sets = [make_inputs(shape, shape.seed + i) for i in range(3)]
    pinned = [[t.pin_memory() for t in s] for s in sets]
    outs = [torch.empty(sets[0][0].shape, dtype=torch.float16).pin_memory() for _ in sets]
    ws = torch.empty(na.na2d_forward_host_workspace_size(sets[0][0].shape, 7, 1, torch.float16),
                     dtype=torch.uint8, device="cuda")
    for (q, k, v, rpb), o in zip(pinned, outs):
        na.na2d_forward_host(q, k, v, rpb, 7, 1, out=o, workspace=ws)
    torch.cuda.current_stream().synchronize()
    for (q, k, v, rpb), o in zip(sets, outs):
        want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), 7, 1)
        assert max_err(o.double().numpy(), want) <= TOL["f16"]


def test_misaligned_tensor_is_rejected():
    q = torch.zeros(2 * 14 * 14 * 32 + 4, dtype=torch.float16, device="cuda")[4:].view(1, 2, 14, 14, 32)
    with pytest.raises(na.Na2dError) as e:
        na.na2d_forward(q, q, q, None, 7, 1, out=torch.empty(1, 2, 14, 14, 32, dtype=torch.float16, device="cuda"))
    assert e.value.status == 6


@pytest.mark.parametrize("name", ["nat_tiny_s1_fp16", "dinat_s1_bf16"])
def test_bench_buffers_sampled(name):
    """The benchmark's rotating input sets (seeds shape.seed + 1000 r), as the
    benchmark calls them, checked at sampled queries including all four corners."""
    shape = WORKLOADS[name].shapes[0]
    rnd = random.Random(9)
    for r in (1, 3):
        q, k, v, rpb = make_inputs(shape, shape.seed + 1000 * r)
        out = na.na2d_forward(q.cuda(), k.cuda(), v.cuda(), rpb.cuda(), shape.k, shape.d).double().cpu().numpy()
        pts = [(0, 0, 0, 0), (shape.B - 1, shape.heads - 1, shape.H - 1, shape.W - 1),
               (0, 1, 0, shape.W - 1), (1, 0, shape.H - 1, 0)]
        pts += [(rnd.randrange(shape.B), rnd.randrange(shape.heads), rnd.randrange(shape.H), rnd.randrange(shape.W))
                for _ in range(60)]
        q64, k64, v64, r64 = f64(q), f64(k), f64(v), f64(rpb)
        for (b, h, i, j) in pts:
            want = oracle.forward_query(q64, k64, v64, r64, shape.k, shape.d, b, h, i, j)
            assert float(np.abs(out[b, h, i, j] - want).max()) <= TOL[shape.dtype]


# ---------------------------------------------------------------------------
# Dispatch: which kernel each kind of problem reaches (na2d_last_kernel), with
# parity.  Every branch of na2d_forward's dispatch has a row here.
DISPATCH = [
    (Shape(1, 3, 14, 14, 32, 7, 2, "bf16", 601), "fwd_umma_kernel"),            # every group exactly 7 x 7
    (Shape(1, 2, 16, 16, 32, 7, 1, "f16", 602), "fwd_stream_kernel"),           # k = 7 sliding rows
    (Shape(1, 2, 12, 100, 32, 7, 1, "bf16", 613), "fwd_stream_kernel"),         # k = 7 sliding rows, column bands
    (Shape(1, 2, 28, 28, 32, 7, 2, "bf16", 603), "fwd_sync_kernel/full_tma"),   # k <= 7, equal groups >= 14 long
    (Shape(1, 2, 12, 12, 32, 3, 1, "f16", 604), "fwd_sync_kernel/full_tma"),
    (Shape(1, 2, 6, 6, 32, 3, 2, "bf16", 605), "fwd_sync_kernel/dense_tma"),    # k <= 5, every group exactly k
    (Shape(1, 2, 30, 30, 32, 9, 1, "f16", 606), "fwd_tc_kernel/full"),          # k >= 9, long groups
    (Shape(1, 2, 13, 13, 32, 13, 1, "bf16", 607), "fwd_ugrp_kernel"),           # k >= 9, groups k .. 16 long
    (Shape(1, 2, 32, 32, 32, 13, 2, "f16", 614), "fwd_ugrp_kernel"),
    (Shape(1, 2, 20, 18, 32, 7, 2, "bf16", 608), "fwd_tc_kernel/generic"),      # short groups
    (Shape(1, 2, 23, 19, 32, 5, 2, "f16", 609), "fwd_tc_kernel/full"),          # ragged groups (H, W not multiples of d)
    (Shape(1, 2, 15, 17, 32, 5, 2, "bf16", 612), "fwd_tc_kernel/generic"),      # ragged short groups
    (Shape(1, 2, 14, 14, 32, 7, 1, "f32", 610), "fwd_simt_kernel"),             # fp32
    (Shape(1, 2, 5, 6, 32, 1, 1, "f16", 611), "fwd_simt_kernel"),               # k = 1
]


@pytest.mark.parametrize("shape,kernel", DISPATCH, ids=[f"{k}:{s.describe()}" for s, k in DISPATCH])
def test_dispatch_table(shape, kernel):
    (q, k, v, rpb), got = run_forward(shape)
    assert na.na2d_last_kernel() == kernel
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), shape.k, shape.d)
    assert max_err(got, want) <= TOL[shape.dtype]


def _chain_cases():
    return [s for s, _ in DISPATCH[:3]] + [DISPATCH[5][0], DISPATCH[7][0], DISPATCH[9][0]]


@pytest.mark.parametrize("graph", [False, True], ids=["eager", "graph"])
@pytest.mark.parametrize("shape", _chain_cases(), ids=lambda s: s.describe())
def test_chained_calls_same_stream(shape, graph):
    """out1 = f(q, k, v); out2 = f(out1, k, v); out3 = f(out2, k, v), queued on
    one stream with no host synchronisation (and, in the graph variant,
    captured in one CUDA graph).  The streaming and tcgen05 kernels are
    launched with programmatic stream serialisation; a global read placed
    before their wait for the previous grid would read a stale out1 / out2
    here.  Each output is checked against the oracle applied to the previous
    GPU output."""
    q, k, v, rpb = make_inputs(shape)
    qd, kd, vd, rd = (t.cuda() for t in (q, k, v, rpb))
    outs = [torch.full_like(qd, float("nan")) for _ in range(3)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def chain():
        x = qd
        for o in outs:
            na.na2d_forward(x, kd, vd, rd, shape.k, shape.d, out=o)
            x = o

    with torch.cuda.stream(s):
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                chain()
            for o in outs:
                o.fill_(float("nan"))
            g.replay()
        else:
            chain()
    s.synchronize()
    prev = q
    for o in outs:
        got = o.cpu()
        want = oracle.forward(f64(prev), f64(k), f64(v), f64(rpb), shape.k, shape.d)
        assert max_err(got.double().numpy(), want) <= TOL[shape.dtype]
        prev = got


def test_bounded_wait_error_path_runs_out_and_recovers():
    """The error path of the bounded waits, run on purpose without any fault:
    with the streaming kernel's wait limit cut to 200 SM clocks, a CTA with
    several steps cannot see its stages released in time (the consumers need
    microseconds for their first step, the producer reaches the wait for the
    fourth stage at once); the kernel must count the event, drain its copies
    in flight and return.  The count is then non-zero, and with the default
    limit restored the next call is correct and counts nothing."""
    from neighborhood_attention_na2d_b200 import _native
    shape = Shape(32, 2, 56, 56, 32, 7, 1, "f16", 1701)   # 14 query-row pairs (7 steps) per CTA
    q, k, v, rpb = make_inputs(shape)
    qd, kd, vd, rd = (t.cuda() for t in (q, k, v, rpb))
    assert na.na2d_device_faults() == 0
    try:
        _native.lib().na2d_debug_set_wait_limit(200)
        na.na2d_forward(qd, kd, vd, rd, 7, 1)
        assert na.na2d_last_kernel() == "fwd_stream_kernel"
        assert na.na2d_device_faults() > 0
    finally:
        _native.lib().na2d_debug_set_wait_limit(0)
    out = na.na2d_forward(qd, kd, vd, rd, 7, 1)
    torch.cuda.synchronize()
    assert na.na2d_device_faults() == 0
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), 7, 1)
    assert max_err(out.double().cpu().numpy(), want) <= TOL["f16"]


def test_bounded_wait_error_path_tcgen05_groups():
    """The same error path in the tcgen05 kernel for groups of up to 16 x 16
    pixels: with the wait limit cut to 200 SM clocks the MMA warps' wait for
    the first 48 KB copy and the softmax warps' wait for the first scores run
    out; the kernel counts the event, waits for its copies and products in
    flight, releases its tensor memory and returns.  With the default limit
    restored the next call is correct and counts nothing."""
    from neighborhood_attention_na2d_b200 import _native
    shape = Shape(2, 4, 128, 128, 32, 13, 8, "bf16", 1702)
    q, k, v, rpb = make_inputs(shape)
    qd, kd, vd, rd = (t.cuda() for t in (q, k, v, rpb))
    assert na.na2d_device_faults() == 0
    try:
        _native.lib().na2d_debug_set_wait_limit(200)
        na.na2d_forward(qd, kd, vd, rd, 13, 8)
        assert na.na2d_last_kernel() == "fwd_ugrp_kernel"
        assert na.na2d_device_faults() > 0
    finally:
        _native.lib().na2d_debug_set_wait_limit(0)
    out = na.na2d_forward(qd, kd, vd, rd, 13, 8)
    torch.cuda.synchronize()
    assert na.na2d_device_faults() == 0
    want = oracle.forward(f64(q), f64(k), f64(v), f64(rpb), 13, 8)
    assert max_err(out.double().cpu().numpy(), want) <= TOL["bf16"]


def test_no_device_wait_timed_out():
    """Runs after the parity tests above (same module): no kernel gave up on a
    bounded wait."""
    assert na.na2d_device_faults() == 0
