"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch.  ``test_oracle_pins.py`` runs them on the real oracle;
``test_oracle_mutants.py`` runs them on copies of the C source with planted
mistakes and requires every mutant to fail at least one pin.

What fixes each expected value (never the oracle's own formula retyped):
  * full self attention when the window covers the image (dense numpy softmax
    attention) -- "Neighborhood Attention Transformer" README, figure caption;
  * the brute-force search formulation in ``brute.py`` (nearest window found by
    search, explicit Python loops) -- same caption ("nearest neighborhood",
    "edges are special cases");
  * the window key-set properties (k distinct keys, inside the query's dilation
    group, contiguous there, containing the query) -- DiNA "every d-th pixel",
    the fixed key count noted in the gitcode DiNAT article ("DiNAT 的核心思想");
  * dilation = plain NA on the d x d interleaved sub-grids;
  * softmax invariants and closed forms (uniform weights -> window mean,
    constant values -> that constant, bias shift -> no change);
  * a one-hot bias with zero q, k: closed form of the weights, which fixes the
    bias table's orientation (row = vertical offset key' - i' + k - 1);
  * translation equivariance of unclamped queries (NA abstract, HF NAT page);
  * the pages' DiNAT stage table (tests/golden/dinat_stage_table.txt);
  * backward: central finite differences of the (pinned) forward, exhaustively
    on tiny maps; gradients of dense softmax attention from torch autograd in
    fp64 when the window covers the image; calculus identities (softmax
    gradients sum to zero, so every head's bias gradient sums to zero; the
    weights sum to one, so the value gradients sum to the output gradients);
    the dilation decomposition carried over to the gradients;
  * dropout: the generator's published known-answer values
    (tests/golden/philox4x32_10_kat.txt); p = 0 equals the plain forward; kept
    weights equal the (pinned) softmax weights / (1 - p) and dropped ones are
    zero, at the positions an independent Python restatement of the generator
    selects; the returned weights reproduce the output through the pinned
    weighted-sum stage; the keep rate is 1 - p within 5 sigma; the backward
    equals finite differences of the forward with the mask fixed;
  * maps shorter than k * d (zero padding, then crop): unchanged when no
    padding is needed; dense attention over the zero-padded map when the
    padded window covers it; with q = 0 and no bias, the mean of v over the
    searched window counting padded pixels as zeros; the backward equals
    finite differences.
"""
from __future__ import annotations

import math
import random
from pathlib import Path

import numpy as np

from brute import axis_window_search, forward_brute

GOLDEN = Path(__file__).resolve().parent / "golden"
TOL = 1e-12


def _rand(rng: np.random.Generator, B, heads, H, W, D, k, with_rpb=True):
    q = rng.standard_normal((B, heads, H, W, D))
    kk = rng.standard_normal((B, heads, H, W, D))
    v = rng.standard_normal((B, heads, H, W, D))
    rpb = rng.standard_normal((heads, 2 * k - 1, 2 * k - 1)) * 0.5 if with_rpb else None
    return q, kk, v, rpb


def dense_attention(q, kk, v, bias=None):
    """softmax(Q K^T / sqrt(D) + bias) V over all pixels of each (b, head) map."""
    B, heads, H, W, D = q.shape
    Q = q.reshape(B, heads, H * W, D)
    K = kk.reshape(B, heads, H * W, D)
    V = v.reshape(B, heads, H * W, D)
    S = Q @ np.swapaxes(K, -1, -2) / math.sqrt(D)
    if bias is not None:
        S = S + bias
    S = S - S.max(axis=-1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(axis=-1, keepdims=True)
    return (P @ V).reshape(B, heads, H, W, D)


def read_stage_table():
    rows = []
    for line in (GOLDEN / "dinat_stage_table.txt").read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        stage, depth, kernel, dil, spans, heads, res = line.split()
        rows.append(dict(stage=int(stage), depth=int(depth), kernel=int(kernel),
                         dilations=[int(x) for x in dil.split(",")],
                         spans=[int(x) for x in spans.split(",")],
                         heads=int(heads), resolution=int(res)))
    return rows


def axis_cases():
    """(L, k, d) triples: every workload axis plus a seeded random sweep."""
    cases = {(14, 7, 1), (56, 7, 1), (56, 7, 8), (28, 7, 1), (28, 7, 4), (14, 7, 2), (7, 7, 1),
             (128, 13, 1), (128, 13, 8), (128, 7, 1), (9, 3, 3), (6, 3, 2), (3, 3, 1)}
    rnd = random.Random(7)
    while len(cases) < 120:
        k = rnd.choice([1, 3, 5, 7, 9, 11, 13])
        d = rnd.randint(1, 9)
        L = rnd.randint(k * d, k * d + 3 * d + 5)
        cases.add((L, k, d))
    return sorted(cases)


# ---------------------------------------------------------------------------
def pin_window_keyset(orc):
    """k distinct keys per axis (k*k in 2D), all in the query's dilation group,
    consecutive members of it, containing the query, bias index key'-i'+k-1 in
    [0, 2k-2], and equal to the nearest window found by search."""
    for L, k, d in axis_cases():
        for i in range(L):
            keys, bidx = orc.axis_neighbors(L, k, d, i)
            assert len(set(keys)) == k, (L, k, d, i, keys)
            assert all(0 <= x < L for x in keys), (L, k, d, i, keys)
            assert all(x % d == i % d for x in keys), (L, k, d, i, keys)
            assert i in keys, (L, k, d, i, keys)
            assert all(b - a == d for a, b in zip(keys, keys[1:])), (L, k, d, i, keys)
            assert all(0 <= b <= 2 * k - 2 for b in bidx), (L, k, d, i, bidx)
            skeys, srel = axis_window_search(L, k, d, i)
            assert keys == skeys, (L, k, d, i, keys, skeys)
            assert bidx == srel, (L, k, d, i, bidx, srel)


def pin_full_attention(orc):
    """k = H = W, d = 1: every query sees the whole image, so NA is dense self
    attention (no bias); with H = W = k*d the same holds on each sub-grid."""
    rng = np.random.default_rng(11)
    for k in (1, 3, 5, 7):
        q, kk, v, _ = _rand(rng, 2, 2, k, k, 8, k, with_rpb=False)
        got = orc.forward(q, kk, v, None, k, 1)
        np.testing.assert_allclose(got, dense_attention(q, kk, v), rtol=0, atol=TOL)
    for k, d in ((3, 2), (3, 3), (5, 2)):
        L = k * d
        q, kk, v, _ = _rand(rng, 1, 2, L, L, 4, k, with_rpb=False)
        got = orc.forward(q, kk, v, None, k, d)
        for gy in range(d):
            for gx in range(d):
                sub = [a[:, :, gy::d, gx::d] for a in (q, kk, v)]
                np.testing.assert_allclose(got[:, :, gy::d, gx::d], dense_attention(*sub), rtol=0, atol=TOL)


def pin_brute_force(orc):
    """Tiny maps, with bias: the oracle equals the search formulation."""
    rng = np.random.default_rng(12)
    cases = [(5, 5, 1, 1), (6, 7, 3, 1), (7, 6, 3, 2), (9, 9, 3, 3), (10, 11, 5, 2), (8, 8, 5, 1),
             (9, 6, 3, 2), (12, 10, 3, 3), (7, 7, 7, 1)]
    for H, W, k, d in cases:
        q, kk, v, rpb = _rand(rng, 1, 2, H, W, 3, k)
        got = orc.forward(q, kk, v, rpb, k, d)
        want = np.array(forward_brute(q.tolist(), kk.tolist(), v.tolist(), rpb.tolist(), k, d))
        np.testing.assert_allclose(got, want, rtol=0, atol=TOL, err_msg=str((H, W, k, d)))


def pin_dilation_decomposition(orc):
    """NA(x; k, d) equals the d x d interleave of NA(x[gy::d, gx::d]; k, 1)."""
    rng = np.random.default_rng(13)
    for H, W, k, d in [(14, 14, 3, 2), (15, 13, 3, 2), (21, 23, 5, 3), (16, 16, 7, 2), (24, 17, 3, 4)]:
        q, kk, v, rpb = _rand(rng, 1, 2, H, W, 4, k)
        got = orc.forward(q, kk, v, rpb, k, d)
        for gy in range(d):
            for gx in range(d):
                sub = [np.ascontiguousarray(a[:, :, gy::d, gx::d]) for a in (q, kk, v)]
                want = orc.forward(*sub, rpb, k, 1)
                np.testing.assert_allclose(got[:, :, gy::d, gx::d], want, rtol=0, atol=TOL)


def pin_invariants(orc):
    """Softmax closed forms: a constant added to the bias changes nothing;
    constant values come back unchanged; q = 0 and no bias give the plain mean
    of v over the window (window from the search formulation)."""
    rng = np.random.default_rng(14)
    H, W, k, d = 11, 9, 3, 2
    q, kk, v, rpb = _rand(rng, 2, 2, H, W, 4, k)
    base = orc.forward(q, kk, v, rpb, k, d)
    np.testing.assert_allclose(orc.forward(q, kk, v, rpb + 3.25, k, d), base, rtol=0, atol=1e-11)
    const = np.broadcast_to(np.array([1.5, -2.0, 0.25, 7.0]), v.shape).copy()
    np.testing.assert_allclose(orc.forward(q, kk, const, rpb, k, d), const, rtol=0, atol=1e-12)
    got = orc.forward(np.zeros_like(q), kk, v, None, k, d)
    for i in range(H):
        ky, _ = axis_window_search(H, k, d, i)
        for j in range(W):
            kx, _ = axis_window_search(W, k, d, j)
            want = v[:, :, ky][:, :, :, kx].mean(axis=(2, 3))
            np.testing.assert_allclose(got[:, :, i, j], want, rtol=0, atol=TOL)


def pin_rpb_orientation(orc):
    """q = k = 0 and a single non-zero bias entry rpb[h, a, b] = beta: the key at
    group offset (a - (k-1), b - (k-1)) from the query, if in its window, gets
    weight e^beta / (k^2 - 1 + e^beta) and every other key 1 / (same); v holds
    each pixel's (row, col), so the output is a closed-form weighted mean."""
    H, W, k, d, beta = 9, 8, 3, 2, 1.75
    z = np.zeros((1, 1, H, W, 2))
    v = np.zeros((1, 1, H, W, 2))
    for y in range(H):
        for x in range(W):
            v[0, 0, y, x] = (y, x)
    for a in range(2 * k - 1):
        for b in range(2 * k - 1):
            rpb = np.zeros((1, 2 * k - 1, 2 * k - 1))
            rpb[0, a, b] = beta
            got = orc.forward(z, z, v, rpb, k, d)
            for i in range(H):
                ky, ry = axis_window_search(H, k, d, i)
                for j in range(W):
                    kx, rx = axis_window_search(W, k, d, j)
                    w = np.array([[math.exp(beta) if (ry[p] == a and rx[c] == b) else 1.0
                                   for c in range(k)] for p in range(k)])
                    w /= w.sum()
                    want = (w[:, :, None] * v[0, 0][np.ix_(ky, kx)]).sum(axis=(0, 1))
                    np.testing.assert_allclose(got[0, 0, i, j], want, rtol=0, atol=TOL,
                                               err_msg=str((a, b, i, j)))


def pin_translation(orc):
    """Shifting the inputs by d pixels along an axis shifts the output of every
    query whose window along that axis is unclamped in both frames
    (translational equivariance)."""
    rng = np.random.default_rng(15)
    for H, W, k, d in [(16, 15, 3, 1), (20, 21, 3, 2), (24, 24, 5, 2)]:
        q, kk, v, rpb = _rand(rng, 1, 1, H, W, 4, k)
        base = orc.forward(q, kk, v, rpb, k, d)
        r = k // 2
        for axis, L in ((2, H), (3, W)):
            moved = orc.forward(*[np.roll(a, d, axis=axis) for a in (q, kk, v)], rpb, k, d)
            idx = [i for i in range(L - d)
                   if i // d - r >= 0 and i // d + 1 + r <= (L - i % d + d - 1) // d - 1]
            assert idx, (H, W, k, d, axis)
            np.testing.assert_allclose(np.take(moved, [i + d for i in idx], axis=axis),
                                       np.take(base, idx, axis=axis), rtol=0, atol=TOL)


def pin_split_stages(orc):
    """Scores equal explicit dot products plus bias on the searched window;
    softmax rows are exp(s - max) / sum; av(softmax(qk_rpb)) equals forward."""
    rng = np.random.default_rng(16)
    H, W, k, d, D = 10, 9, 3, 2, 5
    q, kk, v, rpb = _rand(rng, 1, 2, H, W, D, k)
    attn = orc.qk_rpb(q, kk, rpb, k, d)
    for h in range(2):
        for i in range(H):
            ky, ry = axis_window_search(H, k, d, i)
            for j in range(W):
                kx, rx = axis_window_search(W, k, d, j)
                want = [sum(q[0, h, i, j, e] * kk[0, h, y, x, e] for e in range(D)) / math.sqrt(D)
                        + rpb[h, ry[a], rx[c]] for a, y in enumerate(ky) for c, x in enumerate(kx)]
                np.testing.assert_allclose(attn[0, h, i, j], want, rtol=0, atol=TOL)
    p = orc.softmax(attn, k, d, D)
    e = np.exp(attn - attn.max(axis=-1, keepdims=True))
    np.testing.assert_allclose(p, e / e.sum(axis=-1, keepdims=True), rtol=0, atol=TOL)
    np.testing.assert_allclose(orc.av(p, v, k, d), orc.forward(q, kk, v, rpb, k, d), rtol=0, atol=TOL)
    # av alone: one-hot weights pick out exactly the searched key's value
    onehot = np.zeros_like(p)
    onehot[..., k * k - 1] = 1.0
    got = orc.av(onehot, v, k, d)
    for i in range(H):
        ky, _ = axis_window_search(H, k, d, i)
        for j in range(W):
            kx, _ = axis_window_search(W, k, d, j)
            np.testing.assert_allclose(got[0, :, i, j], v[0, :, ky[-1], kx[-1]], rtol=0, atol=TOL)


def pin_stage_table(orc):
    """The pages' DiNAT stage table: span = kernel x dilation; on a map of side
    span every dilated layer's window is the query's whole dilation group, so
    the layer is dense attention on each sub-grid."""
    rng = np.random.default_rng(17)
    rows = read_stage_table()
    assert [r["stage"] for r in rows] == [1, 2, 3, 4]
    for r in rows:
        k = r["kernel"]
        assert len(r["dilations"]) == r["depth"] == len(r["spans"])
        assert max(r["spans"]) == r["resolution"]
        for d, span in zip(r["dilations"], r["spans"]):
            assert span == k * d
            for i in range(span):
                keys, _ = orc.axis_neighbors(span, k, d, i)
                assert keys == list(range(i % d, span, d))
        d = max(r["dilations"])
        L = r["resolution"]
        q, kk, v, _ = _rand(rng, 1, 1, L, L, 4, k, with_rpb=False)
        got = orc.forward(q, kk, v, None, k, d)
        for gy in range(d):
            for gx in range(d):
                sub = [a[:, :, gy::d, gx::d] for a in (q, kk, v)]
                np.testing.assert_allclose(got[:, :, gy::d, gx::d], dense_attention(*sub), rtol=0, atol=TOL)


def pin_forward_query(orc):
    """The per-query numpy path equals the fused C path at sampled queries."""
    rng = np.random.default_rng(18)
    H, W, k, d = 17, 19, 5, 3
    q, kk, v, rpb = _rand(rng, 2, 3, H, W, 6, k)
    full = orc.forward(q, kk, v, rpb, k, d)
    for (b, h, i, j) in [(0, 0, 0, 0), (1, 2, 16, 18), (0, 1, 8, 9), (1, 0, 3, 17), (0, 2, 15, 1)]:
        np.testing.assert_allclose(orc.forward_query(q, kk, v, rpb, k, d, b, h, i, j), full[b, h, i, j],
                                   rtol=0, atol=TOL)


# ---------------------------------------------------------------------------
# Backward.
def _loss(orc, q, kk, v, rpb, dout, k, d):
    return float((orc.forward(q, kk, v, rpb, k, d) * dout).sum())


def pin_backward_finite_differences(orc):
    """Every entry of dq, dk, dv and drpb equals the central difference of
    L = sum(dout * forward) with step 1e-5 (error O(1e-10)), on tiny maps with
    clamped edges and dilation."""
    rng = np.random.default_rng(21)
    for (B, heads, H, W, D, k, d) in [(1, 2, 5, 6, 3, 3, 1), (1, 1, 7, 6, 2, 3, 2), (2, 1, 5, 5, 2, 5, 1)]:
        q, kk, v, rpb = _rand(rng, B, heads, H, W, D, k)
        dout = rng.standard_normal(q.shape)
        dq, dk, dv, drpb = orc.backward(q, kk, v, rpb, dout, k, d)
        eps = 1e-5
        for name, x, grad in (("q", q, dq), ("k", kk, dk), ("v", v, dv), ("rpb", rpb, drpb)):
            num = np.empty_like(x)
            flat, nflat = x.reshape(-1), num.reshape(-1)
            for e in range(flat.size):
                old = flat[e]
                flat[e] = old + eps
                up = _loss(orc, q, kk, v, rpb, dout, k, d)
                flat[e] = old - eps
                dn = _loss(orc, q, kk, v, rpb, dout, k, d)
                flat[e] = old
                nflat[e] = (up - dn) / (2 * eps)
            np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-7, err_msg=f"d{name} {(H, W, k, d)}")


def pin_backward_dense_autograd(orc):
    """k = H = W, d = 1: NA is dense softmax attention with the bias matrix
    Bias[(iy, ix), (jy, jx)] = rpb[h, jy - iy + k - 1, jx - ix + k - 1]; its
    gradients come from torch autograd (fp64), not from the oracle."""
    import torch
    rng = np.random.default_rng(22)
    for k in (3, 5):
        B, heads, D = 2, 2, 4
        q, kk, v, rpb = _rand(rng, B, heads, k, k, D, k)
        dout = rng.standard_normal(q.shape)
        T = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, kk, v, rpb)]
        iy, ix = np.divmod(np.arange(k * k), k)
        ry = torch.tensor(iy[None, :] - iy[:, None] + k - 1)
        rx = torch.tensor(ix[None, :] - ix[:, None] + k - 1)
        bias = T[3][:, ry, rx]                                   # [heads, k*k, k*k]
        Q, K, V = (t.reshape(B, heads, k * k, D) for t in T[:3])
        S = Q @ K.transpose(-1, -2) / math.sqrt(D) + bias
        O = torch.softmax(S, dim=-1) @ V
        O.reshape(q.shape).backward(torch.tensor(dout))
        got = orc.backward(q, kk, v, rpb, dout, k, 1)
        for g, t in zip(got, T):
            np.testing.assert_allclose(g, t.grad.numpy(), rtol=0, atol=1e-11)


def pin_backward_identities(orc):
    """Softmax gradients sum to zero over a window, so each head's bias
    gradient sums to zero; the weights of every window sum to one, so per
    (b, head) the value gradients sum to the output gradients; with q = 0
    and no bias (uniform weights) dv at a key is dout summed over the queries
    whose (searched) window holds it, divided by k*k."""
    rng = np.random.default_rng(23)
    H, W, k, d = 9, 11, 3, 2
    q, kk, v, rpb = _rand(rng, 2, 3, H, W, 4, k)
    dout = rng.standard_normal(q.shape)
    dq, dk, dv, drpb = orc.backward(q, kk, v, rpb, dout, k, d)
    np.testing.assert_allclose(drpb.sum(axis=(1, 2)), 0.0, rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv.sum(axis=(2, 3)), dout.sum(axis=(2, 3)), rtol=0, atol=1e-11)
    _, _, dv0, _ = orc.backward(np.zeros_like(q), kk, v, None, dout, k, d)
    want = np.zeros_like(dv0)
    for i in range(H):
        ky, _ = axis_window_search(H, k, d, i)
        for j in range(W):
            kx, _ = axis_window_search(W, k, d, j)
            for y in ky:
                for x in kx:
                    want[:, :, y, x] += dout[:, :, i, j] / (k * k)
    np.testing.assert_allclose(dv0, want, rtol=0, atol=1e-12)


def pin_backward_dilation_decomposition(orc):
    """Gradients of NA(x; k, d) are the d x d interleave of the gradients of
    NA(x[gy::d, gx::d]; k, 1); the bias gradient is their sum."""
    rng = np.random.default_rng(24)
    for H, W, k, d in [(14, 13, 3, 2), (16, 16, 5, 3)]:
        q, kk, v, rpb = _rand(rng, 1, 2, H, W, 3, k)
        dout = rng.standard_normal(q.shape)
        got = orc.backward(q, kk, v, rpb, dout, k, d)
        drpb_sum = np.zeros_like(got[3])
        for gy in range(d):
            for gx in range(d):
                sub = [np.ascontiguousarray(a[:, :, gy::d, gx::d]) for a in (q, kk, v, dout)]
                want = orc.backward(sub[0], sub[1], sub[2], rpb, sub[3], k, 1)
                for g, w in zip(got[:3], want[:3]):
                    np.testing.assert_allclose(g[:, :, gy::d, gx::d], w, rtol=0, atol=TOL)
                drpb_sum += want[3]
        np.testing.assert_allclose(got[3], drpb_sum, rtol=0, atol=1e-11)


# ---------------------------------------------------------------------------
# Dropout.
def _philox_py(ctr, key):
    """Philox4x32-10 restated from its publication (SC 2011), independent of
    the oracle's C: 10 rounds, multipliers 0xD2511F53 / 0xCD9E8D57, Weyl key
    increments 0x9E3779B9 / 0xBB67AE85."""
    c, k = list(ctr), list(key)
    for r in range(10):
        if r:
            k = [(k[0] + 0x9E3779B9) & 0xFFFFFFFF, (k[1] + 0xBB67AE85) & 0xFFFFFFFF]
        p0, p1 = 0xD2511F53 * c[0], 0xCD9E8D57 * c[2]
        c = [((p1 >> 32) ^ c[1] ^ k[0]) & 0xFFFFFFFF, p1 & 0xFFFFFFFF, ((p0 >> 32) ^ c[3] ^ k[1]) & 0xFFFFFFFF,
             p0 & 0xFFFFFFFF]
    return c


def _keep_py(e, p, seed, offset):
    blk = e >> 2
    w = _philox_py((blk & 0xFFFFFFFF, blk >> 32, offset & 0xFFFFFFFF, offset >> 32),
                   (seed & 0xFFFFFFFF, seed >> 32))[e & 3]
    t = float(np.float32(p)) * 4294967296.0
    thresh = 0xFFFFFFFF if t >= 4294967295.0 else int(t + 0.5)
    return w >= thresh


def pin_philox_kat(orc):
    """The oracle's generator reproduces the published known-answer values."""
    for line in (GOLDEN / "philox4x32_10_kat.txt").read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        x = [int(t, 16) for t in line.split()]
        assert orc.philox(x[0:4], x[4:6]) == x[6:10], line
        assert _philox_py(x[0:4], x[4:6]) == x[6:10], line


def pin_dropout(orc):
    """Dropout between softmax and the weighted sum, and the returned weights."""
    rng = np.random.default_rng(31)
    H, W, k, d, D = 9, 10, 3, 2, 4
    q, kk, v, rpb = _rand(rng, 2, 2, H, W, D, k)
    base = orc.forward(q, kk, v, rpb, k, d)
    out0, a0 = orc.forward_ex(q, kk, v, rpb, k, d, 0.0, 7, 0, return_attn=True)
    np.testing.assert_allclose(out0, base, rtol=0, atol=TOL)
    soft = orc.softmax(orc.qk_rpb(q, kk, rpb, k, d), k, d, D)
    np.testing.assert_allclose(a0, soft, rtol=0, atol=TOL)
    p, seed, offset = 0.3, (5 << 33) + 11, 3
    out, a = orc.forward_ex(q, kk, v, rpb, k, d, p, seed, offset, return_attn=True)
    np.testing.assert_allclose(orc.av(a, v, k, d), out, rtol=0, atol=TOL)
    keep = np.array([_keep_py(e, p, seed, offset) for e in range(a.size)]).reshape(a.shape)
    scale = 1.0 / (1.0 - float(np.float32(p)))
    np.testing.assert_allclose(a, np.where(keep, soft * scale, 0.0), rtol=0, atol=TOL)
    # keep rate over many weights
    big = np.zeros((1, 1, 60, 60, 1))
    _, ab = orc.forward_ex(big, big, big, None, 7, 1, 0.25, 123, 0, return_attn=True)
    frac = float((ab > 0).mean())
    n = ab.size
    assert abs(frac - 0.75) < 5 * math.sqrt(0.75 * 0.25 / n), frac


def pin_dropout_backward(orc):
    """With the mask fixed by (seed, offset), the dropout forward is a smooth
    function of q, k, v, rpb; its gradients equal central differences."""
    rng = np.random.default_rng(32)
    B, heads, H, W, D, k, d = 1, 2, 5, 6, 2, 3, 1
    q, kk, v, rpb = _rand(rng, B, heads, H, W, D, k)
    dout = rng.standard_normal(q.shape)
    p, seed = 0.35, 99
    got = orc.backward_ex(q, kk, v, rpb, dout, k, d, p, seed, 0)
    eps = 1e-5

    def loss():
        return float((orc.forward_ex(q, kk, v, rpb, k, d, p, seed, 0) * dout).sum())

    for name, x, grad in (("q", q, got[0]), ("k", kk, got[1]), ("v", v, got[2]), ("rpb", rpb, got[3])):
        flat, num = x.reshape(-1), np.empty(x.size)
        for e in range(flat.size):
            old = flat[e]
            flat[e] = old + eps
            up = loss()
            flat[e] = old - eps
            dn = loss()
            flat[e] = old
            num[e] = (up - dn) / (2 * eps)
        np.testing.assert_allclose(grad.reshape(-1), num, rtol=1e-6, atol=1e-7, err_msg=f"d{name}")
    # p = 0: the plain backward
    for g0, g1 in zip(orc.backward_ex(q, kk, v, rpb, dout, k, d, 0.0, seed, 0),
                      orc.backward(q, kk, v, rpb, dout, k, d)):
        np.testing.assert_allclose(g0, g1, rtol=0, atol=1e-12)
    # a map shorter than k * d: without dropout, the padded forward/backward;
    # with dropout, weights numbered over the real map (the mask of weight
    # (b, h, i, j, n) does not depend on the padding)
    H2, W2, k2, d2 = 4, 5, 3, 2
    q2, k2_, v2, r2 = _rand(rng, 1, 2, H2, W2, 3, k2)
    g2 = rng.standard_normal(q2.shape)
    np.testing.assert_allclose(orc.forward_ex(q2, k2_, v2, r2, k2, d2), orc.forward_padded(q2, k2_, v2, r2, k2, d2),
                               rtol=0, atol=TOL)
    for a, b in zip(orc.backward_ex(q2, k2_, v2, r2, g2, k2, d2), orc.backward_padded(q2, k2_, v2, r2, g2, k2, d2)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    _, a2 = orc.forward_ex(q2, k2_, v2, r2, k2, d2, 0.4, 17, 2, return_attn=True)
    keep = np.array([_keep_py(e, 0.4, 17, 2) for e in range(a2.size)]).reshape(a2.shape)
    assert np.array_equal(a2 > 0, keep)


# ---------------------------------------------------------------------------
# Maps shorter than k * d.
def pin_padding(orc):
    rng = np.random.default_rng(33)
    # no padding needed: unchanged
    q, kk, v, rpb = _rand(rng, 1, 2, 9, 8, 3, 3)
    np.testing.assert_allclose(orc.forward_padded(q, kk, v, rpb, 3, 2), orc.forward(q, kk, v, rpb, 3, 2),
                               rtol=0, atol=TOL)
    # d = 1, H, W < k: every padded window is the whole k x k padded map, so
    # the real queries see dense attention over it (bias by relative offset)
    k = 5
    for (H, W) in [(3, 4), (5, 2), (1, 1)]:
        q, kk, v, rpb = _rand(rng, 1, 2, H, W, 4, k)
        pads = ((0, 0), (0, 0), (0, k - H), (0, k - W), (0, 0))
        Q, K, V = (np.pad(a, pads) for a in (q, kk, v))
        iy, ix = np.divmod(np.arange(k * k), k)
        bias = rpb[:, iy[None, :] - iy[:, None] + k - 1, ix[None, :] - ix[:, None] + k - 1][None]
        want = dense_attention(Q, K, V, bias)[:, :, :H, :W]
        np.testing.assert_allclose(orc.forward_padded(q, kk, v, rpb, k, 1), want, rtol=0, atol=TOL)
    # q = 0, no bias: the plain mean over the searched (padded) window
    H, W, k, d = 4, 7, 3, 2
    q, kk, v, _ = _rand(rng, 1, 1, H, W, 3, k, with_rpb=False)
    got = orc.forward_padded(np.zeros_like(q), kk, v, None, k, d)
    Hp, Wp = max(H, k * d), max(W, k * d)
    for i in range(H):
        ky, _ = axis_window_search(Hp, k, d, i)
        for j in range(W):
            kx, _ = axis_window_search(Wp, k, d, j)
            tot = sum(v[0, 0, y, x] for y in ky for x in kx if y < H and x < W)
            np.testing.assert_allclose(got[0, 0, i, j], tot / (k * k), rtol=0, atol=TOL)


def pin_padding_backward(orc):
    """Gradients of the padded forward equal central differences."""
    rng = np.random.default_rng(34)
    H, W, k, d = 3, 5, 3, 2
    q, kk, v, rpb = _rand(rng, 1, 1, H, W, 2, k)
    dout = rng.standard_normal(q.shape)
    got = orc.backward_padded(q, kk, v, rpb, dout, k, d)
    eps = 1e-5

    def loss():
        return float((orc.forward_padded(q, kk, v, rpb, k, d) * dout).sum())

    for name, x, grad in (("q", q, got[0]), ("k", kk, got[1]), ("v", v, got[2]), ("rpb", rpb, got[3])):
        flat, num = x.reshape(-1), np.empty(x.size)
        for e in range(flat.size):
            old = flat[e]
            flat[e] = old + eps
            up = loss()
            flat[e] = old - eps
            dn = loss()
            flat[e] = old
            num[e] = (up - dn) / (2 * eps)
        np.testing.assert_allclose(grad.reshape(-1), num, rtol=1e-6, atol=1e-7, err_msg=f"d{name}")


ALL_PINS = [pin_window_keyset, pin_full_attention, pin_brute_force, pin_dilation_decomposition,
            pin_invariants, pin_rpb_orientation, pin_translation, pin_split_stages, pin_stage_table,
            pin_forward_query, pin_backward_finite_differences, pin_backward_dense_autograd,
            pin_backward_identities, pin_backward_dilation_decomposition, pin_philox_kat, pin_dropout,
            pin_dropout_backward, pin_padding, pin_padding_backward]
