"""Pure-Python brute force for tiny maps -- a second, deliberately different
formulation of neighborhood attention, used to pin the oracle.

The window is found by SEARCH rather than by the clamp formula: along each axis
the query's dilation group is listed explicitly, every run of k consecutive
group members is a candidate, and the run whose start is nearest to the
centred start (i' - k//2) is taken -- "localizes the receptive field to its
nearest neighborhood", with the window kept inside the image at the edges
("Neighborhood Attention Transformer", README figure caption).  Dilation is
"every d-th pixel" ("Dilated Neighborhood Attention Transformer", overview).
Scores, softmax and the weighted sum are written as explicit Python loops.
"""
from __future__ import annotations

import math


def axis_window_search(L: int, k: int, d: int, i: int) -> tuple[list[int], list[int]]:
    group = [p for p in range(L) if p % d == i % d]          # the query's dilation group
    pos = group.index(i)                                      # i' : position inside the group
    starts = range(0, len(group) - k + 1)                     # every window that fits
    best = min(starts, key=lambda s: abs(s - (pos - k // 2)))
    keys = group[best:best + k]
    rel = [group.index(key) - pos + (k - 1) for key in keys]  # relative position -> bias index
    return keys, rel


def forward_brute(q, kk, v, rpb, k: int, d: int):
    """q, kk, v: nested lists [B][heads][H][W][D]; rpb: [heads][2k-1][2k-1] or None."""
    B, heads, H, W, D = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0]), len(q[0][0][0][0])
    out = [[[[[0.0] * D for _ in range(W)] for _ in range(H)] for _ in range(heads)] for _ in range(B)]
    for b in range(B):
        for h in range(heads):
            for i in range(H):
                ky, ry = axis_window_search(H, k, d, i)
                for j in range(W):
                    kx, rx = axis_window_search(W, k, d, j)
                    scores, vals = [], []
                    for a, y in enumerate(ky):
                        for c, x in enumerate(kx):
                            s = sum(q[b][h][i][j][e] * kk[b][h][y][x][e] for e in range(D)) / math.sqrt(D)
                            if rpb is not None:
                                s += rpb[h][ry[a]][rx[c]]
                            scores.append(s)
                            vals.append(v[b][h][y][x])
                    m = max(scores)
                    w = [math.exp(s - m) for s in scores]
                    z = sum(w)
                    for e in range(D):
                        out[b][h][i][j][e] = sum(w[n] * vals[n][e] for n in range(len(w))) / z
    return out
