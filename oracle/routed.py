"""Float64 CPU oracle of mask routing: per-token mask weights and top-k
selection -- test infrastructure.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU legs
may import this module; the product library never loads it.

"Masked Gated Linear Unit", "Measured effects reported in the paper": two
ablations route each token to 1 or 2 of its 4 masks instead of summing all
of them. The method builds on mixture-of-experts routing (the page's list of
prior work names the Switch Transformer). The page defines no router. The
plainest readings, taken here:

* a router scores the masks per token with one linear map,
  r[b, i] = sum_k x[b, k] Wr[i, k] (no bias);
* top-k keeps the k masks with the highest scores; equal scores go to the
  lower mask index;
* a routed token sums only its kept masks' terms. Two weightings are offered:
  - "hard": each kept term with weight 1, the plain restriction of the sum;
  - "softmax": each kept term weighted by the softmax of all n_m scores, as
    the Switch Transformer scales an expert's output by its router
    probability.

Both are instances of one weighted forward,
out[b, j] = sum_i w[b, i] act(g_i[b, j]) v_i[b, j], with w = 1 giving the
unrouted method.

Conventions as in :mod:`oracle.core` (x [T][d], Ws [h][d], masks
[n_m][h][d]); Wr [n_m][d]; weights and scores [T][n_m].
"""
from __future__ import annotations

import numpy as np

from . import train


def router_scores(x, Wr) -> np.ndarray:
    """r [T][n_m] = x Wr^T in float64."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(Wr, dtype=np.float64).T


def topk_select(scores, k: int) -> np.ndarray:
    """[T][n_m] uint8: 1 for the k highest scores of each row. Of equal
    scores, the lower mask index wins."""
    s = np.asarray(scores, dtype=np.float64)
    T, n_m = s.shape
    if not 0 <= k <= n_m:
        raise ValueError("k out of range")
    sel = np.zeros((T, n_m), dtype=np.uint8)
    for b in range(T):
        # rank by (score descending, index ascending)
        order = sorted(range(n_m), key=lambda i: (-s[b, i], i))
        for i in order[:k]:
            sel[b, i] = 1
    return sel


def route_weights(scores, k: int, mode: str = "hard") -> np.ndarray:
    """Per-token mask weights [T][n_m] from router scores."""
    s = np.asarray(scores, dtype=np.float64)
    sel = topk_select(s, k).astype(np.float64)
    if mode == "hard":
        return sel
    if mode == "softmax":
        e = np.exp(s - s.max(axis=1, keepdims=True))
        return sel * (e / e.sum(axis=1, keepdims=True))
    raise ValueError(mode)


def forward_weighted(x, Ws, masks, a: int, weights) -> np.ndarray:
    """out [T][h] = sum_i w[b, i] act(g_i) v_i."""
    w = np.asarray(weights, dtype=np.float64)
    g, v = train.gates_values(x, Ws, masks)
    if w.shape != (g.shape[1], g.shape[0]):
        raise ValueError("weights must be [T][n_m]")
    return sum(w[:, i:i + 1] * train.act(a, g[i]) * v[i] for i in range(g.shape[0]))


def forward_routed(x, Ws, masks, a: int, Wr, k: int, mode: str = "hard"):
    """Route, then the weighted forward. Returns (out [T][h], weights [T][n_m])."""
    w = route_weights(router_scores(x, Wr), k, mode)
    return forward_weighted(x, Ws, masks, a, w), w
