"""Pins for the mask-routing oracle (``oracle/routed.py``), no GPU.

The routed forward of "Masked Gated Linear Unit" ("Measured effects": each
token routed to 1 or 2 of its 4 masks instead of summing all of them) is
tied to things other than itself:
* the unrouted C forward oracle (weights 1, or k = n_m);
* the pure-Python brute force run on each token's kept masks alone;
* torch.topk and torch.softmax for the selection and the weights;
* a hand-made tie;
* linearity in the weights.

Each mistake planted in a copy of the routed forward must fail one of these
pins.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import brute, routed, train

ACTS = [train.ACT_SWISH, train.ACT_GELU, train.ACT_RELU]


def _case(seed, T, d, h, n_m):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    Ws = rng.standard_normal((h, d)) * 0.5
    masks = (rng.random((n_m, h, d)) < 0.5).astype(np.uint8)
    Wr = rng.standard_normal((n_m, d))
    return x, Ws, masks, Wr


def _c_forward(x, Ws, masks, a):
    out, _ = oracle.forward(x, Ws, oracle.pack_masks(masks), masks.shape[0], a)
    return out


def _brute_subset(x, Ws, masks, a, sel):
    """Brute force per token on the masks the token keeps (logical tensors)."""
    W_log = np.asarray(Ws).T.tolist()
    rows = []
    for b in range(x.shape[0]):
        kept = [masks[i].T.tolist() for i in range(masks.shape[0]) if sel[b, i]]
        if kept:
            rows.append(brute.mglu_logical([x[b].tolist()], W_log, kept, a)[0])
        else:
            rows.append([0.0] * Ws.shape[0])
    return np.array(rows)


# ---------------------------------------------------------------- pins, usable on any routed forward
def _pins(fwd):
    fails = []
    for n_m in (1, 2, 4, 8):
        for a in ACTS:
            x, Ws, masks, Wr = _case(100 + 3 * n_m + a, 5, 16, 7, n_m)
            full = _c_forward(x, Ws, masks, a)
            out, _ = fwd(x, Ws, masks, a, Wr, n_m, "hard")
            if np.max(np.abs(out - full)) > 1e-12 * max(1.0, np.max(np.abs(full))):
                fails.append(f"k=n_m equals the sum n_m={n_m} act={a}")
            for k in range(0, n_m + 1):
                out, w = fwd(x, Ws, masks, a, Wr, k, "hard")
                sel = routed.topk_select(routed.router_scores(x, Wr), k)
                ref = _brute_subset(x, Ws, masks, a, sel)
                if np.max(np.abs(out - ref)) > 1e-12 * max(1.0, np.max(np.abs(ref))):
                    fails.append(f"hard top-{k} vs brute n_m={n_m} act={a}")
    # the softmax weighting scales each kept term by its router probability
    x, Ws, masks, Wr = _case(7, 4, 16, 6, 4)
    out, w = fwd(x, Ws, masks, train.ACT_SWISH, Wr, 2, "softmax")
    p = torch.softmax(torch.tensor(routed.router_scores(x, Wr)), dim=1).numpy()
    sel = routed.topk_select(routed.router_scores(x, Wr), 2)
    g, v = train.gates_values(x, Ws, masks)
    ref = sum((p[:, i] * sel[:, i])[:, None] * train.act(train.ACT_SWISH, g[i]) * v[i] for i in range(4))
    if np.max(np.abs(out - ref)) > 1e-12 * max(1.0, np.max(np.abs(ref))):
        fails.append("softmax weighting")
    return fails


def test_routed_forward_passes_pins():
    assert _pins(routed.forward_routed) == []


def _mutant(kind):
    def fwd(x, Ws, masks, a, Wr, k, mode="hard"):
        s = routed.router_scores(x, Wr)
        if kind == "lowest_scores":
            s = -s
        w = routed.route_weights(s, k, mode)
        if kind == "softmax_over_kept_only" and mode == "softmax":
            sel = routed.topk_select(s, k).astype(float)
            e = np.exp(s - s.max(axis=1, keepdims=True)) * sel
            w = e / np.maximum(e.sum(axis=1, keepdims=True), 1e-300)
        g, v = train.gates_values(x, Ws, masks)
        out = 0.0
        for i in range(g.shape[0]):
            if kind == "weight_inside_act":
                out = out + train.act(a, w[:, i:i + 1] * g[i]) * v[i]
            elif kind == "weight_on_value_only_of_first":
                out = out + (w[:, i:i + 1] if i else 1.0) * train.act(a, g[i]) * v[i]
            else:
                out = out + w[:, i:i + 1] * train.act(a, g[i]) * v[i]
        return out, w
    return fwd


def test_unplanted_copy_passes():
    assert _pins(_mutant("none")) == []


@pytest.mark.parametrize("kind", ["lowest_scores", "softmax_over_kept_only", "weight_inside_act",
                                  "weight_on_value_only_of_first"])
def test_each_planted_mistake_fails_a_pin(kind):
    assert _pins(_mutant(kind)), f"mutant {kind} passed every pin"


# ---------------------------------------------------------------- selection and weights
def test_topk_matches_torch_on_distinct_scores():
    rng = np.random.default_rng(12)
    s = rng.standard_normal((50, 8))
    for k in range(9):
        sel = routed.topk_select(s, k)
        ref = np.zeros_like(sel)
        if k:
            idx = torch.topk(torch.tensor(s), k, dim=1).indices.numpy()
            np.put_along_axis(ref, idx, 1, axis=1)
        np.testing.assert_array_equal(sel, ref)
        assert (sel.sum(axis=1) == k).all()


def test_topk_ties_go_to_the_lower_index():
    s = np.array([[1.0, 2.0, 2.0, 0.5], [3.0, 3.0, 3.0, 3.0], [-1.0, -1.0, 0.0, -1.0]])
    np.testing.assert_array_equal(routed.topk_select(s, 1), [[0, 1, 0, 0], [1, 0, 0, 0], [0, 0, 1, 0]])
    np.testing.assert_array_equal(routed.topk_select(s, 2), [[0, 1, 1, 0], [1, 1, 0, 0], [1, 0, 1, 0]])


def test_topk_rejects_bad_k():
    with pytest.raises(ValueError):
        routed.topk_select(np.zeros((2, 4)), 5)
    with pytest.raises(ValueError):
        routed.topk_select(np.zeros((2, 4)), -1)


def test_unit_weights_give_the_unrouted_forward():
    for a in ACTS:
        x, Ws, masks, _ = _case(3 + a, 6, 24, 10, 4)
        out = routed.forward_weighted(x, Ws, masks, a, np.ones((6, 4)))
        full = _c_forward(x, Ws, masks, a)
        assert np.max(np.abs(out - full)) <= 1e-13 * max(1.0, np.max(np.abs(full)))


def test_weighted_forward_is_linear_in_the_weights():
    x, Ws, masks, _ = _case(5, 4, 16, 8, 4)
    rng = np.random.default_rng(5)
    w1, w2 = rng.random((4, 4)), rng.random((4, 4))
    lhs = routed.forward_weighted(x, Ws, masks, train.ACT_GELU, w1 + 2.0 * w2)
    rhs = (routed.forward_weighted(x, Ws, masks, train.ACT_GELU, w1)
           + 2.0 * routed.forward_weighted(x, Ws, masks, train.ACT_GELU, w2))
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * max(1.0, np.max(np.abs(lhs)))
