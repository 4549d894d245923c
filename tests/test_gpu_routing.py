"""GPU parity of mask routing against oracle/routed.py, through the C ABI:
the router (scores, top-k, hard or softmax weights) and the forward with
per-token mask weights ("Masked Gated Linear Unit", "Measured effects": each
token routed to 1 or 2 of its 4 masks instead of summing all of them)."""
import numpy as np
import pytest
import torch

from oracle import routed, train
from masked_glu_b200 import inputs, mglu

from gpu_util import assert_close, device_case, to_device, to_f64

pytestmark = pytest.mark.gpu
ACT = {"swish": train.ACT_SWISH, "gelu": train.ACT_GELU, "relu": train.ACT_RELU}


def _router_case(T, d, n_m, seed, dtype="bf16"):
    rng = np.random.default_rng(seed)
    x = inputs.normal(rng, (T, d), 1.0, dtype)
    Wr = inputs.normal(rng, (n_m, d), 1.0 / np.sqrt(d), dtype)
    return x, Wr


@pytest.mark.parametrize("n_m", [2, 4, 8])
@pytest.mark.parametrize("mode", ["hard", "softmax"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_route_topk_matches_oracle(n_m, mode, dtype):
    T, d = 37, 200
    x, Wr = _router_case(T, d, n_m, seed=2200 + n_m, dtype=dtype)
    ref_scores = routed.router_scores(x.values, Wr.values)
    bound = 1e-5 * (np.abs(x.values) @ np.abs(Wr.values).T) + 1e-30
    for k in range(n_m + 1):
        w, s = mglu.route_topk(to_device(x), to_device(Wr), k, mode)
        s64 = s.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(s64 - ref_scores) <= bound), "router scores beyond fp32 accumulation error"
        # the selection is an integer decision: the oracle takes it on the GPU's fp32 scores
        want = routed.route_weights(s64, k, mode)
        got = w.cpu().numpy().astype(np.float64)
        np.testing.assert_array_equal(got > 0, want > 0)
        if mode == "hard":
            np.testing.assert_array_equal(got, want)
        else:
            np.testing.assert_allclose(got, want, rtol=2e-6, atol=0)


def test_route_ties_go_to_the_lower_index():
    """Masks 1 and 2 share a router row, so they tie on every token: with
    k = 1 the kept mask is the lower index of the best pair."""
    T, d, n_m = 8, 64, 4
    x, Wr = _router_case(T, d, n_m, seed=2300)
    Wr.values[2] = Wr.values[1]
    Wr.storage[2] = Wr.storage[1]
    w, s = mglu.route_topk(to_device(x), to_device(Wr), 2, "hard")
    s = s.cpu().numpy()
    assert np.array_equal(s[:, 1], s[:, 2])
    want = routed.route_weights(s.astype(np.float64), 2, "hard")
    np.testing.assert_array_equal(w.cpu().numpy(), want)


@pytest.mark.parametrize("n_m,T,d,h", [(4, 1, 512, 200), (8, 3, 256, 96), (8, 9, 256, 96), (4, 16, 384, 130),
                                       (4, 40, 256, 100), (8, 200, 384, 72), (2, 5, 96, 40),
                                       (8, 390, 256, 86), (8, 70, 256, 60)])
def test_weighted_forward_matches_oracle(n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=2400 + n_m + T + d)
    x, W, packed, _ = device_case(case)
    rng = np.random.default_rng(2401 + T)
    wts = rng.random((T, n_m)).astype(np.float32)
    wts[rng.random((T, n_m)) < 0.4] = 0.0
    wts[:, 0] = 0.0  # one mask no token uses: the decode kernel skips its products
    out = mglu.forward_weighted(x, W, packed, n_m, torch.from_numpy(wts).cuda(), "gelu")
    assert mglu.last_device_status() == 0
    ref = routed.forward_weighted(case.x.values, case.W.values, case.masks, train.ACT_GELU,
                                  wts.astype(np.float64))
    assert_close(to_f64(out), ref, "bf16", f"weighted n_m={n_m} T={T}")


@pytest.mark.parametrize("T", [2, 40])
def test_unit_weights_give_the_plain_forward_bit_for_bit(T):
    case = inputs.make_case(T, 256, 96, 8, seed=2500 + T)
    x, W, packed, _ = device_case(case)
    ones = torch.ones((T, 8), dtype=torch.float32, device="cuda")
    assert torch.equal(mglu.forward_weighted(x, W, packed, 8, ones), mglu.forward(x, W, packed, 8))


@pytest.mark.parametrize("T,k,mode", [(1, 2, "hard"), (1, 1, "softmax"), (7, 2, "softmax"), (64, 2, "hard")])
def test_routed_forward_end_to_end(T, k, mode):
    """Router then weighted forward, against the oracle's routed forward with
    the GPU's selection."""
    n_m, d, h = 4, 512, 160
    case = inputs.make_case(T, d, h, n_m, seed=2600 + T)
    _, Wr = _router_case(T, d, n_m, seed=2601 + T)
    x, W, packed, _ = device_case(case)
    w, s = mglu.route_topk(x, to_device(Wr), k, mode)
    out = mglu.forward_weighted(x, W, packed, n_m, w)
    want_w = routed.route_weights(s.cpu().numpy().astype(np.float64), k, mode)
    ref = routed.forward_weighted(case.x.values, case.W.values, case.masks, train.ACT_SWISH, want_w)
    assert_close(to_f64(out), ref, "bf16", f"routed T={T} k={k} {mode}")


@pytest.mark.parametrize("n_m,T,d,h,k,mode", [(4, 1, 512, 160, 2, "hard"), (8, 2, 4096, 300, 2, "hard"),
                                              (8, 5, 1024, 200, 1, "softmax"), (2, 16, 256, 96, 1, "hard"),
                                              (1, 9, 200, 64, 1, "softmax"), (4, 40, 512, 160, 2, "softmax"),
                                              (8, 1, 4096, 14336, 2, "hard")])
def test_forward_routed_equals_router_then_weighted_forward(n_m, T, d, h, k, mode):
    """The routed forward in one call (on the decode kernel: the router inside
    the forward kernel, every CTA routing the tokens itself) gives the same
    weights, scores and output, bit for bit, as mglu_route_topk followed by
    mglu_forward_weighted; and the output matches the oracle's routed forward
    with those weights."""
    case = inputs.make_case(T, d, h, n_m, seed=2800 + n_m + T)
    _, Wr = _router_case(T, d, n_m, seed=2801 + T)
    x, W, packed, _ = device_case(case)
    Wr_d = to_device(Wr)
    w_ref, s_ref = mglu.route_topk(x, Wr_d, k, mode)
    out_ref = mglu.forward_weighted(x, W, packed, n_m, w_ref)
    out, w, s = mglu.forward_routed(x, W, packed, n_m, Wr_d, k, mode)
    torch.cuda.synchronize()
    assert mglu.last_device_status() == 0
    assert torch.equal(w, w_ref), "weights differ from mglu_route_topk"
    assert torch.equal(s, s_ref), "scores differ from mglu_route_topk"
    assert torch.equal(out, out_ref), "output differs from the two-call routed forward"
    if h * d <= 1 << 22:
        ref = routed.forward_weighted(case.x.values, case.W.values, case.masks, train.ACT_SWISH,
                                      w.cpu().numpy().astype(np.float64))
        assert_close(to_f64(out), ref, "bf16", f"forward_routed n_m={n_m} T={T}")


@pytest.mark.parametrize("T,k,dtype", [(3, 0, "bf16"), (4, 4, "bf16"), (40, 2, "bf16"), (5, 2, "f32")])
def test_forward_routed_edges(T, k, dtype):
    """k = 0 (no mask kept: every output 0), k = n_m (every mask kept), the
    tensor-core path (T = 40) and the fp32 path: the one call equals the
    router followed by the weighted forward."""
    n_m, d, h = 4, 256, 96
    case = inputs.make_case(T, d, h, n_m, seed=2900 + T + k, dtype=dtype)
    _, Wr = _router_case(T, d, n_m, seed=2901 + T, dtype=dtype)
    x, W, packed, _ = device_case(case)
    Wr_d = to_device(Wr)
    w_ref, s_ref = mglu.route_topk(x, Wr_d, k, "softmax")
    out_ref = mglu.forward_weighted(x, W, packed, n_m, w_ref)
    out, w, s = mglu.forward_routed(x, W, packed, n_m, Wr_d, k, "softmax")
    torch.cuda.synchronize()
    assert mglu.last_device_status() == 0
    assert torch.equal(w, w_ref) and torch.equal(s, s_ref)
    assert torch.equal(out, out_ref)
    if k == 0:
        assert not torch.any(out.float() != 0)
