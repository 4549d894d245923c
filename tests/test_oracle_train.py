"""Pins for the training-path oracle (``oracle/train.py``), no GPU.

The oracle states the straight-through backward of the MGLU forward of
"Masked Gated Linear Unit". Its masks are held as logits while training
("Limitations"), and the method builds on the straight-through estimator. The
tests tie the oracle to things other than itself:

* central finite differences of the float64 C forward oracle (dx, dW) and of
  the pure-Python brute force with real-valued mask entries (mask gradients);
* torch autograd on the textbook SwiGLU / GEGLU / ReGLU that MGLU reduces to;
* closed forms of a hand-worked case;
* the degree-2 homogeneity of the ReLU form.

Each mistake planted in a copy of the backward must fail one of these pins.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute, train

ACTS = [train.ACT_SWISH, train.ACT_GELU, train.ACT_RELU]


# ---------------------------------------------------------------- helpers
def _case(seed, T, d, h, n_m, p=0.5):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    Ws = rng.standard_normal((h, d)) * 0.5
    masks = (rng.random((n_m, h, d)) < p).astype(np.uint8)
    dout = rng.standard_normal((T, h))
    return x, Ws, masks, dout


def _c_forward(x, Ws, masks, a):
    out, _ = oracle.forward(x, Ws, oracle.pack_masks(masks), masks.shape[0], a)
    return out


def _soft_forward(x, Ws, mf, a):
    """Brute force on logical tensors with real-valued mask entries."""
    W_log = np.asarray(Ws).T.tolist()
    M_log = np.asarray(mf).transpose(0, 2, 1).tolist()
    return np.array(brute.mglu_logical_soft(np.asarray(x).tolist(), W_log, M_log, a))


def _fd(f, theta, step=1e-6):
    """Central differences of the scalar f at every entry of theta (a copy is perturbed)."""
    g = np.zeros_like(theta, dtype=np.float64)
    t = theta.astype(np.float64).copy()
    for idx in np.ndindex(t.shape):
        old = t[idx]
        t[idx] = old + step
        fp = f(t)
        t[idx] = old - step
        fm = f(t)
        t[idx] = old
        g[idx] = (fp - fm) / (2 * step)
    return g


def _close(got, exp, rel=1e-7):
    scale = max(1.0, float(np.max(np.abs(exp))))
    return float(np.max(np.abs(np.asarray(got) - np.asarray(exp)))) <= rel * scale


# ---------------------------------------------------------------- pins, usable on any backward
def _pin_fd(bw, seed=11, T=3, d=8, h=5):
    fails = []
    for n_m in (1, 2, 4, 8):
        for a in ACTS:
            x, Ws, masks, dout = _case(seed + 17 * n_m + a, T, d, h, n_m)
            # every mask selects a weight in every column, so no gate is exactly
            # 0, where ReLU has its kink and a difference quotient is one-sided
            for i in range(n_m):
                for j in range(h):
                    masks[i, j, (i + j) % d] = 1
            dx, dWs, dM = bw(x, Ws, masks, a, dout)
            gx = _fd(lambda t: float(np.sum(dout * _c_forward(t, Ws, masks, a))), x)
            gW = _fd(lambda t: float(np.sum(dout * _c_forward(x, t, masks, a))), Ws)
            gM = _fd(lambda t: float(np.sum(dout * _soft_forward(x, Ws, t, a))),
                     masks.astype(np.float64))
            for name, got, exp in (("dx", dx, gx), ("dW", dWs, gW), ("dM", dM, gM)):
                if not _close(got, exp):
                    fails.append(f"fd {name} n_m={n_m} act={a}")
    return fails


def _pin_glu_autograd(bw, seed=5, T=4, dp=6, h=3):
    """n_m = 1, x = [x', x'], W = [W_g; W_v] stacked along k, mask 1 on the
    first d' rows: MGLU is act(x' W_g) * (x' W_v); its gradients come from torch
    autograd of that textbook form."""
    fails = []
    rng = np.random.default_rng(seed)
    xp = rng.standard_normal((T, dp))
    Wg = rng.standard_normal((dp, h))
    Wv = rng.standard_normal((dp, h))
    dout = rng.standard_normal((T, h))
    x = np.concatenate([xp, xp], axis=1)
    Ws = np.concatenate([Wg, Wv], axis=0).T.copy()
    masks = np.zeros((1, h, 2 * dp), dtype=np.uint8)
    masks[0, :, :dp] = 1
    fns = {train.ACT_SWISH: torch.nn.functional.silu,
           train.ACT_GELU: lambda z: torch.nn.functional.gelu(z, approximate="none"),
           train.ACT_RELU: torch.nn.functional.relu}
    for a, fn in fns.items():
        txp = torch.tensor(xp, requires_grad=True)
        tWg = torch.tensor(Wg, requires_grad=True)
        tWv = torch.tensor(Wv, requires_grad=True)
        out = fn(txp @ tWg) * (txp @ tWv)
        out.backward(torch.tensor(dout))
        dx, dWs, _ = bw(x, Ws, masks, a, dout)
        if not _close(dx[:, :dp] + dx[:, dp:], txp.grad.numpy(), 1e-12):
            fails.append(f"glu dx act={a}")
        if not _close(dWs[:, :dp].T, tWg.grad.numpy(), 1e-12):
            fails.append(f"glu dW_gate act={a}")
        if not _close(dWs[:, dp:].T, tWv.grad.numpy(), 1e-12):
            fails.append(f"glu dW_value act={a}")
    return fails


def _pin_hand_case(bw):
    """d=2, h=1, x=[1,2], W=[[3],[4]], one mask selecting k=0: g = 3, v = 8.
    With dL/dout = 1: dx = [3 act'(3) 8, 4 act(3)], dW = [act'(3) 8, 2 act(3)],
    dM = [3 (8 act'(3) - act(3)), 8 (8 act'(3) - act(3))]."""
    fails = []
    sig = 1.0 / (1.0 + math.exp(-3.0))
    Phi = 0.5 * (1.0 + math.erf(3.0 / math.sqrt(2.0)))
    phi = math.exp(-4.5) / math.sqrt(2.0 * math.pi)
    forms = {train.ACT_SWISH: (3.0 * sig, sig + 3.0 * sig * (1.0 - sig)),
             train.ACT_GELU: (3.0 * Phi, Phi + 3.0 * phi),
             train.ACT_RELU: (3.0, 1.0)}
    x = np.array([[1.0, 2.0]])
    Ws = np.array([[3.0, 4.0]])
    masks = np.array([[[1, 0]]], dtype=np.uint8)
    for a, (f, fp) in forms.items():
        dx, dWs, dM = bw(x, Ws, masks, a, np.ones((1, 1)))
        if not _close(dx, [[3.0 * fp * 8.0, 4.0 * f]], 1e-14):
            fails.append(f"hand dx act={a}")
        if not _close(dWs, [[fp * 8.0, 2.0 * f]], 1e-14):
            fails.append(f"hand dW act={a}")
        if not _close(dM, [[[3.0 * (8.0 * fp - f), 8.0 * (8.0 * fp - f)]]], 1e-14):
            fails.append(f"hand dM act={a}")
    return fails


def _pin_relu_homogeneity(bw, seed=3):
    """ReLU MGLU is homogeneous of degree 2 in x and in W, so
    sum(x . dx) = sum(W . dW) = 2 sum(dout . out)."""
    fails = []
    x, Ws, masks, dout = _case(seed, 6, 40, 24, 4)
    dx, dWs, _ = bw(x, Ws, masks, train.ACT_RELU, dout)
    two_l = 2.0 * float(np.sum(dout * _c_forward(x, Ws, masks, train.ACT_RELU)))
    if abs(float(np.sum(x * dx)) - two_l) > 1e-10 * max(1.0, abs(two_l)):
        fails.append("relu homogeneity x")
    if abs(float(np.sum(Ws * dWs)) - two_l) > 1e-10 * max(1.0, abs(two_l)):
        fails.append("relu homogeneity W")
    return fails


def _pin_suite(bw):
    return _pin_hand_case(bw) + _pin_glu_autograd(bw) + _pin_relu_homogeneity(bw) + _pin_fd(bw)


# ---------------------------------------------------------------- the oracle passes every pin
def test_hand_case():
    assert _pin_hand_case(train.backward) == []


def test_reduces_to_glu_autograd():
    assert _pin_glu_autograd(train.backward) == []


def test_relu_homogeneity():
    assert _pin_relu_homogeneity(train.backward) == []


def test_finite_differences():
    assert _pin_fd(train.backward) == []


# ---------------------------------------------------------------- planted mistakes
def _mutant(kind):
    """A copy of the chain rule with one planted mistake."""
    def bw(x, Ws, masks, a, dout):
        m = masks.astype(np.float64)
        g, v = train.gates_values(x, Ws, m)
        dx, dWs, dM = np.zeros_like(x), np.zeros_like(Ws), np.zeros_like(m)
        for i in range(m.shape[0]):
            ag = train.act_grad(a, g[i])
            if kind == "swish_grad_sigma_only" and a == train.ACT_SWISH:
                ag = 1.0 / (1.0 + np.exp(-g[i]))
            dg = dout * ag * v[i]
            dv = dout * train.act(a, g[i])
            if kind == "swap_gate_value_grads":
                dg, dv = dv, dg
            gate_w, value_w = m[i] * Ws, (1.0 - m[i]) * Ws
            dx += dg @ gate_w + (0.0 if kind == "drop_value_path_dx" else dv @ value_w)
            if kind == "unmasked_dW":
                dWs += dg.T @ x + dv.T @ x
            else:
                dWs += m[i] * (dg.T @ x) + (1.0 - m[i]) * (dv.T @ x)
            dM[i] = Ws * (((dv - dg) if kind == "mask_grad_sign" else (dg - dv)).T @ x)
            if kind == "mask_grad_gate_only":
                dM[i] = Ws * (dg.T @ x)
        return dx, dWs, dM
    return bw


MUTANTS = ["swish_grad_sigma_only", "swap_gate_value_grads", "drop_value_path_dx", "unmasked_dW",
           "mask_grad_sign", "mask_grad_gate_only"]


def test_unplanted_copy_passes():
    assert _pin_suite(_mutant("none")) == []


@pytest.mark.parametrize("kind", MUTANTS)
def test_each_planted_mistake_fails_a_pin(kind):
    assert _pin_suite(_mutant(kind)), f"mutant {kind} passed every pin"


# ---------------------------------------------------------------- activation and its derivative
def test_act_matches_forward_oracles():
    zs = np.array([-40.0, -7.5, -1.0, -1e-3, 0.0, 1e-3, 0.5, 3.0, 12.0, 40.0])
    for a in ACTS:
        got = train.act(a, zs)
        for z, gv in zip(zs, got):
            assert abs(gv - oracle.activation(a, float(z))) <= 1e-15 * max(1.0, abs(gv))
            assert abs(gv - brute.act_ref(a, float(z))) <= 1e-15 * max(1.0, abs(gv))


def test_act_grad_against_differences_and_values():
    zs = [-9.0, -2.5, -0.7, -0.01, 0.02, 0.9, 2.0, 6.0]
    for a in ACTS:
        for z in zs:
            fd = (brute.act_ref(a, z + 1e-6) - brute.act_ref(a, z - 1e-6)) / 2e-6
            assert abs(float(train.act_grad(a, np.array(z))) - fd) < 1e-8, (a, z)
    # values at zero: Swish and GELU have slope 1/2; ReLU takes the subgradient 0
    assert float(train.act_grad(train.ACT_SWISH, np.array(0.0))) == 0.5
    assert float(train.act_grad(train.ACT_GELU, np.array(0.0))) == 0.5
    assert float(train.act_grad(train.ACT_RELU, np.array(0.0))) == 0.0


def test_forward_matches_c_oracle():
    for n_m in (1, 2, 4, 8):
        for a in ACTS:
            x, Ws, masks, _ = _case(40 + n_m, 5, 24, 9, n_m)
            assert _close(train.forward(x, Ws, masks, a), _c_forward(x, Ws, masks, a), 1e-13)


# ---------------------------------------------------------------- binarisation of mask logits
def test_binarize_special_values():
    z = np.array([1e-4, 0.0, -0.0, -1e-4, np.nan, np.inf, -np.inf, 65504.0, 2.0 ** -24, -(2.0 ** -24)],
                 dtype=np.float16)
    np.testing.assert_array_equal(train.binarize(z), [1, 0, 0, 0, 0, 1, 0, 1, 1, 0])
    assert train.binarize(z).dtype == np.uint8


def test_binarize_then_pack_matches_brute_pack():
    rng = np.random.default_rng(9)
    for n_m, d, h in ((1, 8, 3), (2, 16, 5), (4, 8, 7), (8, 24, 2)):
        logits = rng.standard_normal((n_m, h, d)).astype(np.float16)
        masks = train.binarize(logits)
        M_log = masks.transpose(0, 2, 1).tolist()
        assert bytes(oracle.pack_masks(masks)) == brute.pack_logical(M_log)


def test_logit_scale_does_not_change_gradients():
    """Straight-through reading: only the sign of a logit enters, and its
    gradient is the mask gradient with no factor that depends on the logit."""
    rng = np.random.default_rng(2)
    x, Ws, _, dout = _case(8, 3, 16, 6, 2)
    logits = rng.standard_normal((2, 6, 16))
    r1 = train.backward(x, Ws, train.binarize(logits), train.ACT_SWISH, dout)
    r2 = train.backward(x, Ws, train.binarize(7.5 * logits), train.ACT_SWISH, dout)
    for u, w in zip(r1, r2):
        np.testing.assert_array_equal(u, w)


# ---------------------------------------------------------------- down-projection and the block
def test_down_backward_finite_differences():
    rng = np.random.default_rng(4)
    hid = rng.standard_normal((3, 7))
    Wd = rng.standard_normal((5, 7))
    dy = rng.standard_normal((3, 5))
    dhid, dWd = train.down_backward(hid, Wd, dy)
    assert _close(dhid, _fd(lambda t: float(np.sum(dy * oracle.down(t, Wd))), hid))
    assert _close(dWd, _fd(lambda t: float(np.sum(dy * oracle.down(hid, t))), Wd))


def test_block_backward_composes():
    """dL/dx of the FFN block y = down(MGLU(x)) by the chain of the two
    backward steps, against differences of the two forward oracles."""
    x, Ws, masks, _ = _case(21, 2, 8, 6, 4)
    rng = np.random.default_rng(21)
    Wd = rng.standard_normal((8, 6))
    dy = rng.standard_normal((2, 8))
    a = train.ACT_GELU
    hid = _c_forward(x, Ws, masks, a)
    dhid, _ = train.down_backward(hid, Wd, dy)
    dx, _, _ = train.backward(x, Ws, masks, a, dhid)
    g = _fd(lambda t: float(np.sum(dy * oracle.down(_c_forward(t, Ws, masks, a), Wd))), x)
    assert _close(dx, g)


def test_sampled_backward_matches_full():
    """The sampled form gives exactly the full backward's entries (same
    arithmetic on the restricted operands), including repeated indices."""
    for n_m, a in ((1, train.ACT_RELU), (4, train.ACT_SWISH), (8, train.ACT_GELU)):
        x, Ws, masks, dout = _case(30 + n_m, 9, 32, 20, n_m)
        dx, dWs, dM = train.backward(x, Ws, masks, a, dout)
        tokens, rows = [0, 4, 8, 4], [19, 0, 7]
        sx, sW, sM = train.backward_sampled(x, Ws, masks, a, dout, tokens, rows)
        np.testing.assert_allclose(sx, dx[tokens], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sW, dWs[rows], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sM, dM[:, rows], rtol=1e-12, atol=1e-12)
