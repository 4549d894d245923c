"""Float64 CPU oracle of the MGLU training path -- test infrastructure.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU legs
may import this module; the product library never loads it, and this module
never loads the product library.

What "Masked Gated Linear Unit" fixes: the masks are learned, and are held
as FP16 logits while training ("Limitations"). The method builds on the
straight-through estimator (the page's list of prior work). It states no
formula for either. The plainest readings, taken here:

* forward masks are the binarised logits: M_i[j, k] = 1 where
  logit_i[j, k] > 0, else 0 (a logit of exactly zero, of either sign, or a NaN
  gives 0);
* the straight-through estimator passes the loss gradient with respect to
  the binary mask entry M_i[j, k] unchanged to its logit (no clipping, no
  sigmoid factor);
* the gradients of x and W are the exact derivatives of the forward with the
  binary masks held fixed.

Each step follows the chain rule through the forward's definition
(out = sum_i act(g_i) * v_i, g_i = x (M_i . W), v_i = x ((1 - M_i) . W)), with
numpy float64 matmul as the only library step.

Conventions as in :mod:`oracle.core`:
  x      [T][d]        activations
  Ws     [h][d]        W stored transposed, Ws[j, k] = W[k, j]
  masks  [n_m][h][d]   {0, 1}, masks[i, j, k] = M_i[k, j]
  logits [n_m][h][d]   mask logits, same layout as masks
  dout   [T][h]        gradient of the loss with respect to out
  Wd     [d][h]        down-projection, y = hid @ Wd^T
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import expit, ndtr

ACT_SWISH = 0
ACT_GELU = 1
ACT_RELU = 2
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def binarize(logits) -> np.ndarray:
    """Forward masks from logits: 1 where logit > 0, else 0 (uint8)."""
    z = np.asarray(logits)
    return (z > 0).astype(np.uint8)


def act(a: int, z: np.ndarray) -> np.ndarray:
    """act(z) elementwise: Swish z*sigma(z), exact GELU z*Phi(z), ReLU."""
    z = np.asarray(z, dtype=np.float64)
    if a == ACT_SWISH:
        return z * expit(z)
    if a == ACT_GELU:
        return z * ndtr(z)
    if a == ACT_RELU:
        return np.where(z > 0, z, 0.0)
    raise ValueError(a)


def act_grad(a: int, z: np.ndarray) -> np.ndarray:
    """d act / dz elementwise.

    Swish: sigma(z) + z sigma(z) (1 - sigma(z)); GELU: Phi(z) + z phi(z);
    ReLU: 1 for z > 0, else 0 (the subgradient 0 is taken at z = 0)."""
    z = np.asarray(z, dtype=np.float64)
    if a == ACT_SWISH:
        s = expit(z)
        return s + z * s * (1.0 - s)
    if a == ACT_GELU:
        return ndtr(z) + z * np.exp(-0.5 * z * z) * _INV_SQRT_2PI
    if a == ACT_RELU:
        return np.where(z > 0, 1.0, 0.0)
    raise ValueError(a)


def gates_values(x, Ws, masks):
    """g_i = x (M_i . W) and, separately, v_i = x ((1 - M_i) . W): [n_m][T][h] each."""
    x = np.asarray(x, dtype=np.float64)
    Ws = np.asarray(Ws, dtype=np.float64)
    m = np.asarray(masks, dtype=np.float64)
    g = np.stack([x @ (m[i] * Ws).T for i in range(m.shape[0])])
    v = np.stack([x @ ((1.0 - m[i]) * Ws).T for i in range(m.shape[0])])
    return g, v


def forward(x, Ws, masks, a: int) -> np.ndarray:
    """out [T][h] = sum_i act(g_i) * v_i (the same definition as the C oracle)."""
    g, v = gates_values(x, Ws, masks)
    return sum(act(a, g[i]) * v[i] for i in range(g.shape[0]))


def backward(x, Ws, masks, a: int, dout):
    """Gradients of L through out = MGLU(x; W, M) for a given dL/dout.

    Returns (dx [T][d], dWs [h][d], dlogits [n_m][h][d]). dlogits is the
    straight-through gradient: dL/dM_i evaluated at the binary masks.

    For each mask i, per token b and column j:
      dL/dg_i = dout * act'(g_i) * v_i      (gate side, weights with M = 1)
      dL/dv_i = dout * act(g_i)             (value side, weights with M = 0)
    and since g_i and v_i are linear in x, W and M:
      dx   = sum_i dL/dg_i @ (M_i . W) + dL/dv_i @ ((1 - M_i) . W)
      dW   = sum_i M_i . (dL/dg_i^T @ x) + (1 - M_i) . (dL/dv_i^T @ x)
      dM_i = W . ((dL/dg_i - dL/dv_i)^T @ x)
    (dg_i/dM_i[j,k] = x_k W[j,k], dv_i/dM_i[j,k] = -x_k W[j,k]).
    """
    x = np.asarray(x, dtype=np.float64)
    Ws = np.asarray(Ws, dtype=np.float64)
    m = np.asarray(masks, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    g, v = gates_values(x, Ws, m)
    dx = np.zeros_like(x)
    dWs = np.zeros_like(Ws)
    dM = np.zeros_like(m)
    for i in range(m.shape[0]):
        dg = dout * act_grad(a, g[i]) * v[i]
        dv = dout * act(a, g[i])
        gate_w = m[i] * Ws
        value_w = (1.0 - m[i]) * Ws
        dx += dg @ gate_w + dv @ value_w
        dWs += m[i] * (dg.T @ x) + (1.0 - m[i]) * (dv.T @ x)
        dM[i] = Ws * ((dg - dv).T @ x)
    return dx, dWs, dM


def down_backward(hid, Wd, dy):
    """y = hid @ Wd^T: returns (dhid [T][h], dWd [d][h]) for a given dL/dy [T][d]."""
    hid = np.asarray(hid, dtype=np.float64)
    Wd = np.asarray(Wd, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    return dy @ Wd, dy.T @ hid


def backward_sampled(x, Ws, masks, a: int, dout, tokens, rows):
    """The same gradients for a subset, at sizes where the full backward is
    too slow: dx for the listed tokens (every column j enters), and dW and
    the mask-logit gradients for the listed rows j of W (every token enters).

    Returns (dx [len(tokens)][d], dWs [len(rows)][d], dM [n_m][len(rows)][d]).
    Each piece is the chain rule of ``backward`` restricted to what it needs:
    g_i and v_i of the listed tokens for dx, of the listed rows for dW, dM.
    """
    x = np.asarray(x, dtype=np.float64)
    Ws = np.asarray(Ws, dtype=np.float64)
    m = np.asarray(masks, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    tokens = np.asarray(tokens, dtype=np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    n_m = m.shape[0]

    xt = x[tokens]
    g, v = gates_values(xt, Ws, m)
    dx = np.zeros((tokens.size, x.shape[1]))
    for i in range(n_m):
        dg = dout[tokens] * act_grad(a, g[i]) * v[i]
        dv = dout[tokens] * act(a, g[i])
        dx += dg @ (m[i] * Ws) + dv @ ((1.0 - m[i]) * Ws)

    Wr, mr = Ws[rows], m[:, rows]
    g, v = gates_values(x, Wr, mr)
    dWs = np.zeros((rows.size, x.shape[1]))
    dM = np.zeros((n_m, rows.size, x.shape[1]))
    for i in range(n_m):
        dg = dout[:, rows] * act_grad(a, g[i]) * v[i]
        dv = dout[:, rows] * act(a, g[i])
        dWs += mr[i] * (dg.T @ x) + (1.0 - mr[i]) * (dv.T @ x)
        dM[i] = Wr * ((dg - dv).T @ x)
    return dx, dWs, dM
