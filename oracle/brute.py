"""Pure-Python brute force of the MGLU forward -- test infrastructure.

Written independently of ``mglu_oracle.c``: it works on the LOGICAL tensors
(x [T][d], W [d][h], M [n_m][d][h]) with plain nested loops and Python floats
(IEEE float64), so a transposition, indexing or bit-order slip in the C oracle
shows up as a disagreement.  Sizes are meant to stay tiny (d, h <= 16).

Reading of "Masked Gated Linear Unit" ("Approach"; "Measured effects" rows on
summing all masks and on GELU / ReLU): for each mask i the weights it selects
form the gate, the rest form the value, and the n_m gated products are summed.
"""
from __future__ import annotations

import math


def act_ref(act: int, z: float) -> float:
    if act == 0:  # Swish, beta = 1
        return z * (1.0 / (1.0 + math.exp(-z))) if z > -700 else 0.0 * z
    if act == 1:  # exact GELU: z * Phi(z)
        return z * 0.5 * (1.0 + math.erf(z / math.sqrt(2.0)))
    if act == 2:  # ReLU
        return z if z > 0 else 0.0
    raise ValueError(act)


def mglu_logical(x, W, M, act, dense_gate=False):
    """x: T lists of d floats; W: d lists of h floats; M: n_m x d x h of 0/1.

    dense_gate: the "Remove the gate mask (dense gate)" ablation ("Measured
    effects", last row), read as: every gate is the whole product x W and
    each value keeps its mask.  Returns T lists of h floats."""
    T, d, h, n_m = len(x), len(W), len(W[0]), len(M)
    out = []
    for b in range(T):
        row = []
        for j in range(h):
            total = 0.0
            for i in range(n_m):
                gate = 0.0
                value = 0.0
                for k in range(d):
                    if M[i][k][j] or dense_gate:
                        gate += x[b][k] * W[k][j]
                    if not M[i][k][j]:
                        value += x[b][k] * W[k][j]
                total += act_ref(act, gate) * value
            row.append(total)
        out.append(row)
    return out


def pack_logical(M):
    """Pack logical masks M[i][k][j] into the byte stream: weight (j, k) owns
    n_m bits starting at bit (j*d + k)*n_m, bit i = mask i, LSB first."""
    n_m, d, h = len(M), len(M[0]), len(M[0][0])
    nbits = h * d * n_m
    out = bytearray((nbits + 7) // 8)
    for j in range(h):
        for k in range(d):
            for i in range(n_m):
                if M[i][k][j]:
                    pos = (j * d + k) * n_m + i
                    out[pos // 8] |= 1 << (pos % 8)
    return bytes(out)


def matmul_logical(a, b):
    """Plain triple loop a [m][n] @ b [n][p]."""
    m, n, p = len(a), len(b), len(b[0])
    return [[sum(a[r][t] * b[t][c] for t in range(n)) for c in range(p)] for r in range(m)]


def mglu_logical_soft(x, W, M, act):
    """The same sum with the mask entries taken as real numbers: the gate of
    mask i sums x*W*M_i and its value sums x*W*(1 - M_i).  For 0/1 masks it is
    ``mglu_logical``; with real entries it is the function that the
    straight-through gradient of a mask entry differentiates."""
    T, d, h, n_m = len(x), len(W), len(W[0]), len(M)
    out = []
    for b in range(T):
        row = []
        for j in range(h):
            total = 0.0
            for i in range(n_m):
                gate = 0.0
                value = 0.0
                for k in range(d):
                    p = x[b][k] * W[k][j]
                    gate += p * M[i][k][j]
                    value += p * (1.0 - M[i][k][j])
                total += act_ref(act, gate) * value
            row.append(total)
        out.append(row)
    return out
