"""Pins of the oracle's dense-gate variant (no GPU).

"Masked Gated Linear Unit", "Measured effects", last row: "Remove the gate
mask (dense gate)".  Reading: every gate is the whole product x W, each value
keeps its mask, out = sum_i act(x W) * x ((1 - M_i) . W).  The pins tie the
C oracle's variant to hand-worked closed forms, to the naive shared-weight
GLU act(x W) * (x W) that it reduces to with one empty mask ("Surprising
findings": one weight matrix shared by the gate and value streams), to the
pure-Python brute force and to exact zeros; planted mistakes must fail."""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute

from test_oracle import ACTS, logical_to_storage, parse_golden, random_logical

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dense_gate_cases.txt")


def dense_c(x, W_log, M_log, act):
    Ws, masks = logical_to_storage(W_log, M_log)
    out, resid = oracle.forward(np.asarray(x, dtype=np.float64), Ws, oracle.pack_masks(masks), masks.shape[0],
                                act | oracle.GATE_DENSE)
    assert resid <= 1e-12
    return out


@pytest.mark.parametrize("case", parse_golden(GOLDEN), ids=lambda c: c["name"])
@pytest.mark.parametrize("act", list(ACTS))
def test_hand_cases(case, act):
    want = np.array(case["exp"][act])
    np.testing.assert_allclose(dense_c(case["x"], case["W"], case["M"], ACTS[act]), want, rtol=1e-12, atol=1e-13)
    got = brute.mglu_logical(case["x"], case["W"], case["M"], ACTS[act], dense_gate=True)
    np.testing.assert_allclose(np.array(got), want, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("act", [0, 1, 2])
def test_one_empty_mask_is_the_naive_shared_weight_glu(act):
    rng = np.random.default_rng(40 + act)
    x, W, _ = random_logical(rng, 3, 12, 7, 1)
    M = np.zeros((1, 12, 7), dtype=np.uint8)
    z = torch.from_numpy(x @ W)
    f = {0: torch.nn.functional.silu, 1: torch.nn.functional.gelu, 2: torch.relu}[act]
    np.testing.assert_allclose(dense_c(x, W, M, act), (f(z) * z).numpy(), rtol=1e-12, atol=1e-13)


def test_full_masks_give_exact_zero():
    rng = np.random.default_rng(41)
    x, W, _ = random_logical(rng, 2, 9, 5, 3)
    M = np.ones((3, 9, 5), dtype=np.uint8)
    assert np.all(dense_c(x, W, M, 0) == 0.0)


@pytest.mark.parametrize("n_m", [1, 2, 4, 8])
@pytest.mark.parametrize("act", [0, 1, 2])
def test_brute_force_agrees(n_m, act):
    rng = np.random.default_rng(50 + n_m * 10 + act)
    for T, d, h in [(1, 3, 2), (3, 16, 16)]:
        x, W, M = random_logical(rng, T, d, h, n_m)
        ref = np.array(brute.mglu_logical(x.tolist(), W.tolist(), M.tolist(), act, dense_gate=True))
        out = dense_c(x, W, M, act)
        assert np.abs(out - ref).max() <= 1e-12 * max(1.0, float(np.abs(ref).max()))


def test_plain_forward_is_unchanged_by_the_flag_bit_being_clear():
    rng = np.random.default_rng(42)
    x, W, M = random_logical(rng, 2, 8, 6, 4)
    Ws, masks = logical_to_storage(W, M)
    plain, _ = oracle.forward(x, Ws, oracle.pack_masks(masks), 4, 0)
    np.testing.assert_allclose(plain, np.array(brute.mglu_logical(x.tolist(), W.tolist(), M.tolist(), 0)),
                               rtol=1e-12, atol=1e-13)
    assert not np.allclose(plain, dense_c(x, W, M, 0))


def _pins(fwd):
    """The pins above as one function of fwd(x, W_log, M_log, act)."""
    failed = []
    for case in parse_golden(GOLDEN):
        for a, act in ACTS.items():
            if not np.allclose(np.array(fwd(case["x"], case["W"], case["M"], act)), np.array(case["exp"][a]),
                               rtol=1e-9, atol=1e-12):
                failed.append(f"{case['name']}/{a}")
    rng = np.random.default_rng(43)
    x, W, _ = random_logical(rng, 2, 6, 4, 1)
    z = x @ W
    if not np.allclose(np.array(fwd(x.tolist(), W.tolist(), np.zeros((1, 6, 4), np.uint8).tolist(), 2)),
                       np.maximum(z, 0) * z, rtol=1e-9):
        failed.append("naive_glu")
    if np.any(np.array(fwd(x.tolist(), W.tolist(), np.ones((1, 6, 4), np.uint8).tolist(), 0)) != 0):
        failed.append("full_masks")
    return failed


def _mutant(kind):
    def fwd(x, W, M, act):
        T, d, h, n_m = len(x), len(W), len(W[0]), len(M)
        out = np.zeros((T, h))
        for b in range(T):
            for j in range(h):
                for i in range(n_m):
                    D = sum(x[b][k] * W[k][j] for k in range(d))
                    g = sum(x[b][k] * W[k][j] for k in range(d) if M[i][k][j])
                    v = sum(x[b][k] * W[k][j] for k in range(d) if not M[i][k][j])
                    if kind == "gate_keeps_mask":
                        out[b, j] += brute.act_ref(act, g) * v
                    elif kind == "value_dense_too":
                        out[b, j] += brute.act_ref(act, D) * D
                    elif kind == "value_is_gate_side":
                        out[b, j] += brute.act_ref(act, D) * g
        return out
    return fwd


def test_pins_pass_on_the_brute_force():
    assert _pins(lambda x, W, M, act: brute.mglu_logical(x, W, M, act, dense_gate=True)) == []


@pytest.mark.parametrize("kind", ["gate_keeps_mask", "value_dense_too", "value_is_gate_side"])
def test_each_planted_mistake_fails_a_pin(kind):
    assert _pins(_mutant(kind)), f"mutant {kind} passed every pin"
