"""Pins for the CPU oracle (no GPU).

The oracle (``oracle/``) is the float64 statement of the MGLU forward read from
"Masked Gated Linear Unit" ("Approach"; "Measured effects" rows on summing all
masks and on GELU / ReLU gating).  These tests tie it to things other than
itself: hand-worked closed forms (tests/golden/hand_cases.txt), an independent
pure-Python brute force on logical tensors, the reduction to textbook SwiGLU,
exact special cases, symmetries of the definition, and mutants that each
break one of these pins.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from masked_glu_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.txt")
ACTS = {"swish": oracle.ACT_SWISH, "gelu": oracle.ACT_GELU, "relu": oracle.ACT_RELU}


# ---------------------------------------------------------------- helpers
def parse_golden(path=GOLDEN):
    cases, cur = [], None
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "case":
            cur = {"name": vals[0], "x": [], "W": [], "M": {}, "exp": {a: [] for a in ACTS}}
            cases.append(cur)
        elif key == "x":
            cur["x"].append([float(v) for v in vals])
        elif key == "W":
            cur["W"].append([float(v) for v in vals])
        elif key.startswith("M"):
            cur["M"].setdefault(int(key[1:]), []).append([int(v) for v in vals])
        elif key in ACTS:
            cur["exp"][key].append([float(v) for v in vals])
    for c in cases:
        c["M"] = [c["M"][i] for i in sorted(c["M"])]
    return cases


def logical_to_storage(W_log, M_log):
    """logical W [d][h], M [n_m][d][h] -> storage Ws [h][d], masks [n_m][h][d]."""
    W_log = np.asarray(W_log, dtype=np.float64)
    M_log = np.asarray(M_log, dtype=np.uint8)
    return np.ascontiguousarray(W_log.T), np.ascontiguousarray(M_log.transpose(0, 2, 1))


def c_oracle_logical(x, W_log, M_log, act):
    Ws, masks = logical_to_storage(W_log, M_log)
    out, resid = oracle.forward(np.asarray(x, dtype=np.float64), Ws, oracle.pack_masks(masks),
                                masks.shape[0], act)
    assert resid <= 1e-12
    return out


def random_logical(rng, T, d, h, n_m, p=0.5):
    x = rng.standard_normal((T, d))
    W = rng.standard_normal((d, h)) * 0.5
    M = (rng.random((n_m, d, h)) < p).astype(np.uint8)
    return x, W, M


# ---------------------------------------------------------------- hand cases
@pytest.mark.parametrize("case", parse_golden(), ids=lambda c: c["name"])
@pytest.mark.parametrize("act", list(ACTS))
def test_hand_cases_c_oracle(case, act):
    out = c_oracle_logical(case["x"], case["W"], case["M"], ACTS[act])
    np.testing.assert_allclose(out, np.array(case["exp"][act]), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("case", parse_golden(), ids=lambda c: c["name"])
@pytest.mark.parametrize("act", list(ACTS))
def test_hand_cases_brute(case, act):
    out = brute.mglu_logical(case["x"], case["W"], case["M"], ACTS[act])
    np.testing.assert_allclose(np.array(out), np.array(case["exp"][act]), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("n_m", [1, 2, 4, 8])
@pytest.mark.parametrize("act", [0, 1, 2])
def test_brute_force_agrees(n_m, act):
    rng = np.random.default_rng(7 + n_m * 10 + act)
    for T, d, h in [(1, 3, 2), (4, 16, 16), (3, 9, 5)]:
        x, W, M = random_logical(rng, T, d, h, n_m)
        ref = np.array(brute.mglu_logical(x.tolist(), W.tolist(), M.tolist(), act))
        out = c_oracle_logical(x, W, M, act)
        scale = max(1.0, float(np.abs(ref).max()))
        assert np.abs(out - ref).max() <= 1e-12 * scale


def test_elems_match_full():
    rng = np.random.default_rng(3)
    x, W, M = random_logical(rng, 5, 24, 11, 4)
    Ws, masks = logical_to_storage(W, M)
    pk = oracle.pack_masks(masks)
    full, _ = oracle.forward(x, Ws, pk, 4, oracle.ACT_GELU)
    b = rng.integers(0, 5, 40)
    j = rng.integers(0, 11, 40)
    el, _ = oracle.forward_elems(x, Ws, pk, 4, oracle.ACT_GELU, b, j)
    np.testing.assert_array_equal(el, full[b, j])


# ---------------------------------------------------------------- invariant
def test_gate_plus_value_is_dense():
    """x (M . W) + x ((1 - M) . W) = x W for every mask ("Approach": the two
    subspaces are complementary)."""
    rng = np.random.default_rng(11)
    x, W, M = random_logical(rng, 2, 64, 8, 8, p=0.3)
    Ws, masks = logical_to_storage(W, M)
    pk = oracle.pack_masks(masks)
    for b in range(2):
        for j in range(8):
            D, g, v, absw, res = oracle.gate_value(x, Ws, pk, 8, b, j)
            assert res <= 1e-12 * absw
            np.testing.assert_allclose(D, float(x[b] @ W[:, j]), rtol=1e-12, atol=1e-14)
            for i in range(8):
                sel = M[i, :, j].astype(bool)
                np.testing.assert_allclose(g[i], float(x[b, sel] @ W[sel, j]), rtol=1e-12, atol=1e-14)
                np.testing.assert_allclose(v[i], float(x[b, ~sel] @ W[~sel, j]), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- exact special cases
@pytest.mark.parametrize("act", [0, 1, 2])
def test_all_ones_single_mask_is_zero(act):
    """n_m = 1 with every weight in the gate: the value is empty, out = 0."""
    rng = np.random.default_rng(5)
    x, W, _ = random_logical(rng, 3, 32, 16, 1)
    M = np.ones((1, 32, 16), dtype=np.uint8)
    out = c_oracle_logical(x, W, M, act)
    assert np.all(out == 0.0)


@pytest.mark.parametrize("n_m", [1, 2, 4, 8])
@pytest.mark.parametrize("act", [0, 1, 2])
def test_all_zeros_masks_give_zero(n_m, act):
    """Every mask empty: each gate is 0 and act(0) = 0 for all three acts."""
    rng = np.random.default_rng(6)
    x, W, _ = random_logical(rng, 3, 32, 16, n_m)
    M = np.zeros((n_m, 32, 16), dtype=np.uint8)
    out = c_oracle_logical(x, W, M, act)
    assert np.all(out == 0.0)


def test_reduces_to_swiglu():
    """With d = 2d', x = [x', x'], W = [W_g; W_v] and one mask that is 1 on
    the W_g half, MGLU is SwiGLU: silu(x' W_g) * (x' W_v).  The right side is
    torch's own silu / gelu / relu in float64."""
    rng = np.random.default_rng(21)
    T, dp, h = 4, 24, 10
    xp = rng.standard_normal((T, dp))
    Wg = rng.standard_normal((dp, h)) * 0.3
    Wv = rng.standard_normal((dp, h)) * 0.3
    x = np.concatenate([xp, xp], axis=1)
    W = np.concatenate([Wg, Wv], axis=0)
    M = np.zeros((1, 2 * dp, h), dtype=np.uint8)
    M[0, :dp, :] = 1
    gate = torch.from_numpy(xp @ Wg)
    val = torch.from_numpy(xp @ Wv)
    fns = {0: torch.nn.functional.silu, 1: torch.nn.functional.gelu, 2: torch.relu}
    for act, fn in fns.items():
        ref = (fn(gate) * val).numpy()
        out = c_oracle_logical(x, W, M, act)
        np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- symmetries
def test_mask_permutation_invariance():
    rng = np.random.default_rng(8)
    x, W, M = random_logical(rng, 3, 20, 9, 4)
    a = c_oracle_logical(x, W, M, 0)
    b = c_oracle_logical(x, W, M[[2, 0, 3, 1]], 0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_identical_masks_scale():
    rng = np.random.default_rng(9)
    x, W, M = random_logical(rng, 3, 20, 9, 1)
    one = c_oracle_logical(x, W, M, 1)
    four = c_oracle_logical(x, W, np.repeat(M, 4, axis=0), 1)
    np.testing.assert_allclose(four, 4 * one, rtol=1e-12, atol=1e-14)


def test_complementary_pair():
    """Masks M and 1 - M give act(g) v + act(v) g: the sum of the two
    single-mask outputs."""
    rng = np.random.default_rng(10)
    x, W, M = random_logical(rng, 3, 20, 9, 1)
    pair = np.concatenate([M, 1 - M], axis=0)
    for act in (0, 1, 2):
        a = c_oracle_logical(x, W, M, act)
        b = c_oracle_logical(x, W, 1 - M, act)
        both = c_oracle_logical(x, W, pair, act)
        np.testing.assert_allclose(both, a + b, rtol=1e-12, atol=1e-14)


def test_relu_homogeneity():
    """ReLU-MGLU is homogeneous of degree 2 in x (exact for c = 2)."""
    rng = np.random.default_rng(12)
    x, W, M = random_logical(rng, 3, 20, 9, 4)
    a = c_oracle_logical(x, W, M, 2)
    b = c_oracle_logical(2 * x, W, M, 2)
    np.testing.assert_array_equal(b, 4 * a)


# ---------------------------------------------------------------- down-projection
def test_down_matches_numpy():
    rng = np.random.default_rng(13)
    hid = rng.standard_normal((5, 33))
    Wd = rng.standard_normal((17, 33))
    y = oracle.down(hid, Wd)
    np.testing.assert_allclose(y, hid @ Wd.T, rtol=1e-12, atol=1e-12)
    b = np.array([0, 4, 2])
    c = np.array([16, 0, 5])
    ye = oracle.down_elems(hid, Wd, b, c)
    np.testing.assert_allclose(ye, (hid @ Wd.T)[b, c], rtol=1e-12, atol=1e-12)


def test_down_brute():
    rng = np.random.default_rng(14)
    hid = rng.standard_normal((2, 7))
    Wd = rng.standard_normal((3, 7))
    ref = np.array(brute.matmul_logical(hid.tolist(), Wd.T.tolist()))
    np.testing.assert_allclose(oracle.down(hid, Wd), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- packed format
def test_pack_known_bytes():
    """n_m = 4, h = 1, d = 2: weight k = 0 carries bits (1,0,1,1) for masks
    0..3 -> low nibble 0b1101; weight k = 1 carries (0,1,0,0) -> high nibble
    0b0010; the byte is 0x2D."""
    masks = np.array([[[1, 0]], [[0, 1]], [[1, 0]], [[1, 0]]], dtype=np.uint8)  # [i][j][k]
    assert oracle.pack_masks(masks).tolist() == [0x2D]
    # n_m = 8: one byte per weight, bit i = mask i
    m8 = np.zeros((8, 1, 2), dtype=np.uint8)
    m8[0, 0, 0] = m8[7, 0, 0] = 1
    m8[3, 0, 1] = 1
    assert oracle.pack_masks(m8).tolist() == [0x81, 0x08]
    # n_m = 1: eight weights per byte, LSB first
    m1 = np.zeros((1, 1, 8), dtype=np.uint8)
    m1[0, 0, [0, 2, 7]] = 1
    assert oracle.pack_masks(m1).tolist() == [0x85]


@pytest.mark.parametrize("n_m", [1, 2, 4, 8])
def test_pack_matches_brute_and_roundtrips(n_m):
    rng = np.random.default_rng(100 + n_m)
    d, h = 16, 5
    M = (rng.random((n_m, d, h)) < 0.5).astype(np.uint8)
    _, masks = logical_to_storage(np.zeros((d, h)), M)
    pk = oracle.pack_masks(masks)
    assert bytes(pk) == brute.pack_logical(M.tolist())
    np.testing.assert_array_equal(oracle.unpack_masks(pk, n_m, d, h), masks)


# ---------------------------------------------------------------- planted mistakes
def _pin_suite(fwd):
    """Run the pins above against a candidate forward fwd(x, W_log, M_log, act)
    (logical tensors, lists in and out).  Returns the names of failed pins."""
    failed = []
    for case in parse_golden():
        for a, act in ACTS.items():
            out = np.array(fwd(case["x"], case["W"], case["M"], act))
            if not np.allclose(out, np.array(case["exp"][a]), rtol=1e-9, atol=1e-12):
                failed.append(f"hand:{case['name']}:{a}")
    rng = np.random.default_rng(4)
    dp, h = 3, 2
    xp = rng.standard_normal((2, dp))
    Wg = rng.standard_normal((dp, h))
    Wv = rng.standard_normal((dp, h))
    x = np.concatenate([xp, xp], 1)
    W = np.concatenate([Wg, Wv], 0)
    M = np.zeros((1, 2 * dp, h), dtype=np.uint8)
    M[0, :dp] = 1
    ref = (torch.nn.functional.silu(torch.from_numpy(xp @ Wg)) * torch.from_numpy(xp @ Wv)).numpy()
    if not np.allclose(np.array(fwd(x.tolist(), W.tolist(), M.tolist(), 0)), ref, rtol=1e-9):
        failed.append("swiglu")
    ones = np.ones((1, 4, 3), dtype=np.uint8)
    xr = rng.standard_normal((2, 4))
    Wr = rng.standard_normal((4, 3))
    if np.any(np.array(fwd(xr.tolist(), Wr.tolist(), ones.tolist(), 0)) != 0):
        failed.append("all_ones")
    return failed


def test_pins_pass_on_brute_force():
    assert _pin_suite(brute.mglu_logical) == []


def _mutant(kind):
    def fwd(x, W, M, act):
        T, d, h, n_m = len(x), len(W), len(W[0]), len(M)
        out = []
        for b in range(T):
            row = []
            for j in range(h):
                total = 0.0
                for i in range(n_m):
                    g = v = 0.0
                    for k in range(d):
                        kk = k
                        if kind == "drop_first_k" and k == 0:
                            continue
                        w = W[kk][j]
                        sel = M[i][k][j]
                        if kind == "swap_gate_value":
                            sel = 1 - sel
                        if sel:
                            g += x[b][k] * w
                        else:
                            v += x[b][k] * w
                    if kind == "value_is_dense":
                        v = g + v
                    term = brute.act_ref(act, g) * v
                    if kind == "wrong_sign":
                        term = -term
                    total += term
                if kind == "mean_not_sum":
                    total /= n_m
                row.append(total)
            out.append(row)
        return out
    return fwd


@pytest.mark.parametrize("kind", ["swap_gate_value", "drop_first_k", "value_is_dense",
                                  "wrong_sign", "mean_not_sum"])
def test_each_planted_mistake_fails_a_pin(kind):
    assert _pin_suite(_mutant(kind)), f"mutant {kind} passed every pin"


def test_gelu_is_exact_erf_not_tanh():
    """The GELU reading is z * Phi(z) with the exact erf; the tanh
    approximation differs by more than 1e-4 at z = 2 and must not pass."""
    z = 2.0
    exact = z * 0.5 * (1 + math.erf(z / math.sqrt(2)))
    tanh_form = 0.5 * z * (1 + math.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))
    assert abs(oracle.activation(oracle.ACT_GELU, z) - exact) < 1e-15
    assert abs(exact - tanh_form) > 1e-5


# ---------------------------------------------------------------- input recipe (host logic)
def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38, 1e-40], dtype=np.float32)
    bits = inputs.f32_to_bf16_bits(vals)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6: ties to even -> 1+2^-6
    exp = np.array([1.0, 1.0, 1.0 + 2 ** -6, -2.5], dtype=np.float64)
    np.testing.assert_array_equal(inputs.bf16_bits_to_f64(bits[:4]), exp)
    back = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, back)


def test_make_case_is_seeded_and_shaped():
    a = inputs.make_case(3, 16, 8, 4, seed=5, with_down=True)
    b = inputs.make_case(3, 16, 8, 4, seed=5, with_down=True)
    assert a.x.storage.shape == (3, 16) and a.W.storage.shape == (8, 16)
    assert a.masks.shape == (4, 8, 16) and a.W_down.storage.shape == (16, 8)
    np.testing.assert_array_equal(a.W.storage, b.W.storage)
    np.testing.assert_array_equal(a.masks, b.masks)
    assert set(np.unique(a.masks)) <= {0, 1}
    c = inputs.make_case(1, 64, 64, 2, seed=6, p=0.25)
    assert 0.15 < c.masks.mean() < 0.35
