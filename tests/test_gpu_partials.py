"""GPU check of the decomposition the method rests on ("Masked Gated Linear
Unit", "Approach": each mask splits the one weight matrix into a gate part
M_i . W and a value part (1 - M_i) . W).  The decode kernel's unrounded
partial sums (mglu_forward_partials: D, g_i, v_i in float32) are compared with
the oracle's float64 sums element by element, the invariant g_i + v_i = D is
checked on the GPU's own values, and the act-sum formed from those partials
is checked against the kernel's own output.

Bound on a partial sum: every one of the d - 1 additions of a d-term float32
sum has a relative error of at most 2^-23 (round to nearest gives 2^-24; the
bound also covers truncating adders), so |err| <= (d - 1) 2^-23 sum_k |x_k W_jk|
for D and for h_i = x (S_i . W); g_i = (D + h_i) / 2 and v_i = (D - h_i) / 2
add one rounding of at most 2^-24 |D +- h_i| <= 2^-23 sum_k |x_k W_jk|.  So
d 2^-23 sum_k |x_k W_jk| bounds all three.  A single wrong mask bit moves a
gate by one term, about sum_k |x_k W_jk| / d, which is above that bound for
the widths used here."""
import numpy as np
import pytest
import torch

import oracle
from masked_glu_b200 import inputs
from masked_glu_b200 import mglu

from gpu_util import device_case, oracle_packed, to_device, to_f64

pytestmark = pytest.mark.gpu
U32 = 2.0 ** -23


@pytest.fixture(autouse=True, scope="module")
def _built():
    from masked_glu_b200 import build
    build.build()
    mglu.set_decode_max_tokens(16)


def _device(case):
    if case.n_m == 0:  # the dense product alone: the mask stream is not read
        return to_device(case.x), to_device(case.W), torch.zeros(16, dtype=torch.uint8, device="cuda")
    x, W, packed, _ = device_case(case)
    return x, W, packed


def _oracle_packed(case):
    return np.zeros(16, dtype=np.uint8) if case.n_m == 0 else oracle_packed(case)


def _planes(case):
    x, W, packed = _device(case)
    gv = mglu.forward_partials(x, W, packed, case.n_m)
    torch.cuda.synchronize()
    assert mglu.last_device_status() == 0
    return gv.cpu().numpy().astype(np.float64), (x, W, packed)


def _check_elements(case, gv, elems):
    """Compare D, g_i, v_i of the listed (token, row) pairs with the oracle."""
    pk = _oracle_packed(case)
    n_m, d = case.n_m, case.d
    for b, j in elems:
        D, g, v, absw, _ = oracle.gate_value(case.x.values, case.W.values, pk, n_m, b, j)
        bound = d * U32 * absw + 1e-30
        assert abs(gv[0, b, j] - D) <= bound, f"D[{b},{j}] {gv[0, b, j]} vs {D} (bound {bound:.3e})"
        for i in range(n_m):
            assert abs(gv[1 + 2 * i, b, j] - g[i]) <= bound, f"g_{i}[{b},{j}] {gv[1 + 2 * i, b, j]} vs {g[i]}"
            assert abs(gv[2 + 2 * i, b, j] - v[i]) <= bound, f"v_{i}[{b},{j}] {gv[2 + 2 * i, b, j]} vs {v[i]}"


def _check_invariant(gv, n_m):
    D = gv[0]
    for i in range(n_m):
        g, v = gv[1 + 2 * i], gv[2 + 2 * i]
        # two float32 roundings on the GPU: (D + h)/2 and (D - h)/2
        assert np.all(np.abs(g + v - D) <= U32 * (np.abs(g) + np.abs(v)) + 1e-38), f"g_{i} + v_{i} != D"


def _swish(z):
    return z / (1.0 + np.exp(-z))


@pytest.mark.parametrize("n_m,d,h,T", [
    (8, 512, 200, 1),
    (8, 256, 48, 2),
    (4, 256, 72, 3),
    (2, 1024, 100, 8),
    (1, 64, 40, 16),
    (4, 520, 33, 9),   # ragged k-stage and row block
    (0, 256, 64, 5),
])
def test_partials_match_oracle_elementwise(n_m, d, h, T):
    case = inputs.make_case(T, d, h, n_m, seed=700 + n_m * 11 + d + h + T)
    gv, (x, W, packed) = _planes(case)
    assert gv.shape == (2 * n_m + 1, T, h)
    _check_elements(case, gv, [(b, j) for b in range(T) for j in range(h)])
    _check_invariant(gv, n_m)
    if n_m > 0:
        # the act-sum of the kernel's own partials is the kernel's output,
        # up to its one bf16 rounding and float32 arithmetic
        out = to_f64(mglu.forward(x, W, packed, n_m, "swish"))
        ref = sum(_swish(gv[1 + 2 * i]) * gv[2 + 2 * i] for i in range(n_m))
        scale = sum(np.abs(_swish(gv[1 + 2 * i]) * gv[2 + 2 * i]) for i in range(n_m))
        assert np.all(np.abs(out - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * scale + 1e-30)


@pytest.mark.parametrize("T", [1, 16])
def test_partials_full_size_samples(T):
    """d = 4096, h = 14336, n_m = 8: every row block kind (split between CTAs
    or whole) on sampled elements, and the invariant on every element."""
    case = inputs.make_case(T, 4096, 14336, 8, seed=7100 + T)
    gv, _ = _planes(case)
    rng = np.random.default_rng(5)
    rows = np.concatenate([np.arange(0, 16), np.arange(14336 - 16, 14336), rng.integers(0, 14336, 48)])
    toks = [0, T - 1]
    _check_elements(case, gv, [(b, int(j)) for b in sorted(set(toks)) for j in rows])
    _check_invariant(gv, 8)


def test_partials_reject_prefill_sizes():
    case = inputs.make_case(17, 64, 16, 2, seed=3)
    x, W, packed = _device(case)
    with pytest.raises(mglu.MGLUError) as e:
        mglu.forward_partials(x, W, packed, 2)
    assert e.value.status == mglu.ERR_UNSUPPORTED
