"""GPU parity of the training-path pieces against the float64 oracle of
oracle/train.py, through the C ABI: packing the forward masks straight from
FP16 mask logits ("Masked Gated Linear Unit", "Limitations": masks are held
as FP16 logits while training)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import train as otrain
from masked_glu_b200 import inputs, mglu

from gpu_util import device_case

pytestmark = pytest.mark.gpu

SPECIAL = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x03FF, 0x0400, 0x7BFF, 0x7C00, 0xFC00, 0x7C01, 0x7E00,
                    0xFE00, 0x3C00, 0xBC00], dtype=np.uint16)  # +-0, subnormals, max, +-inf, NaNs, +-1


def _logits(n_m, h, d, seed):
    rng = np.random.default_rng(seed)
    z = (rng.standard_normal((n_m, h, d)) * 2.0).astype(np.float16)
    bits = z.view(np.uint16).reshape(-1)
    idx = rng.choice(bits.size, size=min(bits.size, 4 * SPECIAL.size), replace=False)
    bits[idx] = np.resize(SPECIAL, idx.size)
    return bits.reshape(n_m, h, d).view(np.float16)


@pytest.mark.parametrize("n_m,d,h", [(8, 8, 3), (4, 16, 5), (2, 64, 7), (1, 128, 9), (1, 13, 3), (2, 5, 7),
                                     (4, 100, 37), (8, 4096, 130), (4, 2048, 33)])
def test_pack_mask_logits_bit_exact(n_m, d, h):
    z = _logits(n_m, h, d, seed=2000 + n_m + d + h)
    got = mglu.pack_mask_logits(torch.from_numpy(z).cuda()).cpu().numpy()
    with np.errstate(invalid="ignore"):
        want = oracle.pack_masks(otrain.binarize(z))
    np.testing.assert_array_equal(got, want)


def test_forward_from_logits_equals_forward_from_masks():
    """Masks packed from logits drive the forward exactly as the same masks
    packed from bytes."""
    n_m, T, d, h = 4, 3, 512, 96
    z = _logits(n_m, h, d, seed=2100)
    case = inputs.make_case(T, d, h, n_m, seed=2101)
    with np.errstate(invalid="ignore"):
        case.masks = otrain.binarize(z)
    x, W, packed, _ = device_case(case)
    from_logits = mglu.pack_mask_logits(torch.from_numpy(z).cuda())
    assert torch.equal(from_logits, packed)
    a = mglu.forward(x, W, from_logits, n_m, "swish")
    b = mglu.forward(x, W, packed, n_m, "swish")
    assert torch.equal(a, b)


# ------------------------------------------------------------------ backward (straight-through)
def _abs_refs(x, Ws, masks, a, dout, tokens=None, rows=None):
    """Sums of absolute terms of each gradient element, from the oracle's
    pieces: |dx| <= sum_i |a_i - c_i| |M_i.W| + |sum_i c_i| |W| and so on.
    The kernel rounds each coefficient a_i - c_i and sum_i c_i to bf16 once
    (relative error at most 2^-9) before fp32 products, so the error of an
    element is at most 2^-9 times its absolute-term sum, plus fp32 rounding."""
    x = np.asarray(x, dtype=np.float64)
    Ws = np.asarray(Ws, dtype=np.float64)
    m = np.asarray(masks, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    n_m = m.shape[0]
    res = {}
    if tokens is not None or rows is None:
        xt = x if tokens is None else x[tokens]
        dt = dout if tokens is None else dout[tokens]
        g, v = otrain.gates_values(xt, Ws, m)
        csum = sum(dt * otrain.act(a, g[i]) for i in range(n_m))
        adx = np.abs(csum) @ np.abs(Ws)
        for i in range(n_m):
            coef = dt * (otrain.act_grad(a, g[i]) * v[i] - otrain.act(a, g[i]))
            adx += np.abs(coef) @ (m[i] * np.abs(Ws))
        res["dx"] = adx
    if rows is not None or tokens is None:
        Wr = Ws if rows is None else Ws[rows]
        mr = m if rows is None else m[:, rows]
        dr = dout if rows is None else dout[:, rows]
        g, v = otrain.gates_values(x, Wr, mr)
        csum = sum(dr * otrain.act(a, g[i]) for i in range(n_m))
        adW = np.abs(csum).T @ np.abs(x)
        adM = np.zeros((n_m,) + Wr.shape)
        for i in range(n_m):
            coef = dr * (otrain.act_grad(a, g[i]) * v[i] - otrain.act(a, g[i]))
            aE = np.abs(coef).T @ np.abs(x)
            adW += mr[i] * aE
            adM[i] = np.abs(Wr) * aE
        res["dW"], res["dM"] = adW, adM
    return res


def _grad_bound_check(got, ref, absref, what):
    """|err| <= 2^-8 * (sum of absolute terms) + 1e-5 rms(ref) per element:
    twice the coefficients' one bf16 rounding, plus fp32 accumulation."""
    got = np.asarray(got, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = 2.0 ** -8 * absref + 1e-5 * rms
    err = np.abs(got - ref)
    k = int(np.argmax(err - bound))
    assert np.all(err <= bound), (f"{what}: |err| {err.flat[k]:.3e} > {bound.flat[k]:.3e} (ref {ref.flat[k]:.3e}, "
                                  f"abs-term sum {absref.flat[k]:.3e})")
    # and the bulk is far tighter than the worst case
    assert float(np.sqrt(np.mean((got - ref) ** 2))) <= 1e-2 * rms, f"{what}: rms error above 1e-2 rms"


# the last three run the recompute on CTA pairs (more than 128 tokens, packed
# rows 16-byte strided); (2, 129, 200, 100) reads its mask bits directly
@pytest.mark.parametrize("n_m,T,d,h", [(4, 40, 256, 96), (8, 17, 128, 48), (2, 129, 200, 100), (1, 64, 136, 72),
                                       (4, 300, 256, 100), (8, 260, 128, 40), (1, 200, 256, 72)])
@pytest.mark.parametrize("act", ["swish", "gelu", "relu"])
def test_backward_matches_oracle(n_m, T, d, h, act):
    case = inputs.make_case(T, d, h, n_m, seed=2700 + n_m + T + d)
    x, W, packed, _ = device_case(case)
    rng = np.random.default_rng(2701 + T)
    dout = inputs.normal(rng, (T, h), 1.0, "bf16")
    dx, dW, dM = mglu.backward(x, W, packed, n_m, torch.from_numpy(dout.storage.view(np.int16)).view(torch.bfloat16)
                               .cuda(), act)
    assert mglu.last_device_status() == 0
    a = {"swish": otrain.ACT_SWISH, "gelu": otrain.ACT_GELU, "relu": otrain.ACT_RELU}[act]
    rdx, rdW, rdM = otrain.backward(case.x.values, case.W.values, case.masks, a, dout.values)
    ab = _abs_refs(case.x.values, case.W.values, case.masks, a, dout.values)
    _grad_bound_check(dx.cpu().numpy(), rdx, ab["dx"], f"dx {act}")
    _grad_bound_check(dW.cpu().numpy(), rdW, ab["dW"], f"dW {act}")
    _grad_bound_check(dM.cpu().numpy(), rdM, ab["dM"], f"dlogits {act}")


def test_backward_full_size_sampled():
    """The prefill-shaped layer (T = 4096, d = 2048, h = 8192, n_m = 4):
    dx of sampled tokens and dW / dlogits of sampled rows of W."""
    T, d, h, n_m = 4096, 2048, 8192, 4
    case = inputs.make_case(T, d, h, n_m, seed=2800)
    x, W, packed, _ = device_case(case)
    rng = np.random.default_rng(2801)
    dout = inputs.normal(rng, (T, h), 1.0, "bf16")
    dx, dW, dM = mglu.backward(x, W, packed, n_m,
                               torch.from_numpy(dout.storage.view(np.int16)).view(torch.bfloat16).cuda(), "swish")
    toks = np.array([0, 1337, T - 1])
    rows = np.array([0, 4097, h - 1])
    rdx, rdW, rdM = otrain.backward_sampled(case.x.values, case.W.values, case.masks, otrain.ACT_SWISH, dout.values,
                                            toks, rows)
    abx = _abs_refs(case.x.values, case.W.values, case.masks, otrain.ACT_SWISH, dout.values, tokens=toks)
    abw = _abs_refs(case.x.values, case.W.values, case.masks, otrain.ACT_SWISH, dout.values, rows=rows)
    _grad_bound_check(dx.cpu().numpy()[toks], rdx, abx["dx"], "dx sampled")
    _grad_bound_check(dW.cpu().numpy()[rows], rdW, abw["dW"], "dW sampled")
    _grad_bound_check(dM.cpu().numpy()[:, rows], rdM, abw["dM"], "dlogits sampled")


def test_backward_without_logit_gradients():
    case = inputs.make_case(24, 128, 64, 4, seed=2900)
    x, W, packed, _ = device_case(case)
    dout = torch.randn(24, 64, device="cuda").to(torch.bfloat16)
    dx1, dW1, dM1 = mglu.backward(x, W, packed, 4, dout, "gelu")
    dx2, dW2, dM2 = mglu.backward(x, W, packed, 4, dout, "gelu", with_logits=False)
    assert dM2 is None and torch.equal(dx1, dx2) and torch.equal(dW1, dW2)
