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
