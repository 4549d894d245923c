"""Helpers shared by the GPU parity tests: move seeded cases to the device,
run the oracle on the same rounded values, compare with the stated bars."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from masked_glu_b200 import inputs
from masked_glu_b200 import mglu

# Parity bars.  bf16 inputs with fp32 accumulation: |err_i| <= 1e-2 * rms(ref)
# + 2^-8 * |ref_i|; the second term is the worst-case error of rounding the
# exact result once to bf16 (8-bit significand, round to nearest even), which
# every bf16 output carries.  On top, at least 98% of bf16 outputs must equal
# the oracle value rounded to bf16 (an accurately accumulated result rounded
# once).  The fp32 path: |err_i| <= 1e-5 * rms(ref).
TOL = {"bf16": 1e-2, "f32": 1e-5}
BF16_UNIT_ROUNDOFF = 2.0 ** -8
MIN_EXACT_FRACTION = 0.98
ACT_NAMES = ["swish", "gelu", "relu"]
GUARD = 64  # guard elements on each side of every output buffer


def to_device(t: inputs.Tensor) -> torch.Tensor:
    if t.dtype == "bf16":
        return torch.from_numpy(t.storage.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(t.storage).cuda()


def guarded(shape, dtype):
    """An output buffer with sentinel-filled guard bands on both sides."""
    n = int(np.prod(shape))
    big = torch.full((n + 2 * GUARD,), 1024.0, dtype=dtype, device="cuda")
    return big, big[GUARD:GUARD + n].view(*shape)


def check_guards(big):
    torch.cuda.synchronize()
    head = big[:GUARD].float().cpu()
    tail = big[-GUARD:].float().cpu()
    assert torch.all(head == 1024.0) and torch.all(tail == 1024.0), "write outside the output buffer"


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def round_bf16(a: np.ndarray) -> np.ndarray:
    return inputs.round_bf16(a)[0]


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str = "", exact_check: bool = True):
    if ref.size == 0:
        return
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(ref * ref)))
    err = np.abs(got - ref)
    if dtype == "bf16":
        bound = TOL[dtype] * rms + BF16_UNIT_ROUNDOFF * np.abs(ref)
    else:
        bound = np.full(ref.shape, TOL[dtype] * rms)
    worst = int(np.argmax(err - bound))
    assert np.all(err <= bound), (f"{what}: |err| {err.flat[worst]:.3e} > bound {bound.flat[worst]:.3e} "
                                  f"(ref {ref.flat[worst]:.4e}, rms {rms:.3e})")
    if dtype == "bf16" and exact_check:
        frac = float(np.mean(got == round_bf16(ref)))
        assert frac >= MIN_EXACT_FRACTION, f"{what}: only {frac:.4f} of outputs equal bf16(oracle)"


def device_case(case: inputs.Case):
    x = to_device(case.x)
    W = to_device(case.W)
    masks = torch.from_numpy(case.masks).cuda()
    packed = mglu.pack_masks(masks)
    Wd = to_device(case.W_down) if case.W_down is not None else None
    return x, W, packed, Wd


def oracle_packed(case: inputs.Case) -> np.ndarray:
    return oracle.pack_masks(case.masks)


def run_forward(case: inputs.Case, act: str):
    x, W, packed, _ = device_case(case)
    big, out = guarded((case.T, case.h), x.dtype)
    mglu.forward(x, W, packed, case.n_m, act, out=out)
    check_guards(big)
    assert mglu.last_device_status() == 0
    return to_f64(out)
