"""mglu_forward_decode_static: the decode kernel with the library's built-in
scratch instead of a caller buffer.

The file name sorts last, so in a full run these tests come after every other
GPU test in the same process; they also pass on their own, where the first
call here is the one that sets the built-in scratch up."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from masked_glu_b200 import inputs, mglu

from gpu_util import assert_close, device_case, oracle_packed, to_f64

MAX_ROWS = 262144  # MGLU_STATIC_SCRATCH_MAX_ROWS

# (n_m, T, d, h): one token block (NT = 1) and two-block (NT = 2) launches,
# row counts with ragged row blocks and with row blocks split across CTAs.
CASES = [(4, 1, 2048, 8192), (8, 9, 4096, 1000), (2, 16, 384, 72), (1, 3, 1152, 40), (8, 5, 640, 200)]


def test_header_declares_limit():
    text = open(mglu.HEADER).read()
    assert f"#define MGLU_STATIC_SCRATCH_MAX_ROWS {MAX_ROWS}" in text


def test_rejects_before_any_launch():
    """Argument errors come back before anything touches the device, so this
    runs without a GPU (the pointers are never dereferenced)."""
    L = mglu.lib()
    p = ctypes.c_void_p(1 << 20)
    rc = L.mglu_forward_decode_static(p, 1, 128, p, MAX_ROWS + 1, p, 4, 0, p, None)
    assert rc == -1  # MGLU_ERR_INVALID
    assert str(MAX_ROWS) in mglu.last_cuda_error()
    assert L.mglu_forward_decode_static(p, 17, 128, p, 64, p, 4, 0, p, None) == -2  # UNSUPPORTED
    assert L.mglu_forward_decode_static(p, 1, 128, p, 64, p, 3, 0, p, None) == -2
    assert L.mglu_forward_decode_static(p, 1, 100, p, 64, p, 4, 0, p, None) == -3  # d % 8
    assert L.mglu_forward_decode_static(p, 0, 128, p, 64, p, 4, 0, p, None) == 0  # T == 0: no-op


@pytest.mark.gpu
@pytest.mark.parametrize("n_m,T,d,h", CASES)
def test_two_calls_match_forward(n_m, T, d, h):
    prev = mglu.set_decode_max_tokens(16)
    try:
        case = inputs.make_case(T, d, h, n_m, seed=7100 + 17 * n_m + T)
        x, W, packed, _ = device_case(case)
        ref = mglu.forward(x, W, packed, n_m, "swish")
        first = mglu.forward_decode_static(x, W, packed, n_m, "swish")
        second = mglu.forward_decode_static(x, W, packed, n_m, "swish")
        assert mglu.last_device_status() == 0
        assert torch.equal(first, ref), "first call differs from mglu_forward"
        assert torch.equal(second, ref), "second call differs from mglu_forward"
        if h * d <= 1 << 21:
            want, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, oracle.ACT_SWISH)
            assert_close(to_f64(second), want, "bf16", f"static scratch n_m={n_m} T={T}")
    finally:
        mglu.set_decode_max_tokens(prev)


@pytest.mark.gpu
def test_interleaved_with_caller_scratch():
    """Calls on the built-in scratch and on a caller buffer, alternated on one
    stream, each give the same bits."""
    case = inputs.make_case(4, 1024, 3000, 4, seed=7200)
    x, W, packed, _ = device_case(case)
    outs = []
    for _ in range(2):
        outs.append(mglu.forward_decode_static(x, W, packed, 4, "gelu"))
        outs.append(mglu.forward(x, W, packed, 4, "gelu"))
    assert mglu.last_device_status() == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert np.isfinite(to_f64(outs[0])).all()
