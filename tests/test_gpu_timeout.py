"""The bounded-wait failure path of the tensor-core kernel, driven on purpose
in a test-only build of the library (libmglu_testhooks.so): there, every
mbarrier wait gives up after 20 ms, and mglu_test_set_stall(1) makes the
kernel's producer stop after the loads of its first stage (T = 300: the kernel
on CTA pairs, both producers stop; T = 40: the weights-on-M kernel; d = 200:
the one-CTA token-major kernel, whose builders load the mask bytes
themselves).  Every load it did
issue still lands and is waited for, every MMA issued is drained before TMEM
is released, and every other wait of the CTA runs out, records
MGLU_ERR_TIMEOUT in the device status word and returns.  No trap, no fault,
no unbounded wait: the context stays usable, and the next call is correct."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from masked_glu_b200 import inputs

from gpu_util import assert_close, device_case, oracle_packed, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def hooks():
    from masked_glu_b200 import build
    L = ctypes.CDLL(build.build_test_hooks())
    P, I64, I32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    L.mglu_forward.restype = I32
    L.mglu_forward.argtypes = [P, I64, I64, P, I64, P, I32, I32, I32, P, P, SZ, P]
    L.mglu_forward_path.restype = I32
    L.mglu_forward_path.argtypes = [I64, I32]
    L.mglu_last_device_status.restype = I32
    L.mglu_last_device_status.argtypes = [P]
    L.mglu_test_set_stall.restype = I32
    L.mglu_test_set_stall.argtypes = [I32]
    return L


def _forward(L, x, W, packed, n_m, out):
    T, d = x.shape
    h = W.shape[0]
    s = torch.cuda.current_stream().cuda_stream
    return L.mglu_forward(x.data_ptr(), T, d, W.data_ptr(), h, packed.data_ptr(), n_m, 0, 0, out.data_ptr(),
                          None, 0, s)


@pytest.mark.parametrize("n_m,T,d,h", [(4, 300, 512, 200), (8, 40, 256, 96), (4, 40, 200, 96)])
def test_stalled_producer_times_out_and_the_next_call_is_correct(hooks, n_m, T, d, h):
    L = hooks
    case = inputs.make_case(T, d, h, n_m, seed=1800 + n_m + T)
    x, W, packed, _ = device_case(case)
    assert L.mglu_forward_path(T, 0) == 1  # the tensor-core kernel
    s = torch.cuda.current_stream().cuda_stream
    assert L.mglu_last_device_status(s) == 0
    out = torch.zeros((T, h), dtype=torch.bfloat16, device="cuda")
    assert L.mglu_test_set_stall(1) == 0
    try:
        assert _forward(L, x, W, packed, n_m, out) == 0
        assert L.mglu_last_device_status(s) == -5  # MGLU_ERR_TIMEOUT
        assert L.mglu_last_device_status(s) == 0   # read and cleared
    finally:
        assert L.mglu_test_set_stall(0) == 0
    out2 = torch.zeros((T, h), dtype=torch.bfloat16, device="cuda")
    assert _forward(L, x, W, packed, n_m, out2) == 0
    assert L.mglu_last_device_status(s) == 0
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, oracle.ACT_SWISH)
    assert_close(to_f64(out2), ref, "bf16", "after a timed-out call")
    assert np.isfinite(to_f64(out2)).all()
