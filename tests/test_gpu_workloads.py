"""GPU parity at the full benchmark sizes (Llama-style FFN shapes), in the
launch configuration the benchmark times.  The oracle computes exact samples
of the outputs one element at a time: whole output rows of chosen tokens plus
random (token, column) pairs."""
import numpy as np
import pytest
import torch

import oracle
from masked_glu_b200 import inputs
from masked_glu_b200 import mglu

from gpu_util import assert_close, device_case, oracle_packed, to_f64

pytestmark = pytest.mark.gpu
ACT = {"swish": oracle.ACT_SWISH, "gelu": oracle.ACT_GELU, "relu": oracle.ACT_RELU}


@pytest.fixture(autouse=True, scope="module")
def _built():
    from masked_glu_b200 import build
    build.build()
    mglu.set_decode_max_tokens(16)


def sample(T, h, rows_of, n_rand, seed):
    rng = np.random.default_rng(seed)
    b = [np.full(h, t) for t in rows_of] + [rng.integers(0, T, n_rand)]
    j = [np.arange(h) for _ in rows_of] + [rng.integers(0, h, n_rand)]
    return np.concatenate(b), np.concatenate(j)


def test_decode_d2048_h8192_nm4_full():
    w = inputs.WORKLOADS["decode_d2048_h8192_nm4"]
    case = inputs.make_case(w["T"], w["d"], w["h"], w["n_m"], seed=inputs.WORKLOAD_SEEDS["decode_d2048_h8192_nm4"])
    x, W, packed, _ = device_case(case)
    got = to_f64(mglu.forward(x, W, packed, case.n_m, "swish"))
    assert mglu.last_device_status() == 0
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), case.n_m, ACT["swish"])
    assert_close(got, ref, "bf16", "decode d2048 h8192 n_m4")


@pytest.fixture(scope="module")
def c3():
    w = inputs.WORKLOADS["decode_d4096_h14336_nm8"]
    case = inputs.make_case(16, w["d"], w["h"], w["n_m"], seed=inputs.WORKLOAD_SEEDS["decode_d4096_h14336_nm8"])
    x, W, packed, _ = device_case(case)
    return case, x, W, packed, oracle_packed(case)


@pytest.mark.parametrize("T", [1, 2, 4, 8, 16])
def test_decode_d4096_h14336_nm8_sweep(c3, T):
    case, x, W, packed, opk = c3
    got = to_f64(mglu.forward(x[:T].contiguous(), W, packed, 8, "swish"))
    assert mglu.last_device_status() == 0
    b, j = sample(T, case.h, [0, T - 1], 3000, seed=T)
    ref, _ = oracle.forward_elems(case.x.values[:T], case.W.values, opk, 8, ACT["swish"], b, j)
    assert_close(got[b, j], ref, "bf16", f"decode d4096 h14336 n_m8 T={T}")


@pytest.mark.parametrize("act", ["swish", "gelu"])
def test_prefill_T4096_d2048_h8192_nm4(act):
    w = inputs.WORKLOADS["prefill_T4096_d2048_h8192_nm4"]
    case = inputs.make_case(w["T"], w["d"], w["h"], w["n_m"],
                            seed=inputs.WORKLOAD_SEEDS["prefill_T4096_d2048_h8192_nm4"])
    x, W, packed, _ = device_case(case)
    got = to_f64(mglu.forward(x, W, packed, case.n_m, act))
    assert mglu.last_device_status() == 0
    b, j = sample(case.T, case.h, [0, 1337, case.T - 1], 4000, seed=11)
    ref, _ = oracle.forward_elems(case.x.values, case.W.values, oracle_packed(case), case.n_m, ACT[act], b, j)
    assert_close(got[b, j], ref, "bf16", f"prefill T4096 {act}")


@pytest.fixture(scope="module", params=[0.25, 0.5, 0.75])
def c5(request):
    w = inputs.WORKLOADS["ffn_d4096_h14336_nm8"]
    p = request.param
    case = inputs.make_case(2048, w["d"], w["h"], w["n_m"], seed=inputs.WORKLOAD_SEEDS["ffn_d4096_h14336_nm8"],
                            p=p, with_down=True)
    x, W, packed, Wd = device_case(case)
    return p, case, x, W, packed, Wd, oracle_packed(case)


@pytest.mark.parametrize("T", [1, 16, 64, 512, 2048])
def test_ffn_block_d4096_h14336_nm8(c5, T):
    p, case, x, W, packed, Wd = c5[:6]
    opk = c5[6]
    if p != 0.5 and T not in (1, 2048):
        pytest.skip("mask density sweep at the ends of the token sweep only")
    y = to_f64(mglu.forward_down(x[:T].contiguous(), W, packed, 8, Wd, "swish"))
    assert mglu.last_device_status() == 0
    toks = sorted({0, T // 2, T - 1})
    bs = np.repeat(toks, case.h)
    js = np.tile(np.arange(case.h), len(toks))
    hid, _ = oracle.forward_elems(case.x.values[:T], case.W.values, opk, 8, ACT["swish"], bs, js)
    hid = hid.reshape(len(toks), case.h)
    rows = np.repeat(np.arange(len(toks)), case.d)
    cols = np.tile(np.arange(case.d), len(toks))
    ref = oracle.down_elems(hid, case.W_down.values, rows, cols)
    got = y[np.repeat(toks, case.d), cols]
    assert_close(got, ref, "bf16", f"ffn block T={T} p={p}", exact_check=False)


# Edge sizes: the widest Llama-style FFN hidden (h = 53248) and a very deep
# reduction (d = 16384), through the decode and tensor-core paths, checked on
# whole output rows of chosen tokens plus random elements.
@pytest.mark.parametrize("n_m,T,d,h", [(4, 1, 2048, 53248), (8, 16, 1024, 53248), (2, 5, 16384, 1024),
                                       (4, 300, 16384, 512), (1, 33, 256, 53248)])
def test_edge_sizes(n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=4100 + n_m + T)
    x, W, packed, _ = device_case(case)
    got = to_f64(mglu.forward(x, W, packed, n_m, "swish"))
    assert mglu.last_device_status() == 0
    b, j = sample(T, h, [0, T - 1], 3000, seed=T + h)
    ref, _ = oracle.forward_elems(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"], b, j)
    assert_close(got[b, j], ref, "bf16", f"edge n_m={n_m} T={T} d={d} h={h}")
