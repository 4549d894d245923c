"""The tensor-parallel FFN block's per-rank work on one GPU: every rank's
partial (the library's FFN block on that rank's shard of W, its mask bits and
W_down) is computed in turn on cuda:0, and their sum must match the oracle's
block on the whole layer.  (The all-reduce itself is covered over gloo on
CPU; this pool's calls have one GPU.)  Each partial is rounded to bf16 once,
so the bar adds world * 2^-8 * sum_r |y_r| to the usual bf16 bar."""
import numpy as np
import pytest
import torch

import oracle
from masked_glu_b200 import inputs
from masked_glu_b200 import mglu
from masked_glu_b200 import tp

from gpu_util import device_case, oracle_packed, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from masked_glu_b200 import build
    build.build()
    mglu.set_decode_max_tokens(16)


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("n_m,T,d,h", [(8, 1, 512, 1024), (4, 16, 256, 600), (2, 64, 256, 512), (8, 3, 1024, 200)])
def test_shard_partials_sum_to_the_full_block(world, n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=900 + world + n_m + T, with_down=True)
    x, W, packed, Wd = device_case(case)
    parts = []
    for r in range(world):
        s = tp.shard_layer(W, packed, Wd, n_m, world, r)
        parts.append(to_f64(tp.partial(x, s, n_m, "swish")))
    torch.cuda.synchronize()
    assert mglu.last_device_status() == 0
    got = np.sum(parts, axis=0)
    hid, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, oracle.ACT_SWISH)
    # the one-GPU block reads the bf16-rounded hidden activation
    ref = oracle.down(inputs.round_bf16(hid)[0], case.W_down.values)
    rms = float(np.sqrt(np.mean(ref * ref)))
    bound = 1e-2 * rms + 2.0 ** -8 * np.abs(ref) + world * 2.0 ** -8 * np.sum(np.abs(parts), axis=0)
    assert np.all(np.abs(got - ref) <= bound)
