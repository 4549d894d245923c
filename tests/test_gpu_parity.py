"""GPU parity: every kernel of libmglu.so against the float64 oracle, through
the C ABI, on seeded inputs.  Small cases are compared element by element at
sizes that span several tiles with ragged tails; the full-size workloads are
compared on exact samples the oracle computes one element at a time."""
import numpy as np
import pytest
import torch

import oracle
from masked_glu_b200 import inputs
from masked_glu_b200 import mglu

from gpu_util import (ACT_NAMES, assert_close, check_guards, device_case, guarded, oracle_packed, run_forward,
                      to_device, to_f64)

pytestmark = pytest.mark.gpu
ACT = {"swish": oracle.ACT_SWISH, "gelu": oracle.ACT_GELU, "relu": oracle.ACT_RELU}


@pytest.fixture(autouse=True, scope="module")
def _built():
    from masked_glu_b200 import build
    build.build()
    mglu.set_decode_max_tokens(16)


# ------------------------------------------------------------------ packing (bit-exact)
@pytest.mark.parametrize("n_m,d,h", [(8, 8, 3), (4, 16, 5), (2, 64, 7), (1, 128, 9), (1, 8, 1), (8, 4096, 130),
                                     (4, 2048, 33), (2, 24, 5), (1, 40, 3), (1, 13, 3), (2, 5, 7), (4, 100, 37),
                                     (8, 100, 37)])
def test_pack_unpack_bit_exact(n_m, d, h):
    case = inputs.make_case(1, d, h, n_m, seed=7 + d + h + n_m)
    masks = torch.from_numpy(case.masks).cuda()
    packed = mglu.pack_masks(masks)
    want = oracle_packed(case)
    np.testing.assert_array_equal(packed.cpu().numpy(), want)
    back = mglu.unpack_masks(packed, n_m, d, h)
    np.testing.assert_array_equal(back.cpu().numpy(), case.masks)


def test_pack_treats_nonzero_as_one():
    m = torch.tensor([[[0, 7, 255, 1, 0, 0, 2, 0]]], dtype=torch.uint8).cuda()  # n_m=1, h=1, d=8
    assert mglu.pack_masks(m).cpu().tolist() == [0b01001110]


# ------------------------------------------------------------------ fp32 path
def test_fp32_tiny_full():
    w = inputs.WORKLOADS["tiny_f32"]
    case = inputs.make_case(w["T"], w["d"], w["h"], w["n_m"], seed=inputs.WORKLOAD_SEEDS["tiny_f32"], dtype="f32")
    for act in ACT_NAMES:
        got = run_forward(case, act)
        ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), case.n_m, ACT[act])
        assert_close(got, ref, "f32", f"fp32 {act}")


@pytest.mark.parametrize("n_m,T,d,h", [(8, 9, 100, 37), (1, 3, 13 * 8, 5), (4, 1, 64, 70)])
def test_fp32_odd_shapes(n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=31 + T + d, dtype="f32")
    got = run_forward(case, "gelu")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["gelu"])
    assert_close(got, ref, "f32", "fp32 odd")


def test_fp32_down():
    rng = np.random.default_rng(5)
    hid = rng.standard_normal((6, 77)).astype(np.float32)
    Wd = (rng.standard_normal((45, 77)) * 0.02).astype(np.float32)
    big, y = guarded((6, 45), torch.float32)
    mglu.down_proj(torch.from_numpy(hid).cuda(), torch.from_numpy(Wd).cuda(), out=y)
    check_guards(big)
    assert_close(to_f64(y), oracle.down(hid.astype(np.float64), Wd.astype(np.float64)), "f32", "fp32 down")


# ------------------------------------------------------------------ decode kernel (T <= 16)
DECODE_CASES = [
    # n_m, d, h: ragged row block (h % 16 != 0) and ragged k stage (d % 512 != 0);
    # with few units per CTA most row blocks are split between CTAs
    (8, 640, 200),
    (4, 896, 200),
    (2, 384, 72),
    (1, 1152, 40),
    (8, 2048, 256),   # each row block shared by several CTAs
    (8, 4096, 64),
    (4, 128 * 5, 16),  # one row block
    (4, 2048, 8192),   # many units per CTA: whole row blocks inside one CTA
]


@pytest.mark.parametrize("n_m,d,h", DECODE_CASES)
@pytest.mark.parametrize("T", [1, 3, 8, 9, 16])
def test_decode_parity(n_m, d, h, T):
    case = inputs.make_case(T, d, h, n_m, seed=100 + n_m * 7 + d + h + T)
    assert mglu.forward_path(T) == mglu.PATH_DECODE
    got = run_forward(case, "swish")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"])
    assert_close(got, ref, "bf16", f"decode n_m={n_m} d={d} h={h} T={T}")


@pytest.mark.parametrize("act", ACT_NAMES)
@pytest.mark.parametrize("n_m", [1, 2, 4, 8])
def test_decode_acts(act, n_m):
    case = inputs.make_case(5, 512, 48, n_m, seed=200 + n_m)
    got = run_forward(case, act)
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT[act])
    assert_close(got, ref, "bf16", f"decode {act}")


# ------------------------------------------------------------------ prefill kernel (tcgen05)
PREFILL_CASES = [
    # n_m, T, d, h: ragged token tile, ragged weight tile
    (4, 17, 384, 200),
    (4, 129, 640, 200),
    (4, 300, 256, 100),
    (8, 129, 384, 40),
    (8, 200, 512, 72),
    (2, 150, 384, 170),
    (1, 130, 384, 300),
    (1, 40, 256, 128),
]


@pytest.mark.parametrize("n_m,T,d,h", PREFILL_CASES)
def test_prefill_parity(n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=300 + n_m + T + d + h)
    assert mglu.forward_path(T) == mglu.PATH_PREFILL
    got = run_forward(case, "swish")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"])
    assert_close(got, ref, "bf16", f"prefill n_m={n_m} T={T} d={d} h={h}")


# More than 128 tokens with 16-byte strided packed rows run on CTA pairs (256
# tokens per tile; each CTA of a pair holds half of every weight block).
# Cases where the second CTA of the last token tile has no valid token, where
# the last weight tile ends inside the first CTA's half, and several pair tiles
# per CTA pair.
PAIR_CASES = [
    (8, 257, 256, 50),
    # n_m = 8 pairs take 28 weight rows per tile (14 per CTA, padded to 16):
    # a whole tile, one CTA's rows only, a 2-row tail, an odd h
    (8, 300, 192, 28),
    (8, 260, 64, 14),
    (8, 513, 320, 30),
    (8, 400, 128, 57),
    (4, 385, 192, 121),
    (2, 700, 128, 97),
    (1, 640, 320, 200),
    (4, 2100, 128, 1000),
]


@pytest.mark.parametrize("n_m,T,d,h", PAIR_CASES)
def test_prefill_pair_parity(n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=330 + n_m + T + d + h)
    got = run_forward(case, "swish")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"])
    assert_close(got, ref, "bf16", f"prefill pair n_m={n_m} T={T} d={d} h={h}")


@pytest.mark.parametrize("n_m,T,d,h", [(4, 1536, 1024, 3000), (8, 1024, 512, 2000), (1, 2048, 512, 1024)])
def test_prefill_pair_repeatable(n_m, T, d, h):
    """The CTA pairs hand data and accumulators across CTAs through mbarriers;
    any missing ordering shows up as a run that differs.  Thirty back-to-back
    runs must be bit-identical, and the first must match the oracle on an
    exact sample of elements."""
    case = inputs.make_case(T, d, h, n_m, seed=360 + n_m)
    x, W, packed, _ = device_case(case)
    first = torch.empty((T, h), dtype=torch.bfloat16, device="cuda")
    mglu.forward(x, W, packed, n_m, "swish", out=first)
    out = torch.empty_like(first)
    for rep in range(30):
        mglu.forward(x, W, packed, n_m, "swish", out=out)
        torch.cuda.synchronize()
        assert torch.equal(out, first), f"pair prefill n_m={n_m} repeat {rep} differs"
    assert mglu.last_device_status() == 0
    rng = np.random.default_rng(361 + n_m)
    b = rng.integers(0, T, 2000)
    j = rng.integers(0, h, 2000)
    ref, _ = oracle.forward_elems(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"], b, j)
    assert_close(to_f64(first)[b, j], ref, "bf16", f"pair prefill n_m={n_m} sampled")


# up to 128 tokens at n_m = 8, 96 at n_m = 4 and 32 at n_m <= 2: the
# weights-on-M kernel (weight rows on the MMA's M side, tokens on N): ragged
# token counts (NT = T rounded up to 16), 14-, 25-, 42- and 64-row weight
# tiles with ragged last tiles, several tiles per CTA, a ragged last
# k-stage; above those token counts the same shapes take the token-major
# kernels
WM_CASES = [
    (8, 17, 256, 100),
    (8, 40, 512, 14),
    (8, 128, 384, 300),
    (8, 96, 256, 4000),
    (8, 50, 144, 60),
    (8, 113, 320, 29),
    (4, 33, 256, 101),
    (4, 100, 640, 25),
    (2, 64, 384, 170),
    (2, 120, 256, 42),
    (1, 48, 256, 130),
    (1, 128, 512, 64),
    (4, 70, 160, 77),
    (4, 96, 384, 260),
    (4, 17, 128, 50),
    (2, 20, 256, 90),
    (2, 32, 320, 200),
    (1, 32, 384, 130),
    (1, 17, 256, 64),
]


@pytest.mark.parametrize("n_m,T,d,h", WM_CASES)
def test_prefill_wm_parity(n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=370 + n_m + T + d + h)
    got = run_forward(case, "swish")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"])
    assert_close(got, ref, "bf16", f"prefill wm n_m={n_m} T={T} d={d} h={h}")


@pytest.mark.parametrize("n_m,T,d,h", [(8, 100, 1024, 3000), (8, 24, 2048, 1000), (4, 64, 2048, 1000),
                                       (1, 32, 2048, 1000)])
def test_prefill_wm_repeatable(n_m, T, d, h):
    """The epilogue hands a staging buffer between its four warps through two
    mbarriers, chunk after chunk; thirty runs must be bit-identical, and the
    first must match the oracle on an exact sample of elements."""
    case = inputs.make_case(T, d, h, n_m, seed=380 + n_m)
    x, W, packed, _ = device_case(case)
    first = torch.empty((T, h), dtype=torch.bfloat16, device="cuda")
    mglu.forward(x, W, packed, n_m, "swish", out=first)
    out = torch.empty_like(first)
    for rep in range(30):
        mglu.forward(x, W, packed, n_m, "swish", out=out)
        torch.cuda.synchronize()
        assert torch.equal(out, first), f"wm prefill n_m={n_m} repeat {rep} differs"
    assert mglu.last_device_status() == 0
    rng = np.random.default_rng(381 + n_m)
    b = rng.integers(0, T, 2000)
    j = rng.integers(0, h, 2000)
    ref, _ = oracle.forward_elems(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"], b, j)
    assert_close(to_f64(first)[b, j], ref, "bf16", f"wm prefill n_m={n_m} sampled")


@pytest.mark.parametrize("T,want", [(40, {1}), (200, {1}), (1, {1, 2})])
def test_kernel_launch_counter(T, want):
    """One tensor-core launch per forward (one CTA or a CTA pair); the decode
    forward is its kernel plus, when CTAs share a row block, the split kernel."""
    case = inputs.make_case(T, 512, 1000, 4, seed=350 + T)
    x, W, packed, _ = device_case(case)
    out = torch.empty((T, 1000), dtype=torch.bfloat16, device="cuda")
    mglu.forward(x, W, packed, 4, "swish", out=out)
    torch.cuda.synchronize()
    before = mglu.kernel_launches()
    mglu.forward(x, W, packed, 4, "swish", out=out)
    torch.cuda.synchronize()
    assert mglu.kernel_launches() - before in want


@pytest.mark.parametrize("act", ACT_NAMES)
def test_prefill_acts(act):
    case = inputs.make_case(160, 256, 96, 4, seed=401)
    got = run_forward(case, act)
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), 4, ACT[act])
    assert_close(got, ref, "bf16", f"prefill {act}")


def test_prefill_many_tiles_per_cta():
    """More tiles than SMs: each persistent CTA runs several tiles through both
    accumulator buffers.  Checked on an exact sample of elements."""
    T, d, h, n_m = 1024, 256, 2048, 4
    case = inputs.make_case(T, d, h, n_m, seed=402)
    got = run_forward(case, "swish")
    rng = np.random.default_rng(3)
    b = np.concatenate([rng.integers(0, T, 3000), np.repeat([0, T - 1], h)])
    j = np.concatenate([rng.integers(0, h, 3000), np.tile(np.arange(h), 2)])
    ref, _ = oracle.forward_elems(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"], b, j)
    assert_close(got[b, j], ref, "bf16", "prefill many tiles")


def test_decode_limit_zero_routes_small_T_to_prefill():
    case = inputs.make_case(3, 256, 64, 8, seed=403)
    prev = mglu.set_decode_max_tokens(0)
    try:
        assert mglu.forward_path(3) == mglu.PATH_PREFILL
        got = run_forward(case, "swish")
    finally:
        mglu.set_decode_max_tokens(prev)
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), 8, ACT["swish"])
    assert_close(got, ref, "bf16", "prefill at T=3")


# ------------------------------------------------------------------ exact special cases
@pytest.mark.parametrize("T", [2, 40])
def test_single_full_mask_gives_exact_zero(T):
    """n_m = 1 with every weight in the gate: the value is empty, out == 0."""
    case = inputs.make_case(T, 256, 48, 1, seed=500 + T)
    case.masks[:] = 1
    got = run_forward(case, "swish")
    assert np.all(got == 0.0)


@pytest.mark.parametrize("T", [2, 40])
@pytest.mark.parametrize("n_m", [2, 8])
def test_empty_masks_give_exact_zero(T, n_m):
    case = inputs.make_case(T, 256, 48, n_m, seed=510 + T + n_m)
    case.masks[:] = 0
    for act in ACT_NAMES:
        got = run_forward(case, act)
        assert np.all(got == 0.0), act


# ------------------------------------------------------------------ down-projection and FFN block
@pytest.mark.parametrize("T,h,d", [(1, 1088, 200), (5, 1088, 200), (16, 14336, 64), (200, 512, 300),
                                   (17, 192, 40)])
def test_down_proj(T, h, d):
    rng = np.random.default_rng(T + h + d)
    hid = inputs.normal(rng, (T, h), 1.0, "bf16")
    Wd = inputs.normal(rng, (d, h), 0.02, "bf16")
    big, y = guarded((T, d), torch.bfloat16)
    mglu.down_proj(to_device(hid), to_device(Wd), out=y)
    check_guards(big)
    assert_close(to_f64(y), oracle.down(hid.values, Wd.values), "bf16", f"down T={T}")


@pytest.mark.parametrize("T", [1, 16, 64])
def test_forward_down_block(T):
    case = inputs.make_case(T, 256, 1024, 8, seed=600 + T, with_down=True)
    x, W, packed, Wd = device_case(case)
    big, y = guarded((T, 256), torch.bfloat16)
    mglu.forward_down(x, W, packed, 8, Wd, "swish", out=y)
    check_guards(big)
    assert mglu.last_device_status() == 0
    hid, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), 8, ACT["swish"])
    ref = oracle.down(hid, case.W_down.values)
    # the hidden activation is rounded to bf16 before the down-projection, so
    # y is not the oracle's y rounded once: value bar only
    assert_close(to_f64(y), ref, "bf16", f"block T={T}", exact_check=False)


@pytest.mark.parametrize("T", [1, 9])
def test_decode_scratch_needs_no_initialization(T):
    """Row blocks split between CTAs pass their partial sums through the
    scratch; every slot is written before it is read, so a scratch full of
    NaN bit patterns gives the same result as a zeroed one, call after call."""
    case = inputs.make_case(T, 2048, 256, 8, seed=700 + T)
    x, W, packed, _ = device_case(case)
    clean = torch.zeros(mglu.scratch_bytes(256), dtype=torch.uint8, device="cuda")
    want = to_f64(mglu.forward(x, W, packed, 8, "swish", scratch=clean))
    dirty = torch.full((mglu.scratch_bytes(256),), 0xFF, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        got = to_f64(mglu.forward(x, W, packed, 8, "swish", scratch=dirty))
        torch.cuda.synchronize()
        assert np.array_equal(got, want), "result depends on the scratch's prior contents"
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), 8, ACT["swish"])
    assert_close(want, ref, "bf16", f"decode T={T}")


# Repeat tests: every repeat must match the oracle and be bit-identical to
# the first call.  The shapes are those on which an earlier decode kernel
# (a TMA ring shared by all warps of a CTA) gave intermittent wrong rows: the
# dense down-projection with K = 14336, which mixes data-parallel and split
# row blocks; n_m = 4 with eight tokens; n_m = 8 with two token blocks.
@pytest.mark.parametrize("T", [1, 16])
def test_dense_decode_repeatable_k14336(T):
    rng = np.random.default_rng(900 + T)
    hid = inputs.normal(rng, (T, 14336), 1.0, "bf16")
    Wd = inputs.normal(rng, (4096, 14336), 0.02, "bf16")
    hd, wd = to_device(hid), to_device(Wd)
    ref = oracle.down(hid.values, Wd.values)
    first = None
    for rep in range(6):
        y = to_f64(mglu.down_proj(hd, wd))
        assert mglu.last_device_status() == 0
        assert_close(y, ref, "bf16", f"dense decode K=14336 T={T} repeat {rep}")
        if first is None:
            first = y
        assert np.array_equal(y, first), f"repeat {rep} differs from the first call"


@pytest.mark.parametrize("n_m,T,d,h,reps", [(4, 8, 2048, 8192, 40), (4, 4, 2048, 8192, 8), (2, 8, 2048, 4096, 8),
                                            (8, 16, 4096, 2048, 8), (8, 1, 4096, 14336, 8)])
def test_decode_repeatable(n_m, T, d, h, reps):
    case = inputs.make_case(T, d, h, n_m, seed=950 + 31 * n_m + T)
    x, W, packed, _ = device_case(case)
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"])
    first = None
    for rep in range(reps):
        got = to_f64(mglu.forward(x, W, packed, n_m, "swish"))
        assert mglu.last_device_status() == 0
        assert_close(got, ref, "bf16", f"decode n_m={n_m} T={T} repeat {rep}")
        if first is None:
            first = got
        assert np.array_equal(got, first), f"repeat {rep} differs from the first call"


@pytest.mark.parametrize("n_m,T,d,h,down", [(4, 1, 1024, 640, False), (8, 9, 512, 300, False),
                                            (2, 40, 384, 200, False), (8, 16, 256, 1024, True),
                                            (4, 200, 256, 512, True)])
def test_forward_host_matches_device_calls(n_m, T, d, h, down):
    """The host-buffer entry point gives the same bits as the device-pointer
    calls (same kernels), with the copies done inside the library call."""
    case = inputs.make_case(T, d, h, n_m, seed=1200 + T + n_m, with_down=down)
    x, W, packed, Wd = device_case(case)
    x_h = x.cpu().pin_memory()
    if down:
        want = mglu.forward_down(x, W, packed, n_m, Wd, "swish")
        got = mglu.forward_host(x_h, W, packed, n_m, "swish", W_down=Wd)
    else:
        want = mglu.forward(x, W, packed, n_m, "swish")
        got = mglu.forward_host(x_h, W, packed, n_m, "swish")
    torch.cuda.synchronize()
    assert mglu.last_device_status() == 0
    assert torch.equal(got, want.cpu())


def test_workspace_reused_across_token_counts_and_block_modes():
    """One workspace reused by FFN-block calls of different token counts
    (tensor-core hidden write, then decode), and by host-buffer calls with and
    without the down-projection: whatever an earlier call left in it, every
    result must equal the same call made on a fresh workspace."""
    d, h, n_m = 256, 1024, 8
    case = inputs.make_case(512, d, h, n_m, seed=1300, with_down=True)
    x, W, packed, Wd = device_case(case)
    ws = torch.zeros(mglu.workspace_bytes(512, d, h, n_m), dtype=torch.uint8, device="cuda")
    for T in (512, 1, 9, 512, 1):
        xt = x[:T].contiguous()
        got = mglu.forward_down(xt, W, packed, n_m, Wd, "swish", workspace=ws)
        want = mglu.forward_down(xt, W, packed, n_m, Wd, "swish")
        torch.cuda.synchronize()
        assert mglu.last_device_status() == 0
        assert torch.equal(got, want), f"T={T} on a reused workspace differs"
    hws = torch.zeros(mglu.host_workspace_bytes(512, d, h, n_m, torch.bfloat16, True), dtype=torch.uint8,
                      device="cuda")
    for T, down in ((512, True), (1, False), (16, True), (3, False), (1, True)):
        xh = x[:T].cpu().pin_memory()
        got = mglu.forward_host(xh, W, packed, n_m, "swish", W_down=Wd if down else None, workspace=hws)
        want = mglu.forward_host(xh, W, packed, n_m, "swish", W_down=Wd if down else None)
        torch.cuda.synchronize()
        assert mglu.last_device_status() == 0
        assert torch.equal(got, want), f"host call T={T} down={down} on a reused workspace differs"


# ------------------------------------------------------------------ widths that are multiples of 8 only
# The bf16 path accepts any d % 8 == 0 (and h % 8 == 0 for the down-projection).
# Packed mask rows of d * n_m / 8 bytes that are not 16-byte strided cannot be
# described by a tensor map; the tensor-core kernel then reads them directly.
@pytest.mark.parametrize("n_m,T,d,h", [
    (4, 1, 200, 100), (1, 3, 200, 64), (8, 9, 72, 50), (2, 16, 8, 24),        # decode
    (2, 40, 200, 100), (1, 150, 136, 70), (4, 40, 1000, 64), (8, 40, 1000, 72),  # prefill, masks read directly
    (8, 40, 1008, 72), (4, 129, 96, 130),                                       # prefill, ragged last k block
])
def test_widths_multiple_of_8(n_m, T, d, h):
    case = inputs.make_case(T, d, h, n_m, seed=1400 + n_m + T + d + h)
    got = run_forward(case, "swish")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"])
    assert_close(got, ref, "bf16", f"d%8 n_m={n_m} T={T} d={d} h={h}")


@pytest.mark.parametrize("T,h,d", [(1, 200, 40), (9, 72, 136), (40, 200, 72), (300, 200, 136)])
def test_down_proj_h_multiple_of_8(T, h, d):
    rng = np.random.default_rng(1500 + T + h + d)
    hid = inputs.normal(rng, (T, h), 1.0, "bf16")
    Wd = inputs.normal(rng, (d, h), 0.02, "bf16")
    big, y = guarded((T, d), torch.bfloat16)
    mglu.down_proj(to_device(hid), to_device(Wd), out=y)
    check_guards(big)
    assert_close(to_f64(y), oracle.down(hid.values, Wd.values), "bf16", f"down h%8 T={T} h={h}")


# ------------------------------------------------------------------ scale range
def _scaled(case, e):
    """The case with x multiplied by 2^e (exact for bf16 values in range)."""
    vals, bits = inputs.round_bf16(case.x.values * 2.0 ** e)
    assert np.array_equal(vals, case.x.values * 2.0 ** e)
    case.x = inputs.Tensor(vals, bits, "bf16")
    return case


@pytest.mark.parametrize("n_m,T", [(8, 1), (8, 9), (4, 3), (8, 40)])
@pytest.mark.parametrize("e", [-60, 60])
def test_extreme_input_scale_matches_oracle(n_m, T, e):
    """Masks select or negate whole weights, so every product is exact at
    any input scale: outputs at x * 2^-60 and x * 2^60 still meet the bar."""
    case = _scaled(inputs.make_case(T, 512, 96, n_m, seed=1600 + n_m + T), e)
    got = run_forward(case, "swish")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT["swish"])
    assert_close(got, ref, "bf16", f"scale 2^{e} n_m={n_m} T={T}")


@pytest.mark.parametrize("n_m,T", [(8, 1), (4, 16), (8, 40)])
def test_relu_is_homogeneous_of_degree_two(n_m, T):
    """ReLU gating: out(c x) = c^2 out(x) exactly for c = 2^-40 (powers of two
    scale every product, sum and rounding exactly while values stay normal)."""
    base = inputs.make_case(T, 512, 96, n_m, seed=1700 + n_m + T)
    got1 = run_forward(base, "relu")
    got2 = run_forward(_scaled(inputs.make_case(T, 512, 96, n_m, seed=1700 + n_m + T), -40), "relu")
    assert np.array_equal(got2, got1 * 2.0 ** -80)


# ------------------------------------------------------------------ dense-gate ablation
@pytest.mark.parametrize("n_m,T,d,h,dtype", [(4, 1, 512, 200, "bf16"), (8, 9, 256, 96, "bf16"),
                                             (4, 150, 384, 200, "bf16"), (1, 40, 256, 64, "bf16"),
                                             (8, 300, 256, 90, "bf16"), (8, 64, 256, 50, "bf16"),
                                             (2, 5, 100, 37, "f32")])
@pytest.mark.parametrize("act", ["swish", "gelu", "relu"])
def test_dense_gate_matches_oracle(n_m, T, d, h, dtype, act):
    """act | MGLU_GATE_DENSE: out = sum_i act(x W) v_i, on the decode, the
    tensor-core and the fp32 kernels."""
    case = inputs.make_case(T, d, h, n_m, seed=1900 + n_m + T + d, dtype=dtype)
    got = run_forward(case, act + "+dense_gate")
    ref, _ = oracle.forward(case.x.values, case.W.values, oracle_packed(case), n_m, ACT[act] | oracle.GATE_DENSE)
    assert_close(got, ref, dtype, f"dense gate {act} n_m={n_m} T={T}")
