"""The tensor-parallel FFN block's host side on CPU: the shard ranges, the
slicing of one layer, and the all-reduce over two gloo ranks (as torchrun
launches one process per GPU).  Each rank's partial here comes from the oracle
on that rank's shard (the library computes it on a GPU); the reduced result
must equal the oracle's FFN block on the whole layer."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from masked_glu_b200 import inputs
from masked_glu_b200 import tp


@pytest.mark.parametrize("h", [0, 1, 15, 16, 17, 200, 14336])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shard_ranges_cover_the_hidden_units_once(h, world):
    ranges = [tp.shard_range(h, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == h
    for (a0, a1), (b0, b1) in zip(ranges, ranges[1:]):
        assert a1 == b0 and a0 <= a1
    sizes = [j1 - j0 for j0, j1 in ranges]
    for j0, j1 in ranges:
        assert j0 % tp.ROW_BLOCK == 0 or j0 == h
    # whole blocks split evenly: shard sizes differ by at most one block
    full = [s for s, (j0, j1) in zip(sizes, ranges) if j1 < h]
    if full:
        assert max(full) - min(full) <= tp.ROW_BLOCK


def test_shard_range_rejects_bad_arguments():
    with pytest.raises(ValueError):
        tp.shard_range(64, 2, 2)
    with pytest.raises(ValueError):
        tp.shard_range(64, 0, 0)


@pytest.mark.parametrize("n_m", [1, 2, 4, 8])
def test_shard_layer_slices_rows_bytes_and_columns(n_m):
    d, h, world = 24, 70, 3
    case = inputs.make_case(1, d, h, n_m, seed=40 + n_m, with_down=True)
    W = torch.from_numpy(case.W.values)
    packed = torch.from_numpy(oracle.pack_masks(case.masks))
    Wd = torch.from_numpy(case.W_down.values)
    for r in range(world):
        s = tp.shard_layer(W, packed, Wd, n_m, world, r)
        assert torch.equal(s.W, W[s.j0:s.j1])
        assert s.W_down.is_contiguous() and torch.equal(s.W_down, Wd[:, s.j0:s.j1])
        # the shard's packed bytes are the packing of the shard's masks
        ref = oracle.pack_masks(np.ascontiguousarray(case.masks[:, s.j0:s.j1, :]))
        assert np.array_equal(s.packed.numpy(), ref)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, n_m, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = inputs.make_case(3, 32, 100, n_m, seed=77 + n_m, with_down=True)
        W = torch.from_numpy(case.W.values)
        packed = torch.from_numpy(oracle.pack_masks(case.masks))
        Wd = torch.from_numpy(case.W_down.values)
        s = tp.shard_layer(W, packed, Wd, n_m, world, rank)
        if s.j1 > s.j0:
            hid, _ = oracle.forward(case.x.values, s.W.numpy(), s.packed.numpy(), n_m, oracle.ACT_SWISH)
            y_r = torch.from_numpy(oracle.down(hid, s.W_down.numpy()))
        else:
            y_r = torch.zeros((3, 32), dtype=torch.float64)
        y = tp.reduce_partial(y_r)
        hid, _ = oracle.forward(case.x.values, case.W.values, oracle.pack_masks(case.masks), n_m, oracle.ACT_SWISH)
        ref = oracle.down(hid, case.W_down.values)
        q.put((rank, float(np.max(np.abs(y.numpy() - ref))), float(np.max(np.abs(ref)))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
@pytest.mark.parametrize("n_m", [2, 8])
def test_two_ranks_all_reduce_the_partials_to_the_full_block(world, n_m):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, n_m, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == list(range(world))
    for _, err, scale in res:
        # float64 sums regrouped by shard: a few ulps of the largest output
        assert err <= 1e-12 * scale
