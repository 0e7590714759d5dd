"""Batch sharding (transposed_convolution_02_b200.shard) on CPU: the split of
one caller's batch over ranks, each rank's slice computed on its own, and the
gather that assembles Y, on two and three gloo ranks.  The per-rank compute
is the fp64 oracle here (the library's kernels need a GPU); the split, the
padding of uneven slices and the gather order are the product's code."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from transposed_convolution_02_b200.shard import ShardedConvTranspose, shard_bounds


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_bounds():
    assert shard_bounds(8, 2) == [(0, 4), (4, 8)]
    assert shard_bounds(7, 3) == [(0, 3), (3, 5), (5, 7)]
    assert shard_bounds(2, 4) == [(0, 1), (1, 2), (2, 2), (2, 2)]
    assert shard_bounds(0, 2) == [(0, 0), (0, 0)]
    for n in range(0, 20):
        for w in range(1, 6):
            b = shard_bounds(n, w)
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(b[i][1] == b[i + 1][0] for i in range(w - 1))
            sizes = [hi - lo for lo, hi in b]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_bounds(4, 0)


CASE = dict(x_shape=[5, 6, 7, 8], w_shape=[6, 4, 3, 3], strides=[2, 2], pads=[1, 1, 0, 1])


def _oracle_compute(w, b):
    from oracle import Attrs, conv_transpose_ref
    attrs = Attrs(strides=CASE["strides"], pads=CASE["pads"])

    def run(x_local):
        y, _ = conv_transpose_ref(x_local.double().numpy(), w.double().numpy(),
                                  b.double().numpy(), attrs)
        return torch.from_numpy(y)
    return run


def _rank_main(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(5)
        x = torch.randn(CASE["x_shape"], generator=g)
        w = torch.randn(CASE["w_shape"], generator=g)
        b = torch.randn(4, generator=g)
        sh = ShardedConvTranspose(w, CASE["x_shape"], b, rank=rank, world=world,
                                  compute=_oracle_compute(w, b))
        y_local = sh(sh.local_slice(x))
        y = sh.gather(y_local, dst=0)
        y_all = sh.gather(y_local, all_ranks=True)
        out[rank] = (sh.lo, sh.hi, None if y is None else y.numpy(), y_all.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_batch_on_gloo_ranks(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    g = torch.Generator().manual_seed(5)
    x = torch.randn(CASE["x_shape"], generator=g)
    w = torch.randn(CASE["w_shape"], generator=g)
    b = torch.randn(4, generator=g)
    whole = _oracle_compute(w, b)(x).numpy()
    assert [(out[r][0], out[r][1]) for r in range(world)] == shard_bounds(5, world)
    for r in range(world):
        _, _, y, y_all = out[r]
        assert (y is not None) == (r == 0)
        np.testing.assert_array_equal(y_all, whole)   # the oracle per image is exact
    np.testing.assert_array_equal(out[0][2], whole)
