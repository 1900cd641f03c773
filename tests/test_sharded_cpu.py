"""Row sharding and the optional Y gather of activation_sparse_gemm_lynx_b200.sharded,
on two and three gloo ranks on CPU.  The layer itself needs the GPU, so these
tests pass a stand-in for it (a float64 matmul of the rank's rows); what they
check is the host logic: which rows a rank owns, that the gathered Y holds
every rank's block in order, and uneven and empty last blocks."""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from activation_sparse_gemm_lynx_b200 import sharded  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("M,world", [(8, 2), (7, 2), (5, 3), (2, 3), (4608, 2)])
def test_row_shards_cover_every_row_once(M, world):
    seen = []
    for r in range(world):
        first, rows = sharded.row_shard(M, world, r)
        seen.extend(range(first, first + rows))
    assert seen == list(range(M))
    with pytest.raises(ValueError):
        sharded.row_shard(M, world, world)


def _rank_main(rank, world, port, M, out_dir):
    import datetime

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from activation_sparse_gemm_lynx_b200 import sharded as sh

        # the same full X and W on every rank; small integers, so every product
        # and sum is exact whatever the blocking of the matmul
        rng = np.random.default_rng(7)
        X = torch.from_numpy(rng.integers(-3, 4, size=(M, 16)).astype(np.float64))
        W = torch.from_numpy(rng.integers(-3, 4, size=(12, 16)).astype(np.float64))
        first, rows = sh.row_shard(M, world, rank)

        def stand_in(x, w, bias, a, b, skip_sparsify=False, workspace=None):
            return x @ w.t()

        y_local = sh.sharded_linear(X[first:first + rows], W, M=M, layer=stand_in)
        assert y_local.shape == (rows, 12)
        y_full = sh.sharded_linear(X[first:first + rows], W, M=M, gather=True, layer=stand_in)
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y_full.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("M,world", [(8, 2), (7, 2), (5, 3), (2, 3)])
def test_gathered_y_holds_every_block_in_order(tmp_path, M, world):
    import torch
    import torch.multiprocessing as mp

    mp.start_processes(_rank_main, args=(world, _free_port(), M, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    rng = np.random.default_rng(7)
    X = rng.integers(-3, 4, size=(M, 16)).astype(np.float64)
    W = rng.integers(-3, 4, size=(12, 16)).astype(np.float64)
    for r in range(world):
        y = np.load(tmp_path / f"y{r}.npy")
        assert y.shape == (M, 12)
        assert np.array_equal(y, X @ W.T), r
