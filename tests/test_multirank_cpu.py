"""Host logic of the data-parallel (row-sharded) bench path, on two gloo ranks.

The layer's token rows are independent, so N GPUs each run the whole layer on
their own batch of rows with replicated weights and no collective on the data
path.  The only collectives are the bench's timing reductions (a barrier and a
max over ranks).  These tests run that logic as two CPU processes over gloo.
"""
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from activation_sparse_gemm_lynx_b200 import workloads

        assert bench.dist_env() == (rank, rank, world)
        # the timing reduction: every rank gets the slowest rank's time
        got = bench.max_over_ranks(1.5 + rank, world)
        bench.barrier(world)
        inp = workloads.make_rank_inputs("tiny", rank)
        digests = {k: (None if v is None else bytes(np.ascontiguousarray(v).view(np.uint8)[:4096]))
                   for k, v in inp.items()}
        gathered = [None] * world
        dist.all_gather_object(gathered, digests)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([got], dtype=np.float64))
        if rank == 0:
            same = {k: all(g[k] == gathered[0][k] for g in gathered) for k in digests}
            np.save(os.path.join(out_dir, "same.npy"),
                    np.array([same[k] for k in ("X", "W", "bias", "A", "B")]))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_sharded_inputs(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for rank in range(world):
        got = np.load(tmp_path / f"rank{rank}.npy")[0]
        assert got == 2.5, "max over ranks must return the slowest rank's time on every rank"
    same = np.load(tmp_path / "same.npy")
    # X differs per rank; weights, bias and LoRA factors are replicated
    assert list(same) == [False, True, True, True, True]


def test_rank_inputs_keep_config_on_rank0():
    from activation_sparse_gemm_lynx_b200 import workloads

    a = workloads.make_rank_inputs("tiny", 0)
    b = workloads.make_config_inputs("tiny")
    for k in a:
        assert np.array_equal(a[k], b[k])
    c = workloads.make_rank_inputs("tiny", 1)
    assert c["X"].shape == a["X"].shape and not np.array_equal(c["X"], a["X"])


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"])
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_weak_scaling_value_counts_all_ranks(world):
    import bench

    # value = all ranks' dense-equivalent flops / the slowest rank's time
    flops = 2.0 * 4608 * 12288 * 3072
    assert bench.aggregate_tflops(flops, 0.2, world) == pytest.approx(world * flops / 0.2e-3 / 1e12)


def test_reference_arm_line_on_rank0(monkeypatch, capsys):
    """The reference arm (the oracle on the host cores) prints one JSON line with
    the contract's keys, on the tiny workload."""
    import json

    import bench

    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("LOCAL_RANK", "0")
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "1",
                             "--warmup", "3"])
    assert bench.run_reference(args) == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["cpu"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["gpu_launches"] == 0


def test_cpu_baseline_reports_cores_model_and_single_thread():
    import bench
    from activation_sparse_gemm_lynx_b200 import workloads

    shape = workloads.CONFIGS["tiny"]
    inp = workloads.make_config_inputs("tiny")
    b = bench.cpu_baseline(inp, shape, 0.5)
    assert b["value"] > 0 and b["cores"] >= 1 and b["kind"] == "oracle" and b["cpu"]
    st = b["single_thread"]
    assert st["cores"] == 1 and st["value"] > 0
