"""The multi-GPU bench path on CPU: two gloo ranks (one process each), the
same reduction and throughput arithmetic bench.py uses under torchrun.  The
layer is token-parallel with read-only weights, so N GPUs run N replicas and
the only cross-rank step is the max of the per-rank step times."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measures" (step, kernel 2, kernel 1) = (1 + r, 0.5 + r, 3 - r) ms
        got = bench.max_over_ranks([1.0 + rank, 0.5 + rank, 3.0 - rank], "cpu")
        value = bench.job_throughput(world, 1e12, got[0])
        dist.barrier()
        out[rank] = (got, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        got, value = res[r]
        assert got == [2.0, 1.5, 3.0]            # element-wise max over the ranks
        assert value == pytest.approx(world * 1e12 / 2e-3 / 1e12)   # whole job, slowest rank


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.0, 2.0], "cpu") == [1.0, 2.0]
    assert bench.job_throughput(1, 2e12, 1.0) == pytest.approx(2000.0)


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    """Under torchrun only rank 0 runs the CPU oracle and prints its line."""
    sys.path.insert(0, ROOT)
    import bench
    from bit_diffusion_transformer_w4a4_b200 import workloads as W
    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 1, 2
    bench.run_reference(A(), W.workloads()["fc1_nvfp4"][0])
    assert capsys.readouterr().out == ""
