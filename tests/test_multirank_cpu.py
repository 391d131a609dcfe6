"""The multi-rank plumbing of bench.py on CPU: two `gloo` ranks on 127.0.0.1.

Under torchrun each rank runs its own replica of the layer on its own token batch (no
data-path collective); the job's time is the slowest rank's device time and its value
counts every rank's tokens. The reference arm runs on rank 0 only.
"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synth

        bench.dist_barrier(world)
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slower one
        ms = bench.dist_max(local_ms, world, "cpu")
        value = bench.job_value(64, 20, world, ms)
        # replicas: each rank seeds its own token batch, the weights are shared
        cfg = synth.CONFIGS["tiny"]
        x = synth.host_inputs(cfg, seed=0, x_seed=rank).x
        gathered = [torch.zeros(x.size, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(x.astype("int32").ravel()))

        class Args:
            steps, warmup = 1, 1

        ref = bench.run_reference(Args, cfg, world, rank) if rank != 0 else "rank0"
        out[rank] = (ms, value, bool((gathered[0] != gathered[1]).any()), ref is None)
        bench.dist_barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_job_value():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, value, differ, ref_none = res[rank]
        assert ms == 15.0                       # every rank sees the slowest rank's time
        assert value == pytest.approx(64 * 20 * 2 / 0.015)
        assert differ                           # replicas hold different token batches
    assert res[1][3]                            # rank 1 does no reference work
