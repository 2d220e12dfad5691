"""The multi-GPU host logic of bench.py on CPU: two gloo ranks take the
maximum of their timings and report the whole-job throughput (weak scaling,
no data-path collective)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.env_rank()
        times = bench.max_over_ranks([10.0 + rank, 20.0 - 3 * rank], "cpu")
        out[rank] = (r, w, local, times, bench.whole_job_tflops(w, 1e12, 4, times[0]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for rank in range(world):
        r, w, local, times, tflops = res[rank]
        assert (r, w, local) == (rank, world, rank)
        assert times == [11.0, 20.0]                      # max over ranks, element-wise
        assert tflops == pytest.approx(world * 1e12 * 4 / 0.011 / 1e12)
