"""Multi-process host logic of the bench (replicas on N ranks): the timed
region is the slowest rank's, the work is summed over ranks.  Runs as two
gloo ranks on the CPU; no GPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        mx = bench.reduce_max(10.0 + rank, w)
        sm = bench.reduce_sum(1.0 + rank, w)
        # rank r times 100 + 50 r ms for 2 steps of 3e12 FLOP each
        max_ms, tflops = bench.aggregate(3e12, 2, 100.0 + 50.0 * rank, w)
        out[rank] = (r, w, local, mx, sm, max_ms, tflops)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], codes
    for rank in range(world):
        r, w, local, mx, sm, max_ms, tflops = res[rank]
        assert (r, w, local) == (rank, world, rank)
        assert mx == 11.0 and sm == 3.0
        # slowest rank: 150 ms for 2 steps; work: 2 ranks x 2 steps x 3e12 FLOP
        assert max_ms == 150.0
        assert tflops == pytest.approx(2 * 2 * 3e12 / 0.150 / 1e12)


def test_single_process_aggregation_is_identity():
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.reduce_sum(3.5, 1) == 3.5
    max_ms, tflops = bench.aggregate(4e12, 5, 250.0, 1)
    assert max_ms == 250.0 and tflops == pytest.approx(5 * 4e12 / 0.25 / 1e12)
