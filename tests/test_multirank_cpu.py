"""The multi-GPU path of bench.py is replicas only: every rank runs its own copy of
the workload and the job's step time is the slowest rank's.  This checks that
plumbing with two gloo ranks on the CPU (no GPU, no collective on the data path)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        # rank r pretends its replica took (1 + r) ms per step for 1e9 bytes
        value, ms = bench.whole_job_value(1e9, 1.0 + rank, ws)
        bench._barrier(ws)
        q.put((rank, value, ms))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ws", [2])
def test_replicas_report_whole_job_value_with_slowest_rank(ws):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(ws))
    for rank, value, ms in got:
        assert ms == pytest.approx(float(ws))                 # max over ranks
        assert value == pytest.approx(ws * 1e9 / (ws * 1e-3) / 1e9)  # all ranks' bytes / slowest time


def test_single_rank_is_identity():
    import bench
    v, ms = bench.whole_job_value(2e9, 4.0, 1)
    assert ms == 4.0 and v == pytest.approx(2e9 / 4e-3 / 1e9)
