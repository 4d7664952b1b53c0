"""The replica plumbing bench.py uses for N > 1 GPUs, exercised with world_size 2 on
gloo over CPU: barrier, max-over-ranks of the measured time, whole-job rate."""
import os
import socket

import torch.multiprocessing as mp

from context_packed_sequence_cp_b200 import replicas


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    info = replicas.init_from_env(backend="gloo", timeout_s=30)
    replicas.barrier(info)
    elapsed = 1.0 + rank          # rank 1 is the slow one
    m = replicas.max_over_ranks(info, elapsed)
    out[rank] = (m, replicas.whole_job_rate(10.0, info.world, m))
    replicas.finalize(info)


def test_two_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert out[0] == out[1] == (2.0, 10.0)


def test_single_process_needs_no_group():
    info = replicas.RankInfo(0, 1, 0, False)
    assert replicas.max_over_ranks(info, 3.5) == 3.5
    assert replicas.whole_job_rate(8.0, 1, 2.0) == 4.0
