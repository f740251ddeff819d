"""Multi-rank plumbing on CPU (gloo, world size 2): the N>1 bench path.

Each rank runs its own independent shard; only the timing is reduced (max over
ranks). These tests run the same helpers bench.py uses, with gloo instead of
NCCL, in two spawned processes.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from gated_block_sparse_gate_b200 import dist as gdist

    assert gdist.init("gloo", timeout_s=60)
    r, local, ws = gdist.world()
    gdist.barrier()
    # a device-timed duration differs per rank; the job time is the slowest rank's
    slowest = gdist.max_over_ranks(1.5 + rank)
    seed = gdist.shard_seed(7, rank)
    gdist.barrier()
    gdist.finalize()
    out.put((r, ws, slowest, seed))


@pytest.mark.timeout(120)
def test_two_ranks_reduce_max_and_distinct_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert all(r[2] == 2.5 for r in res)          # max over ranks seen by every rank
    assert res[0][3] == 7 and res[1][3] != 7       # rank 0 keeps the workload seed


def test_single_process_is_a_no_op():
    from gated_block_sparse_gate_b200 import dist as gdist

    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert gdist.world() == (0, 0, 1)
    assert gdist.init("gloo") is False
    assert gdist.max_over_ranks(3.25) == 3.25
