"""Multi-process host path of the benchmark with two gloo ranks on CPU.

Ranks exchange no solver data (each vector is an independent problem); the
benchmark only needs a barrier, the maximum of the per-rank device times and
per-rank inputs. These run here without a GPU."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from entropy_constrained_unbiased_b200 import dist as D
    from entropy_constrained_unbiased_b200 import workloads as W
    r, n = D.setup("gloo", timeout_s=60)
    D.barrier()
    t_max = D.max_over_ranks(10.0 + 5.0 * r)
    t_sum = D.sum_over_ranks(1.0 + r)
    X = W.make_inputs("small", rank=r)
    D.barrier()
    D.teardown()
    q.put((r, n, t_max, t_sum, float(X[0, :8].sum())))


@pytest.mark.parametrize("world", [2])
def test_two_ranks_barrier_max_and_inputs(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out.sort()
    assert [o[0] for o in out] == list(range(world))
    assert all(o[1] == world for o in out)
    assert all(o[2] == 10.0 + 5.0 * (world - 1) for o in out)   # max over ranks on every rank
    assert all(o[3] == sum(1.0 + r for r in range(world)) for o in out)
    assert out[0][4] != out[1][4]                                # ranks draw different vectors


def test_single_process_is_a_no_op():
    from entropy_constrained_unbiased_b200 import dist as D
    os.environ.pop("WORLD_SIZE", None)
    assert D.world()[1] == 1
    assert D.max_over_ranks(3.5) == 3.5
    D.barrier()
