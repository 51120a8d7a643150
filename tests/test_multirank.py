"""The data-parallel exchange on CPU: two gloo ranks, each holding the float64
gradient sums of its own row shard (computed here by the oracle, standing in for
the GPU's grkan_backward_merge), all-gather them, and add them in rank order.
Checks that blocks arrive in rank order, that both ranks end with identical bits,
and that the rank-order total matches the oracle on the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, rows_per_rank, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    import synth
    from group_rational_kan_b200.dist import all_gather_sums
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.workload("kat_t").with_rows(rows_per_rank * world)
        x, dy = w.x(), w.dy()
        a, b = w.coefficients()
        sl = slice(rank * rows_per_rank, (rank + 1) * rows_per_rank)
        g = oracle.coef_grads(x[sl], dy[sl], a, b, w.n_g)
        mine = torch.from_numpy(np.concatenate([g["dA"], g["dB"]], axis=1).copy())
        gathered = all_gather_sums(mine)
        total = torch.zeros_like(mine)
        for r in range(world):
            total += gathered[r]
        q.put((rank, gathered.numpy().copy(), total.numpy().copy(), mine.numpy().copy()))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, None, repr(e), None))
        raise
    finally:
        dist.destroy_process_group()


def test_two_rank_gather_is_rank_ordered_and_identical():
    world, rows = 2, 40
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, rows, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, gathered, total, mine = q.get(timeout=180)
        assert gathered is not None, "rank %d failed: %s" % (rank, total)
        results[rank] = (gathered, total, mine)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # block r of every rank's gather is rank r's own sums
    for rank in range(world):
        for r in range(world):
            assert np.array_equal(results[rank][0][r], results[r][2])
    # identical bits on every rank
    assert np.array_equal(results[0][1], results[1][1])
    # and the rank-order total is the whole batch's gradient
    import oracle
    import synth
    w = synth.workload("kat_t").with_rows(rows * world)
    g = oracle.coef_grads(w.x(), w.dy(), *w.coefficients(), w.n_g)
    want = np.concatenate([g["dA"], g["dB"]], axis=1)
    scale = np.concatenate([g["sabs_a"], g["sabs_b"]], axis=1)
    assert np.all(np.abs(results[0][1] - want) <= 1e-12 * scale)
