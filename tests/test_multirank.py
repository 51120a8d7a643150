"""The data-parallel exchange on CPU: two gloo ranks run
``dist.data_parallel_backward`` on their own row shards. Its device steps have
CPU stand-ins with the same contract (the oracle's float64 sums of the shard in
the (n_g, m+1+n) layout that ``grkan_backward_merge`` writes to sums64, and a
rank-order float64 addition for ``grkan_merge_ranks``); the orchestration and
the all-gather are the product's. Checks that blocks arrive in rank order, that
both ranks end with identical bits, and that the rank-order total matches the
oracle on the whole batch. The GPU side of the same path (the CUDA local sums
and the rank merge kernel over stacked shards) is tested in
``test_gpu_dataparallel.py``."""
import os
import socket

import numpy as np
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
    from group_rational_kan_b200.dist import data_parallel_backward
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
        mine = {}

        def oracle_local(x, dy, a, b, n_g, dx=None, workspace=None, stream=None):
            g = oracle.coef_grads(x, dy, a, b, n_g)
            s = torch.from_numpy(np.concatenate([g["dA"], g["dB"]], axis=1).copy())
            mine["sums"] = s.numpy().copy()
            return None, s

        def host_merge(gathered, m, n, stream=None):
            mine["gathered"] = gathered.numpy().copy()
            total = gathered[0].clone()
            for r in range(1, gathered.shape[0]):
                total += gathered[r]
            mine["total"] = total.numpy().copy()
            return total[:, :m + 1].float(), total[:, m + 1:].float()

        _, dA, dB = data_parallel_backward(x[sl], dy[sl], a, b, w.n_g, local=oracle_local,
                                           merge=host_merge)
        q.put((rank, mine["gathered"], mine["total"], mine["sums"], dA.numpy(), dB.numpy()))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, None, repr(e), None, None, None))
        raise
    finally:
        dist.destroy_process_group()


def test_two_rank_exchange_is_rank_ordered_and_identical():
    world, rows = 2, 40
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, rows, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, gathered, total, mine, dA, dB = q.get(timeout=180)
        assert gathered is not None, "rank %d failed: %s" % (rank, total)
        results[rank] = (gathered, total, mine, dA, dB)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    import synth
    w = synth.workload("kat_t").with_rows(rows * world)
    K = w.m + 1 + w.n
    # the exchange moves (world, n_g, m+1+n) float64 blocks, block r from rank r
    for rank in range(world):
        assert results[rank][0].shape == (world, w.n_g, K)
        assert results[rank][0].dtype == np.float64
        for r in range(world):
            assert np.array_equal(results[rank][0][r], results[r][2])
    # identical bits on every rank
    assert np.array_equal(results[0][1], results[1][1])
    assert np.array_equal(results[0][3], results[1][3]) and np.array_equal(results[0][4],
                                                                           results[1][4])
    # and the rank-order total is the whole batch's gradient
    g = oracle.coef_grads(w.x(), w.dy(), *w.coefficients(), w.n_g)
    want = np.concatenate([g["dA"], g["dB"]], axis=1)
    scale = np.concatenate([g["sabs_a"], g["sabs_b"]], axis=1)
    assert np.all(np.abs(results[0][1] - want) <= 1e-12 * scale)
    assert np.all(np.abs(results[0][3] - g["dA"]) <= 2 ** -24 * np.abs(g["dA"]) +
                  1e-12 * g["sabs_a"])
