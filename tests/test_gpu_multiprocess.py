"""Two processes on one GPU run the data-parallel backward as two ranks would:
each holds its own row shard, runs this library's backward and float64 merge on
the device (``dist.local_sums``), the ranks exchange their sums over a gloo
process group, and each adds the blocks in rank order on the device
(``grkan_merge_ranks``). No kernel of one rank waits for the other: the only
exchange is on the host. Both ranks must end with the same bits, equal to the
rank-order merge of the same shards done in one process, and within the
coefficient-gradient tolerance of the oracle on the whole batch."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROWS = 1200   # rows per rank
WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, port, q):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import torch.distributed as dist
    import synth
    from group_rational_kan_b200.dist import data_parallel_backward
    from parity import to_torch
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.workload("kat_b").with_rows(ROWS * WORLD)
        x, dy = w.x(), w.dy()
        a, b = w.coefficients()
        sl = slice(rank * ROWS, (rank + 1) * ROWS)
        tx, tdy = to_torch(np.ascontiguousarray(x[sl])), to_torch(np.ascontiguousarray(dy[sl]))
        ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
        dx, dA, dB = data_parallel_backward(tx, tdy, ta, tb, w.n_g)
        torch.cuda.synchronize()
        q.put((rank, dA.cpu().numpy(), dB.cpu().numpy(), None))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, None, None, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def test_two_processes_exchange_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(WORLD):
        rank, dA, dB, err = q.get(timeout=300)
        assert err is None, "rank %d failed: %s" % (rank, err)
        got[rank] = (dA, dB)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # identical bits on both ranks
    assert np.array_equal(got[0][0], got[1][0]) and np.array_equal(got[0][1], got[1][1])

    # the same shards merged in rank order in this process give the same bits
    import oracle
    import synth
    from group_rational_kan_b200.dist import local_sums, merge_gathered
    from parity import check_coef, to_torch
    w = synth.workload("kat_b").with_rows(ROWS * WORLD)
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    tx, tdy = to_torch(x), to_torch(dy)
    blocks = [local_sums(tx[r * ROWS:(r + 1) * ROWS], tdy[r * ROWS:(r + 1) * ROWS], ta, tb,
                         w.n_g)[1] for r in range(WORLD)]
    dA, dB = merge_gathered(torch.stack(blocks), w.m, w.n)
    torch.cuda.synchronize()
    assert np.array_equal(dA.cpu().numpy(), got[0][0])
    assert np.array_equal(dB.cpu().numpy(), got[0][1])
    # and the whole batch's gradients within the coefficient tolerance
    check_coef(got[0][0], got[0][1], oracle.coef_grads(x, dy, a, b, w.n_g), what="2 processes")
