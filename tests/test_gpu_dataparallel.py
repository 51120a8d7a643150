"""Data-parallel row sharding on one GPU: the batch's rows split into 2 to 4
shards as separate ranks would hold them; every shard runs this library's
backward and float64 merge (``dist.local_sums``), the blocks are stacked in rank
order (the layout ``dist.all_gather_sums`` produces) and ``grkan_merge_ranks``
adds them (``dist.merge_gathered``). The coefficient gradients must match the
oracle on the whole batch, be the same bits from run to run, and, for shards
cut at reduction-tile boundaries, agree with a single device's float64 sums up
to float64 rounding. ``data_parallel_backward`` itself runs over a one-rank
NCCL process group (the exchange then has one block) and must give the bits of
``grkan_backward``. The dA / dB reduction domain is every batch, sequence and
in-group element ("FlashKAT: Understanding and Addressing Performance
Bottlenecks in the Kolmogorov-Arnold Transformer", paper notes, section "2. The
atomic-add problem of the original KAT"); the fixed-order merge is the
two-stage reduction of "PolyKAN: Efficient Fused GPU Operators for Polynomial
Kolmogorov-Arnold Network Variants", abstract, technique (iii)."""
import datetime

import numpy as np
import pytest
import torch
import torch.distributed as dist

import group_rational_kan_b200 as grk
import oracle
import synth
from group_rational_kan_b200.dist import data_parallel_backward, local_sums, merge_gathered
from parity import check_coef, to_torch

pytestmark = pytest.mark.gpu


def _tile_rows(w):
    """Rows per reduction tile: the largest row count that needs one tile."""
    one = grk.grkan_backward_workspace_bytes(1, 1, w.d, w.n_g, w.m, w.n, w.dtype)
    s = 1
    while grk.grkan_backward_workspace_bytes(s + 1, 1, w.d, w.n_g, w.m, w.n, w.dtype) == one:
        s += 1
    return s


CASES = [
    ("kat_t", None, 4000, [2016], True),                # 2 ranks, cut at a tile boundary
    ("kat_t", None, 4000, [1024, 2048, 3072], True),    # 4 ranks
    ("kat_b", None, 3001, [1000, 2333], False),         # 3 ranks, shards cut inside tiles
    ("stress", 64, 1500, [704], True),                  # 64 groups, 2 ranks
]


def _data(name, n_g, rows):
    w = synth.workload(name, n_g=n_g).with_rows(rows)
    x, dy = w.x(), w.dy()
    a, b = w.coefficients()
    return w, x, dy, a, b, to_torch(x), to_torch(dy), torch.from_numpy(a).cuda(), \
        torch.from_numpy(b).cuda()


@pytest.mark.parametrize("name,n_g,rows,cuts,aligned", CASES,
                         ids=["%s_%dranks%s" % (c[0], len(c[3]) + 1, "" if c[4] else "_ragged")
                              for c in CASES])
def test_rank_order_merge_of_row_shards(name, n_g, rows, cuts, aligned):
    w, x, dy, a, b, tx, tdy, ta, tb = _data(name, n_g, rows)
    S = _tile_rows(w)
    assert all(c % S == 0 for c in cuts) == aligned
    bounds = [0] + cuts + [rows]

    def shard_sums():
        dxs, blocks = [], []
        for r in range(len(bounds) - 1):
            dx_r, s_r = local_sums(tx[bounds[r]:bounds[r + 1]], tdy[bounds[r]:bounds[r + 1]],
                                   ta, tb, w.n_g)
            dxs.append(dx_r)
            blocks.append(s_r)
        return dxs, torch.stack(blocks)

    dxs, gathered = shard_sums()
    assert gathered.shape == (len(bounds) - 1, w.n_g, w.m + 1 + w.n)
    dA, dB = merge_gathered(gathered, w.m, w.n)
    torch.cuda.synchronize()
    ref = oracle.coef_grads(x, dy, a, b, w.n_g)
    rel = check_coef(dA.cpu().numpy(), dB.cpu().numpy(), ref, what="%d shards" % len(dxs))
    print("%s, %d shards: max relative error of dA/dB %.3g" % (name, len(dxs), rel))

    # dx does not depend on the sharding: the shards' dx is the batch's, bit for bit
    dx_full, dA1, dB1 = grk.backward(tx, tdy, ta, tb, w.n_g)
    assert torch.equal(torch.cat(dxs), dx_full)

    # the same bits on every run
    for _ in range(2):
        _, g2 = shard_sums()
        assert torch.equal(g2, gathered)
        dA2, dB2 = merge_gathered(g2, w.m, w.n)
        assert torch.equal(dA2, dA) and torch.equal(dB2, dB)

    # one block: the rank merge gives the single-device gradients exactly
    _, whole = local_sums(tx, tdy, ta, tb, w.n_g)
    dAw, dBw = merge_gathered(whole[None], w.m, w.n)
    assert torch.equal(dAw, dA1) and torch.equal(dBw, dB1)
    if aligned:
        # shards cut at tile boundaries hold the same float32 tile partials as the
        # whole batch; only the float64 addition order differs
        scale = torch.from_numpy(np.concatenate([ref["sabs_a"], ref["sabs_b"]], axis=1)).cuda()
        assert torch.all((gathered.sum(0) - whole).abs() <= 1e-12 * scale)


def test_data_parallel_backward_over_a_one_rank_nccl_group(tmp_path):
    w, x, dy, a, b, tx, tdy, ta, tb = _data("kat_b", None, 700)
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dx, dA, dB = data_parallel_backward(tx, tdy, ta, tb, w.n_g)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    rdx, rdA, rdB = grk.backward(tx, tdy, ta, tb, w.n_g)
    assert torch.equal(dx, rdx) and torch.equal(dA, rdA) and torch.equal(dB, rdB)
    assert grk.grkan_device_error()[1] == 0
