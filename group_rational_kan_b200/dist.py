"""Data-parallel exchange of the coefficient gradients over torch.distributed.

Rows shard across ranks with no halo; the only exchange is dA / dB. Each rank
merges its own partials to float64 sums (grkan_backward_merge with sums64), the
ranks all-gather those n_g x (m+1+n) doubles, and every rank adds the gathered
blocks in rank order (grkan_merge_ranks). The order never depends on the
transport or the topology, so every rank holds bit-identical gradients, and the
result is bit-reproducible from run to run.

The steps are separate functions so that they can be checked one at a time:
``local_sums`` (this rank's backward and float64 sums), ``all_gather_sums``
(the exchange) and ``merge_gathered`` (the rank-order merge on the device).
"""
import torch
import torch.distributed as dist


def all_gather_sums(sums64: torch.Tensor, group=None) -> torch.Tensor:
    """(n_g, K) float64 per rank -> (world, n_g, K), block r from rank r, on the
    device of sums64. Over NCCL the gather runs device to device; a gloo group
    exchanges host copies (n_g (m+1+n) doubles per rank)."""
    world = dist.get_world_size(group)
    flat = sums64.contiguous().view(-1)
    host = sums64.is_cuda and dist.get_backend(group) == "gloo"
    src = flat.cpu() if host else flat
    out = torch.empty((world * flat.numel(),), dtype=sums64.dtype, device=src.device)
    dist.all_gather_into_tensor(out, src, group=group)
    if host:
        out = out.to(sums64.device)
    return out.view((world,) + tuple(sums64.shape))


def local_sums(x, dy, a, b, n_g, dx=None, workspace=None, stream=None):
    """This rank's backward: dx and the float64 coefficient-gradient sums of its
    rows, laid out (n_g, m+1+n) as a_0..a_m then b_1..b_n per group.

    Returns (dx, sums64)."""
    import group_rational_kan_b200 as grk
    B, N, d, dt = grk._dims(x, n_g)
    m = a.shape[-1] - 1
    n = b.shape[-1] if b is not None else 0
    if dx is None:
        dx = torch.empty_like(x)
    dA = torch.empty((n_g, m + 1), dtype=torch.float32, device=x.device)
    dB = torch.empty((n_g, n), dtype=torch.float32, device=x.device)
    wsb = grk.grkan_backward_workspace_bytes(B, N, d, n_g, m, n, dt)
    if workspace is None:
        workspace = torch.empty(max(wsb, 16), dtype=torch.uint8, device=x.device)
    nbytes = workspace.numel() * workspace.element_size()
    sums = torch.empty((n_g, m + 1 + n), dtype=torch.float64, device=x.device)
    st = grk.grkan_backward_partials(x, dy, a, b, dx, B, N, d, n_g, m, n, dt, workspace, nbytes,
                                     0, stream)
    if st == 0:
        st = grk.grkan_backward_merge(workspace, nbytes, dA, dB, sums, B, N, d, n_g, m, n, dt,
                                      stream)
    if st != 0:
        raise grk.GrkanError(st, "local_sums")
    return dx, sums


def merge_gathered(gathered, m, n, stream=None):
    """(world, n_g, m+1+n) float64 blocks in rank order -> (dA, dB) float32,
    added in rank order on the device (grkan_merge_ranks)."""
    import group_rational_kan_b200 as grk
    world, n_g, K = gathered.shape
    assert K == m + 1 + n
    dA = torch.empty((n_g, m + 1), dtype=torch.float32, device=gathered.device)
    dB = torch.empty((n_g, n), dtype=torch.float32, device=gathered.device)
    st = grk.grkan_merge_ranks(gathered.contiguous(), world, dA, dB, n_g, m, n, stream)
    if st != 0:
        raise grk.GrkanError(st, "grkan_merge_ranks")
    return dA, dB


def data_parallel_backward(x, dy, a, b, n_g, group=None, dx=None, workspace=None, stream=None,
                           local=local_sums, merge=merge_gathered):
    """Backward of this rank's rows, with dA / dB summed over every rank.

    Returns (dx, dA, dB); dA and dB are identical bits on every rank. ``local``
    and ``merge`` default to the CUDA implementations above (a test may pass
    stand-ins with the same contract to run the exchange on CPU ranks)."""
    m = a.shape[-1] - 1
    n = b.shape[-1] if b is not None else 0
    dx, sums = local(x, dy, a, b, n_g, dx=dx, workspace=workspace, stream=stream)
    gathered = all_gather_sums(sums, group)
    dA, dB = merge(gathered, m, n, stream=stream)
    return dx, dA, dB
