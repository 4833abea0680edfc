"""Multi-GPU plumbing for the page indexer (host side only).

The indexer's work is independent per request, so more GPUs take more
requests with no exchange on the data path: each rank (one process per GPU,
torch.distributed over NCCL on B200 boxes, gloo in CPU tests) scores and
selects its own requests.  What crosses ranks is only bookkeeping: the
slowest rank's time and the total page count, or -- when one batch is split
-- the per-rank index rows gathered back in request order.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank ``rank``'s own synthetic batch (weak scaling)."""
    return base_seed + 1000 * rank


def split_requests(B: int, world: int, rank: int):
    """Contiguous request range [lo, hi) of ``rank`` when one batch of B
    requests is split over ``world`` ranks (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(B, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def reduce_timing(ms: float, units: float, device=None):
    """(max over ranks of ms, sum over ranks of units); identity without a
    process group.  Two scalars, one all-reduce each."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(ms), float(units)
    dev = device if device is not None else torch.device("cpu")
    t = torch.tensor([float(ms)], dtype=torch.float64, device=dev)
    u = torch.tensor([float(units)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def gather_rows(local_rows: torch.Tensor, B: int, device=None) -> torch.Tensor:
    """Gather per-rank result rows (rank r holds requests split_requests(B,
    world, r)) into the full [B, ...] tensor on every rank."""
    if not (dist.is_available() and dist.is_initialized()):
        return local_rows
    world = dist.get_world_size()
    sizes = [split_requests(B, world, r) for r in range(world)]
    width = max(hi - lo for lo, hi in sizes)
    pad = torch.zeros((width,) + tuple(local_rows.shape[1:]), dtype=local_rows.dtype,
                      device=local_rows.device)
    pad[: local_rows.shape[0]] = local_rows
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([parts[r][: hi - lo] for r, (lo, hi) in enumerate(sizes)], dim=0)
