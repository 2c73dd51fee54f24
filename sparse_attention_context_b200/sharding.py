"""Head sharding of the ISA forward over ranks (one process per GPU).

Every (b, h) of the ISA forward is an independent unit: pre-selection,
routing and both attention paths are decided per head, so a problem splits
across GPUs by heads with no exchange step.  Each rank runs the C ABI on its
own contiguous slice of heads; only a caller that wants the whole output on
every rank needs one all-gather of the output slices afterwards (NCCL over
NVLink/NVSwitch on GPUs, gloo on CPU tensors).
"""
from __future__ import annotations


def shard_heads(H: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous head range [h0, h1) of `rank`: H split as evenly as
    possible, the first H % world ranks taking one head more."""
    if world < 1 or not 0 <= rank < world or H < 0:
        raise ValueError("bad world/rank/H")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def gather_heads(local, group=None):
    """All-gather of per-rank head slices [B, H_r, N, d] into the whole
    [B, H, N, d] on every rank, in rank order.  The slices may differ in
    size by any amount (``shard_heads`` gives the first H % world ranks one
    head more): each rank pads its slice to the largest H_r, one all-gather
    moves the padded slices, and every rank keeps the first H_r heads of
    each.  Uses the default process group (or `group`); a single process
    returns `local` itself."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return local
    world = dist.get_world_size(group)
    if world == 1:
        return local
    sizes = [torch.zeros(1, dtype=torch.int64, device=local.device) for _ in range(world)]
    dist.all_gather(sizes, torch.tensor([local.shape[1]], dtype=torch.int64, device=local.device), group=group)
    hs = [int(s.item()) for s in sizes]
    hmax = max(hs)
    B, h_r = local.shape[0], local.shape[1]
    if h_r == hmax:
        send = local.contiguous()
    else:
        send = torch.zeros((B, hmax, *local.shape[2:]), dtype=local.dtype, device=local.device)
        send[:, :h_r] = local
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    return torch.cat([p[:, :h] for p, h in zip(parts, hs)], dim=1)
