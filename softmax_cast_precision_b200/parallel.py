"""Head-sharded forward pass over several GPUs (one process per GPU).

The attention of different (batch, head) slabs is independent, so the work
shards by heads with no exchange during the computation: rank r takes a
contiguous range of key/value heads together with the query heads that read
them, runs the forward pass on its shard, and one all-gather over the
process group (NCCL over NVLink/NVSwitch on GPUs) assembles the full output
on every rank.  Shards of unequal size (Hkv not a multiple of the world size)
are padded to the largest shard for the all-gather and trimmed afterwards.
"""
from __future__ import annotations

import torch


def kv_head_range(Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous kv heads [k0, k1) of `rank`: as even as possible, the first
    Hkv % world ranks take one more; ranks past Hkv get an empty range."""
    if world < 1 or not 0 <= rank < world or Hkv < 0:
        raise ValueError("need 0 <= rank < world and Hkv >= 0")
    base, extra = divmod(Hkv, world)
    k0 = rank * base + min(rank, extra)
    return k0, k0 + base + (1 if rank < extra else 0)


def fwd_head_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool, p_scale: float = 256.0,
                     kv_order="reverse", group=None, compute=None):
    """Forward pass of q [B,H,N,d], k, v [B,Hkv,N,d] with the heads split across the ranks of `group`.

    Every rank passes the full inputs (each uses only its shard) and gets the
    full (o [B,H,N,d], lse [B,H,N]).  ``compute(q, k, v, causal=, p_scale=,
    kv_order=)`` runs one shard and returns (o, lse); it defaults to the
    library's ``fwd``.  All ranks make the same collective calls in the same
    order.
    """
    import torch.distributed as dist

    if compute is None:
        from .fp8attn import fwd as compute
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, H, N, d = (int(x) for x in q.shape)
    Hkv = int(k.shape[1])
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    rep = H // Hkv
    k0, k1 = kv_head_range(Hkv, world, rank)
    width = max(kv_head_range(Hkv, world, r)[1] - kv_head_range(Hkv, world, r)[0] for r in range(world)) * rep
    o_pad = torch.zeros((B, width, N, d), dtype=torch.bfloat16, device=q.device)
    lse_pad = torch.zeros((B, width, N), dtype=torch.float32, device=q.device)
    if k1 > k0:
        o_loc, lse_loc = compute(q[:, k0 * rep:k1 * rep].contiguous(), k[:, k0:k1].contiguous(),
                                 v[:, k0:k1].contiguous(), causal=causal, p_scale=p_scale, kv_order=kv_order)
        o_pad[:, :(k1 - k0) * rep] = o_loc
        lse_pad[:, :(k1 - k0) * rep] = lse_loc
    o_all = [torch.empty_like(o_pad) for _ in range(world)]
    lse_all = [torch.empty_like(lse_pad) for _ in range(world)]
    dist.all_gather(o_all, o_pad, group=group)
    dist.all_gather(lse_all, lse_pad, group=group)
    o_parts, lse_parts = [], []
    for r in range(world):
        r0, r1 = kv_head_range(Hkv, world, r)
        o_parts.append(o_all[r][:, :(r1 - r0) * rep])
        lse_parts.append(lse_all[r][:, :(r1 - r0) * rep])
    return torch.cat(o_parts, dim=1), torch.cat(lse_parts, dim=1)
