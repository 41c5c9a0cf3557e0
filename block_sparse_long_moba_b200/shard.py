"""Head-parallel MoBA across GPUs: one process per GPU, each owning a contiguous range of kv-head
groups.

Everything the method computes for a query head — its gate scores against the centroids of its
kv head, its routing, its attention over that kv head's keys — involves only that head and its
kv head [MoBA paper summary (atlas.scime.ai), "Approach": per-head top-k routing over mean-pooled
keys]. A kv head together with the query heads that read it (contiguous GQA groups: query head h
reads kv head h // (Hq / Hkv)) is therefore an independent problem, and N ranks can split the Hkv
groups with no exchange on the data path: rank r runs moba_attn_fwd on q[:, its heads],
k[:, its kv heads], v[:, its kv heads] of the full sequence. This is how a sequence too long for
one GPU at the full head count (e.g. 10M tokens of the Llama-3.1-8B shape: 82 GB of Q alone)
fits: each rank holds 1/N of the heads of every tensor.

The only collective is optional and sits after the computation: gather_heads assembles the full
O [T, Hq, d] and LSE [Hq, T] on every rank with one NCCL all-gather (torch.distributed), for a
caller that needs them whole.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


def kv_groups(world: int, rank: int, hkv: int) -> Tuple[int, int]:
    """Contiguous range [g0, g1) of kv heads owned by `rank` (sizes differ by at most one)."""
    if not (0 <= rank < world) or world < 1:
        raise ValueError(f"rank {rank} outside world {world}")
    if hkv < world:
        raise ValueError(f"{hkv} kv heads cannot be split over {world} ranks")
    base, extra = divmod(hkv, world)
    g0 = rank * base + min(rank, extra)
    return g0, g0 + base + (1 if rank < extra else 0)


def head_range(world: int, rank: int, hq: int, hkv: int) -> Tuple[int, int, int, int]:
    """(h0, h1, g0, g1): the query heads and kv heads of `rank`."""
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    r = hq // hkv
    g0, g1 = kv_groups(world, rank, hkv)
    return g0 * r, g1 * r, g0, g1


def take_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, world: int, rank: int):
    """Contiguous copies of this rank's heads of q [T, Hq, d] and k, v [T, Hkv, d]."""
    h0, h1, g0, g1 = head_range(world, rank, q.shape[1], k.shape[1])
    return (q[:, h0:h1].contiguous(), k[:, g0:g1].contiguous(), v[:, g0:g1].contiguous())


def moba_attn_fwd_heads(q_local: torch.Tensor, k_local: torch.Tensor, v_local: torch.Tensor,
                        cu_seqlens: torch.Tensor, cu_seqlens_host, block_size: int, topk: int,
                        scale: Optional[float] = None, **kw):
    """This rank's share of the forward pass: moba_attn_fwd on its own heads (no collective).
    Returns (o_local [T, h1-h0, d], lse_local [h1-h0, T])."""
    from block_sparse_long_moba_b200 import moba

    return moba.moba_attn_fwd(q_local, k_local, v_local, cu_seqlens, cu_seqlens_host, block_size,
                              topk, scale, **kw)


def gather_heads(o_local: torch.Tensor, lse_local: torch.Tensor, world: int, hq: int, hkv: int,
                 group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather every rank's heads into the full O [T, Hq, d] and LSE [Hq, T] (one collective
    per tensor; ranks may own different head counts when Hkv % world != 0)."""
    import torch.distributed as dist

    T, _, d = o_local.shape
    counts = [head_range(world, r, hq, hkv)[1] - head_range(world, r, hq, hkv)[0]
              for r in range(world)]
    hmax = max(counts)
    # pad to the largest share so that one all-gather moves equal-sized pieces
    o_pad = torch.zeros((hmax, T, d), dtype=o_local.dtype, device=o_local.device)
    o_pad[:o_local.shape[1]] = o_local.permute(1, 0, 2)
    l_pad = torch.zeros((hmax, T), dtype=lse_local.dtype, device=lse_local.device)
    l_pad[:lse_local.shape[0]] = lse_local
    o_all = torch.empty((world * hmax, T, d), dtype=o_local.dtype, device=o_local.device)
    l_all = torch.empty((world * hmax, T), dtype=lse_local.dtype, device=lse_local.device)
    dist.all_gather_into_tensor(o_all, o_pad, group=group)
    dist.all_gather_into_tensor(l_all, l_pad, group=group)
    keep = torch.cat([torch.arange(r * hmax, r * hmax + counts[r]) for r in range(world)])
    keep = keep.to(o_local.device)
    return o_all[keep].permute(1, 0, 2).contiguous(), l_all[keep].contiguous()
