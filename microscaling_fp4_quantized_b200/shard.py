"""One attention problem split across ranks by (batch, head) pairs.

Every (b, h) pair of the problem is an independent attention (its own K mean, its own
rows and keys: the FlashAttention tiling the SageAttention review thread describes in its
reply to Q3 never mixes heads), so N ranks can each take a contiguous slice of the B*H
pairs and run the same forward on it with no exchange at all. The only optional
collective is an all-gather that assembles the full output on every rank.

    lo, hi = head_slice(B * H, world, rank)           # this rank's pairs [lo, hi)
    out_r = attn_slice(q_r, k_r, v_r, causal=...)     # q_r: [hi - lo, N, D] on this rank
    out = gather_heads(out_r, B * H, group)           # optional: [B*H, N, D] everywhere

No TMA multicast and no peer-memory operand is involved: each rank's kernels read only
its own device memory, and the gather is NCCL's (gloo on CPU).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


def head_slice(n_pairs: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous slice [lo, hi) of n_pairs (b, h) pairs for `rank` of `world`: the first
    n_pairs % world ranks take one pair more, so slice sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world or n_pairs < 0:
        raise ValueError(f"bad partition: n_pairs={n_pairs} world={world} rank={rank}")
    base, extra = divmod(n_pairs, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def slice_sizes(n_pairs: int, world: int) -> list:
    return [head_slice(n_pairs, world, r)[1] - head_slice(n_pairs, world, r)[0] for r in range(world)]


def attn_slice(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
               sm_scale: Optional[float] = None) -> torch.Tensor:
    """The forward on this rank's pairs: q, k, v are [pairs, N, D] (a slice of the
    flattened [B*H, N, D] problem); returns [pairs, N, D]. Runs entirely on this rank's
    GPU through the library's dense entry point."""
    from . import attn
    if q.dim() != 3:
        raise ValueError("attn_slice expects [pairs, N, D] tensors")
    if q.shape[0] == 0:
        return torch.empty_like(q)
    return attn(q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0), causal=causal, sm_scale=sm_scale)[0]


def gather_heads(out_r: torch.Tensor, n_pairs: int, group=None) -> torch.Tensor:
    """All-gather the ranks' output slices into [n_pairs, N, D] on every rank (slices
    padded to the largest one for the collective, padding dropped afterwards)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    sizes = slice_sizes(n_pairs, world)
    width = max(sizes)
    rest = tuple(out_r.shape[1:])
    pad = torch.zeros((width,) + rest, dtype=out_r.dtype, device=out_r.device)
    pad[: out_r.shape[0]] = out_r
    buf = torch.empty((world * width,) + rest, dtype=out_r.dtype, device=out_r.device)
    dist.all_gather_into_tensor(buf, pad, group=group)
    parts = [buf[r * width: r * width + sizes[r]] for r in range(world)]
    return torch.cat(parts, 0)
