"""Splitting KDA work across ranks (one process per GPU).

Every (sequence, head) chain of the recurrence is independent of every other
one: the state is per sequence and per head ("深度解读报告" 2.3; zhaixingw.cn
ai-news/151: a fixed-size dk x dv state per request).  The operator therefore
shards with no collective on its data path: a rank owns a contiguous range of
heads (as tensor parallelism over heads would hand it) or a set of whole
sequences, and computes them alone.  The only cross-rank step in this package
is timing: the slowest rank's time.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import torch


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous heads [h0, h1) of rank `rank` out of `world`; the first
    H % world ranks get one extra head."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank / world")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def balance_sequences(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Assigns whole sequences to ranks so that the per-rank token counts are
    balanced: longest first, each to the rank with the fewest tokens so far.
    Returns, per rank, the sorted indices of its sequences."""
    if world <= 0:
        raise ValueError("world must be positive")
    load = [0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i)):
        r = min(range(world), key=lambda r: (load[r], r))
        out[r].append(i)
        load[r] += int(lengths[i])
    return [sorted(x) for x in out]


def slice_heads(x: Dict, h0: int, h1: int) -> Dict:
    """The inputs of heads [h0, h1) of a prefill input dict (layouts
    [B,T,H,d], [B,T,H] and [N,H,dk,dv]), made contiguous."""
    y = dict(x)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        y[n] = x[n][:, :, h0:h1].contiguous()
    if x.get("initial_state") is not None:
        y["initial_state"] = x["initial_state"][:, h0:h1].contiguous()
    y["H"] = h1 - h0
    return y


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks of the default process group
    (the value itself when torch.distributed is not initialised)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
