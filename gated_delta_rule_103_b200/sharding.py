"""Splitting KDA work across ranks (one process per GPU).

Every (sequence, head) chain of the recurrence is independent of every other
one: the state is per sequence and per head ("深度解读报告" 2.3; zhaixingw.cn
ai-news/151: a fixed-size dk x dv state per request).  The operator therefore
shards with no collective on its data path: a rank owns a contiguous range of
heads (as tensor parallelism over heads would hand it) or a set of whole
sequences, and computes them alone.

One long sequence can also be split by tokens (sequence parallelism for the
long contexts of "深度解读报告" 4.5).  The recurrence is affine in the state,
so the tokens of one rank map its entry state S to M S + B, M the product of
the tokens' (I - beta k k^T) Diag(alpha) factors and B the exit state from
zero.  That gives one exchange step: every rank computes (M, B) of its range
(rank 0 runs its range outright from the true initial state), the pairs are
all-gathered (2 x 64 KiB per head and rank), each rank chains its entry state
S_r = M_{r-1} ( ... (M_1 B_0 + B_1) ... ) + B_{r-1} and runs its range from it.
"""
from __future__ import annotations

from typing import Callable, Dict, List, NamedTuple, Optional, Sequence, Tuple

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


def token_range(T: int, world: int, rank: int, chunk: int = 64) -> Tuple[int, int]:
    """Contiguous tokens [t0, t1) of rank `rank` when T tokens are split over
    `world` ranks in whole chunks, the first ranks taking one chunk more when
    the chunks do not divide evenly (the last rank takes the ragged tail)."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank / world")
    chunks = (T + chunk - 1) // chunk
    base, extra = divmod(chunks, world)
    c0 = rank * base + min(rank, extra)
    c1 = c0 + base + (1 if rank < extra else 0)
    return min(T, c0 * chunk), min(T, c1 * chunk)


class RangeOps(NamedTuple):
    """The compute steps of a sequence-parallel prefill: ``chunk_fwd(q, k, v,
    log_alpha, beta, initial_state) -> (out, final_state)``,
    ``chunk_transition(q, k, log_alpha, beta) -> M`` and ``state_affine(M, B,
    S) -> M S + B``."""
    chunk_fwd: Callable
    chunk_transition: Callable
    state_affine: Callable


def cuda_range_ops(scale: Optional[float] = None, **opts) -> RangeOps:
    """The library's kernels (``opts``: the chunk_fwd options l2norm_qk and
    raw_gate, passed to the transition too)."""
    from . import binding

    def fwd(q, k, v, g, b, s0):
        return binding.chunk_fwd(q, k, v, g, b, initial_state=s0, scale=scale, **opts)

    def trans(q, k, g, b):
        return binding.chunk_transition(q, k, g, b, **opts)

    return RangeOps(fwd, trans, binding.state_affine)


def range_maps(q, k, v, log_alpha, beta, initial_state, first: bool, ops: RangeOps):
    """The first step on one rank: the rank holding the sequences' first tokens
    runs them from the initial state (its map is the constant exit state:
    M = 0, B = S_end); every other rank returns its range's (M, B) and no
    output yet.  Returns (out or None, M, B) with M, B [N, H, dk, dv]."""
    if first:
        out, s_end = ops.chunk_fwd(q, k, v, log_alpha, beta, initial_state)
        return out, torch.zeros_like(s_end), s_end
    _, b = ops.chunk_fwd(q, k, v, log_alpha, beta, None)
    m = ops.chunk_transition(q, k, log_alpha, beta)
    return None, m, b


def entry_state(maps: Sequence[Tuple[torch.Tensor, torch.Tensor]], ops: RangeOps) -> torch.Tensor:
    """The entry state of the range after `maps` (the (M, B) of every earlier
    range, in token order): S = M_j S + B_j from S = 0 (the first map's M is 0,
    so S starts at its B, the first range's exit state)."""
    s = torch.zeros_like(maps[0][1])
    for m, b in maps:
        s = ops.state_affine(m, b, s)
    return s


def sequence_parallel_chunk_fwd(q, k, v, log_alpha, beta, initial_state, rank: int, world: int,
                                all_gather: Callable, ops: RangeOps):
    """Prefill of sequences whose tokens are split over `world` ranks in
    token order (see ``token_range``); q, k, v, log_alpha, beta hold this
    rank's range [B, t1 - t0, H, d], initial_state the sequences' initial
    state (used by rank 0).  ``all_gather(x)`` returns the list of every
    rank's x (torch.distributed.all_gather over the group).  Returns this
    rank's output rows and the exit state of its range (on the last rank, the
    sequences' final state)."""
    out, m, b = range_maps(q, k, v, log_alpha, beta, initial_state, rank == 0, ops)
    gathered = all_gather(torch.stack([m, b]))
    if rank == 0:
        return out, b
    s_in = entry_state([(x[0], x[1]) for x in gathered[:rank]], ops)
    return ops.chunk_fwd(q, k, v, log_alpha, beta, s_in)


def torch_all_gather(group=None) -> Callable:
    """all_gather over a torch.distributed group, as a function of one tensor."""
    import torch.distributed as dist

    def gather(x):
        xs = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
        dist.all_gather(xs, x.contiguous(), group=group)
        return xs

    return gather
