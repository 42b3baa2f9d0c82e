"""Seeded synthetic inputs for the KDA operator.

This module only draws random tensors; it holds none of the operator's
arithmetic, so both the CUDA library's tests and the CPU oracle can be fed
from it.  The recipe (shapes and distributions) follows the workloads on the
Kimi Linear pages: head dimension dk = dv = 128 ("深度解读报告", section 3.2),
q and k L2-normalised per head before the operator (same section), a
per-channel gate alpha in (0, 1] given as log_alpha = -exp(u) with u uniform,
and beta = sigmoid(N(0, 1)) per token and head.

Draw order for one call (one torch.Generator seeded once):
q, k, v, beta, log_alpha, initial state.  Varlen lengths come from their own
generator (seed + 7919) so that T is known before the tensors are drawn.

On a CUDA device the same recipe runs on a CUDA generator; it is seeded and
reproducible but draws different numbers than the CPU generator.
"""
from __future__ import annotations

from typing import Optional, Sequence

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def l2_normalise(x: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    """x / max(||x||_2, eps) over the last dimension (the layer's L2Norm of q
    and k, applied here as input preparation, before the dtype cast)."""
    return x / x.norm(dim=-1, keepdim=True).clamp_min(eps)


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> list:
    """n sequence lengths drawn uniformly from the integers [lo, hi]."""
    g = _gen(seed + 7919, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def cu_seqlens_from_lengths(lengths: Sequence[int]) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def prefill_inputs(B: int, T: int, H: int, dk: int = 128, dv: int = 128, *,
                   dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                   u_lo: float = -5.0, u_hi: float = -1.0,
                   init_std: Optional[float] = None,
                   lengths: Optional[Sequence[int]] = None,
                   normalize_qk: bool = True,
                   device="cpu") -> dict:
    """Inputs for ``kda_chunk_fwd``.

    Without ``lengths``: B sequences of T tokens.  With ``lengths``: B must be
    1, T is ignored and the sequences are packed back to back (cu_seqlens).
    ``init_std``: None for a zero initial state (no tensor), else the standard
    deviation of a Gaussian fp32 initial state per (sequence, head).
    ``normalize_qk``: False leaves q and k un-normalised (Gaussian rows times
    a per-row factor drawn from [0.1, 10), for the operator's fused L2Norm).
    Returns a dict with q, k, v (``dtype``), log_alpha and beta (fp32),
    initial_state (fp32 or None), cu_seqlens (int32 or None), scale and the
    sizes B, T, H, dk, dv, N.
    """
    if lengths is not None:
        if B != 1:
            raise ValueError("packed sequences need B == 1")
        cu = cu_seqlens_from_lengths(lengths)
        T = int(cu[-1])
        N = len(lengths)
    else:
        cu = None
        N = B
    g = _gen(seed, device)
    f32 = torch.float32
    q = torch.randn(B, T, H, dk, generator=g, device=device, dtype=f32)
    k = torch.randn(B, T, H, dk, generator=g, device=device, dtype=f32)
    v = torch.randn(B, T, H, dv, generator=g, device=device, dtype=f32)
    beta = torch.sigmoid(torch.randn(B, T, H, generator=g, device=device, dtype=f32))
    u = torch.rand(B, T, H, dk, generator=g, device=device, dtype=f32) * (u_hi - u_lo) + u_lo
    log_alpha = -torch.exp(u)
    s0 = None
    if init_std is not None:
        s0 = init_std * torch.randn(N, H, dk, dv, generator=g, device=device, dtype=f32)
    if normalize_qk:
        q, k = l2_normalise(q), l2_normalise(k)
    else:
        q = q * _row_factors(g, (B, T, H, 1), device)
        k = k * _row_factors(g, (B, T, H, 1), device)
    return dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), log_alpha=log_alpha,
                beta=beta, initial_state=s0,
                cu_seqlens=None if cu is None else cu.to(device),
                scale=dk ** -0.5, B=B, T=T, H=H, dk=dk, dv=dv, N=N)


def _row_factors(g, shape, device) -> torch.Tensor:
    """Positive per-row factors in [0.1, 10), log-uniform."""
    u = torch.rand(*shape, generator=g, device=device, dtype=torch.float32)
    return torch.exp((u * 2.0 - 1.0) * 2.302585092994046)


def out_gate_inputs(shape, dtype: torch.dtype = torch.bfloat16, *, seed: int = 0,
                    device="cpu") -> tuple:
    """Gate pre-activations (standard normal, shaped like the output) and a
    per-channel weight (1 + 0.1 N(0,1), fp32, the last dimension) for the
    output RMSNorm and sigmoid gate."""
    g = _gen(int(seed) + 104729, device)
    gate = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    weight = 1.0 + 0.1 * torch.randn(shape[-1], generator=g, device=device, dtype=torch.float32)
    return gate.to(dtype), weight


def backward_adjoints(out_shape, N: int, H: int, dk: int = 128, dv: int = 128, *,
                      dtype: torch.dtype = torch.bfloat16, seed: int = 0,
                      final_std: Optional[float] = 0.1, device="cpu") -> tuple:
    """Adjoints for the backward pass: d_out (standard normal, shaped like the
    output, ``dtype``) and d_final_state (Gaussian fp32 [N,H,dk,dv] with
    standard deviation ``final_std``, or None when it is None)."""
    g = _gen(int(seed) + 130363, device)
    d_out = torch.randn(*out_shape, generator=g, device=device, dtype=torch.float32).to(dtype)
    dfs = None
    if final_std is not None:
        dfs = final_std * torch.randn(N, H, dk, dv, generator=g, device=device, dtype=torch.float32)
    return d_out, dfs


def decode_state(N: int, H: int, dk: int = 128, dv: int = 128, *, seed: int = 0,
                 std: float = 0.1, device="cpu") -> torch.Tensor:
    """fp32 per-(request, head) state, Gaussian with standard deviation std."""
    g = _gen(seed, device)
    return std * torch.randn(N, H, dk, dv, generator=g, device=device, dtype=torch.float32)


def decode_inputs(N: int, H: int, dk: int = 128, dv: int = 128, *,
                  dtype: torch.dtype = torch.bfloat16, seed: int = 0, step: int = 0,
                  u_lo: float = -5.0, u_hi: float = -1.0, normalize_qk: bool = True,
                  device="cpu") -> dict:
    """One decode token per (request, head) for step ``step``; the step's
    generator is seeded with seed * 10**4 + step.  ``normalize_qk`` as for
    prefill_inputs."""
    g = _gen(int(seed) * 10 ** 4 + int(step), device)
    f32 = torch.float32
    q = torch.randn(N, H, dk, generator=g, device=device, dtype=f32)
    k = torch.randn(N, H, dk, generator=g, device=device, dtype=f32)
    v = torch.randn(N, H, dv, generator=g, device=device, dtype=f32)
    beta = torch.sigmoid(torch.randn(N, H, generator=g, device=device, dtype=f32))
    u = torch.rand(N, H, dk, generator=g, device=device, dtype=f32) * (u_hi - u_lo) + u_lo
    if normalize_qk:
        q, k = l2_normalise(q), l2_normalise(k)
    else:
        q = q * _row_factors(g, (N, H, 1), device)
        k = k * _row_factors(g, (N, H, 1), device)
    return dict(q=q.to(dtype), k=k.to(dtype), v=v.to(dtype), log_alpha=-torch.exp(u),
                beta=beta, scale=dk ** -0.5, N=N, H=H, dk=dk, dv=dv)
