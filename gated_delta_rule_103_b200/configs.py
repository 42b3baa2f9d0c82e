"""The named KDA workloads (sizes, dtypes and input recipe).

All use head dimension dk = dv = 128 and chunk length 64.  ``u_range`` is the
interval of u in log_alpha = -exp(u).
"""
from __future__ import annotations

import torch

from . import inputs as _inputs

WORKLOADS = {
    # fp32 reference case: B=1, H=2, T=512, zero initial state.
    "pr1": dict(kind="prefill", B=1, T=512, H=2, dtype=torch.float32, seed=1001,
                u_range=(-5.0, -1.0), init_std=None, tol=1e-4),
    # short prefill: B=4, H=32, T=4096, bf16 q/k/v, N(0, 0.1) initial state.
    "short": dict(kind="prefill", B=4, T=4096, H=32, dtype=torch.bfloat16, seed=1002,
                  u_range=(-5.0, -1.0), init_std=0.1, tol=2e-2),
    # long prefill: B=1, H=32, T=131072 (128k), longer memory, zero initial state.
    "long": dict(kind="prefill", B=1, T=131072, H=32, dtype=torch.bfloat16, seed=1003,
                 u_range=(-7.0, -2.0), init_std=None, tol=2e-2),
    # varlen: 16 sequences, lengths uniform in [1024, 32768], packed, H=32.
    "varlen": dict(kind="prefill", B=1, T=None, H=32, dtype=torch.bfloat16, seed=1004,
                   u_range=(-5.0, -1.0), init_std=None, n_seqs=16,
                   len_range=(1024, 32768), tol=2e-2),
    # batched decode: 256 requests x 32 heads, one token each, 1000 steps.
    "decode": dict(kind="decode", N=256, H=32, dtype=torch.bfloat16, seed=1005,
                   u_range=(-5.0, -1.0), state_std=0.1, steps=1000, tol=2e-2),
}

DK = DV = 128
CHUNK = 64


def make_prefill(name: str, device="cpu", **override) -> dict:
    """Draw the inputs of a named prefill workload (``override`` replaces any
    size or recipe field, e.g. a smaller T for a quick case)."""
    w = dict(WORKLOADS[name])
    w.update(override)
    lengths = None
    B, T = w["B"], w["T"]
    if w.get("n_seqs"):
        lo, hi = w["len_range"]
        lengths = w.get("lengths") or _inputs.varlen_lengths(w["n_seqs"], lo, hi, w["seed"])
    return _inputs.prefill_inputs(B, T or 0, w["H"], DK, DV, dtype=w["dtype"], seed=w["seed"],
                                  u_lo=w["u_range"][0], u_hi=w["u_range"][1],
                                  init_std=w["init_std"], lengths=lengths,
                                  normalize_qk=w.get("normalize_qk", True), device=device)
