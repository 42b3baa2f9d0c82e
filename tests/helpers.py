"""Shared helpers for the GPU parity tests (not collected as tests)."""
import numpy as np
import torch


def rel_fro(x, ref) -> float:
    """||x - ref||_F / ||ref||_F, computed in fp64."""
    x = np.asarray(x.detach().cpu().double().numpy() if isinstance(x, torch.Tensor) else x,
                   dtype=np.float64)
    ref = np.asarray(ref.detach().cpu().double().numpy() if isinstance(ref, torch.Tensor) else ref,
                     dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


def to_cuda(d: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
