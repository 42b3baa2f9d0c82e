"""Stage-by-stage parity of the bf16 tensor-core prefill kernel.

kda_chunk_debug_stages runs the kernel on one chunk of one head and returns
its intermediate tiles; each is compared with the same intermediate of the
fp64 chunkwise restatement in the oracle package, computed from the same
(bf16-rounded) inputs.
"""
import numpy as np
import pytest
import torch

from oracle import chunked
from gated_delta_rule_103_b200 import binding, inputs
from helpers import rel_fro

pytestmark = pytest.mark.gpu


def prod_err(x, a, b):
    """||x - a b||_F / (||a||_F ||b||_F): the error of a product measured
    against the size of its (rounded) factors, meaningful even when the
    product itself nearly cancels."""
    ref = a @ b
    return float(np.linalg.norm((np.asarray(x) - ref).ravel())
                 / (np.linalg.norm(a.ravel()) * np.linalg.norm(b.ravel())))


@pytest.mark.parametrize("L", [64, 37, 1])
def test_chunk_stages(L):
    x = inputs.prefill_inputs(1, L, 1, dtype=torch.bfloat16, seed=100 + L, init_std=0.1)
    q, k, v = (x[n][0, :, 0] for n in ("q", "k", "v"))
    g, b = x["log_alpha"][0, :, 0], x["beta"][0, :, 0]
    s0 = x["initial_state"][0, 0]
    scale = x["scale"]
    dev = torch.device("cuda")
    out, fs, st = binding.chunk_debug_stages(q.to(dev), k.to(dev), v.to(dev), g.to(dev), b.to(dev),
                                             initial_state=s0.to(dev).contiguous(), scale=scale)
    r = chunked.chunk_step(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                           g.double().numpy(), b.double().numpy(), s0.double().numpy(), scale)
    st = {n: t.cpu().double().numpy() for n, t in st.items()}
    tol = 2e-2
    S0 = s0.double().numpy()
    # products of bf16-rounded factors: error against the factors' size
    assert prod_err(st["AP"][:L, :L], r["Kt"], r["Kh"].T) < tol
    assert prod_err(st["AP"][64:64 + L, :L], scale * r["Qt"], r["Kh"].T) < tol
    assert prod_err(st["O1T"][:, :L].T, scale * r["Qt"], S0) < tol
    assert prod_err(st["DT"].T, r["Kh"].T, r["U"]) < tol
    # the remaining stages and the results: relative Frobenius error
    assert rel_fro(st["T"][:L, :L], r["T"]) < tol
    assert rel_fro(st["WT"][:, :L], r["W"].T) < tol
    assert rel_fro(st["UpT"][:, :L], r["Up"].T) < tol
    assert rel_fro(st["UT"][:, :L], r["U"].T) < tol
    assert rel_fro(st["OT"][:, :L], r["O"].T) < tol
    assert rel_fro(st["ST"], r["S"].T) < tol
    assert rel_fro(out, r["O"]) < tol
    assert rel_fro(fs, r["S"]) < tol
