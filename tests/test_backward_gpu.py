"""kda_chunk_bwd against the fp64 oracle adjoint (oracle.kda_backward).

The backward pass runs in fp32 from the exact input values (bf16 inputs are
upcast, as the oracle upcasts the same values), so every gradient agrees
with the fp64 adjoint to within fp32 rounding accumulated over the chunk
algebra: the bound is 1e-4 relative Frobenius error per gradient, for fp32
and bf16 inputs alike.  Cases span several chunks with a ragged tail,
packed sequences with a zero-length and a one-token sequence, the optional
initial state and final-state adjoint, and, at the short-prefill size
(B=4, H=32, T=4096), one sampled (sequence, head) chain compared whole.
"""
import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu

TOL = 1e-4
NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_initial_state")

CASES = [
    # (B, T, H, dtype, lengths, init_std, final_std)
    (2, 200, 2, torch.float32, None, 0.1, 0.1),
    (1, 0, 3, torch.bfloat16, [130, 1, 0, 64, 257], 0.1, 0.1),
    (3, 64, 1, torch.bfloat16, None, None, None),
    (1, 1, 2, torch.float32, None, 0.1, None),
]


def _run(x, d_out, dfs, need_ds0=True):
    d = to_cuda(x)
    grads = kda.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d_out.cuda(),
                          initial_state=d["initial_state"],
                          d_final_state=None if dfs is None else dfs.cuda(),
                          cu_seqlens=d["cu_seqlens"], scale=d["scale"],
                          need_initial_state_grad=need_ds0)
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    return grads


@pytest.mark.parametrize("B,T,H,dtype,lengths,init_std,final_std", CASES)
def test_backward_matches_oracle(B, T, H, dtype, lengths, init_std, final_std):
    x = inputs.prefill_inputs(B, T, H, dtype=dtype, seed=51 + B + T, init_std=init_std,
                              lengths=lengths)
    d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), x["N"], H, dtype=dtype,
                                          seed=52 + T, final_std=final_std)
    got = _run(x, d_out, dfs)
    ref = oracle.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_out,
                              initial_state=x["initial_state"], d_final_state=dfs,
                              cu_seqlens=x["cu_seqlens"], scale=x["scale"])
    for name, g, r in zip(NAMES, got, ref):
        assert g.shape == r.shape, name
        assert torch.isfinite(g).all(), name
        err = rel_fro(g, r)
        assert err < TOL, f"{name}: {err:.3e}"


def test_backward_without_initial_state_grad():
    x = inputs.prefill_inputs(1, 150, 2, dtype=torch.bfloat16, seed=61, init_std=0.1)
    d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), 1, 2, seed=62)
    a = _run(x, d_out, dfs, need_ds0=True)
    b = _run(x, d_out, dfs, need_ds0=False)
    assert b[5] is None
    for ga, gb in zip(a[:5], b[:5]):
        assert torch.equal(ga, gb)


def test_backward_short_prefill_sampled_chain():
    # the short-prefill configuration, one (sequence, head) chain against the
    # oracle on that chain alone (chains are independent)
    x = inputs.prefill_inputs(4, 4096, 32, dtype=torch.bfloat16, seed=1002, init_std=0.1)
    d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), 4, 32, seed=63)
    got = _run(x, d_out, dfs)
    n, h = 2, 17
    sl = (slice(n, n + 1), slice(None), slice(h, h + 1))
    ref = oracle.kda_backward(x["q"][sl], x["k"][sl], x["v"][sl], x["log_alpha"][sl],
                              x["beta"][sl], d_out[sl],
                              initial_state=x["initial_state"][n:n + 1, h:h + 1],
                              d_final_state=dfs[n:n + 1, h:h + 1], scale=x["scale"])
    picks = [g[sl] for g in got[:4]] + [got[4][n:n + 1, :, h:h + 1], got[5][n:n + 1, h:h + 1]]
    for name, g, r in zip(NAMES, picks, ref):
        err = rel_fro(g, r)
        assert err < TOL, f"{name}: {err:.3e}"


def test_backward_rejects_bad_arguments():
    x = to_cuda(inputs.prefill_inputs(1, 64, 1, dtype=torch.bfloat16, seed=64))
    d_out = torch.zeros_like(x["v"])
    lib = binding.load_library()
    # dk other than 128
    st = lib.kda_chunk_bwd(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                           x["log_alpha"].data_ptr(), x["beta"].data_ptr(), None, None,
                           d_out.data_ptr(), None, 0.1, 64,
                           None, None, None, None, None, None, 1, 64, 1, 64, 128, 1,
                           binding.KDA_DTYPE_BF16, None, 0, None)
    assert st == binding.KDA_ERR_UNSUPPORTED
    # an output aliasing an input
    g = torch.empty(1, 64, 1, 128, dtype=torch.float32, device="cuda")
    gb = torch.empty(1, 64, 1, dtype=torch.float32, device="cuda")
    st = lib.kda_chunk_bwd(x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
                           x["log_alpha"].data_ptr(), x["beta"].data_ptr(), None, None,
                           d_out.data_ptr(), None, 0.1, 64,
                           g.data_ptr(), g.data_ptr(), x["log_alpha"].data_ptr(), g.data_ptr(),
                           gb.data_ptr(), None, 1, 64, 1, 128, 128, 1,
                           binding.KDA_DTYPE_BF16, None, 0, None)
    assert st == binding.KDA_ERR_INVALID_ARG
