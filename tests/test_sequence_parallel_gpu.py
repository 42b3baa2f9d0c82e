"""kda_chunk_transition and kda_state_affine, and a sequence split by tokens.

The recurrence is affine in the state: a run of tokens maps its entry state
S to M S + B.  kda_chunk_transition returns M (the chunked recurrence from the
identity with v = 0), kda_state_affine applies it in fp32.  Checked against
the oracle (M: the oracle run from the identity with v = 0) and against
kda_chunk_fwd itself; then the ranks of a sequence-parallel prefill are
emulated one after another in this process (their exchange is a list), and
the assembled outputs must equal one prefill over all tokens.
"""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs, sharding
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu


def _oracle_transition(x, cu=None):
    B, T, H, dk = x["k"].shape
    N = B if cu is None else len(cu) - 1
    eye = np.broadcast_to(np.eye(dk), (N, H, dk, dk)).copy()
    _, m = oracle.kda_forward(x["q"], x["k"], np.zeros((B, T, H, dk)), x["log_alpha"], x["beta"],
                              initial_state=eye, cu_seqlens=cu, scale=x["scale"])
    return m


@pytest.mark.parametrize("T", [1, 200, 1000])
def test_transition_matches_oracle_and_forward(T):
    x = inputs.prefill_inputs(2, T, 3, dtype=torch.bfloat16, seed=960 + T, init_std=0.1,
                              u_lo=-7.0, u_hi=-4.0)
    d = to_cuda(x)
    m = kda.chunk_transition(d["q"], d["k"], d["log_alpha"], d["beta"])
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    assert rel_fro(m, _oracle_transition(x)) < 2e-2
    # M S0 + (final state from zeros) = final state from S0
    _, f0 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], scale=x["scale"])
    _, f1 = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                          initial_state=d["initial_state"], scale=x["scale"])
    s = kda.state_affine(m, f0, d["initial_state"])
    torch.cuda.synchronize()
    assert rel_fro(s, f1) < 2e-2


def test_transition_varlen_and_empty():
    lengths = [0, 1, 130, 64, 500]
    x = inputs.prefill_inputs(1, 0, 2, dtype=torch.bfloat16, seed=970, lengths=lengths,
                              u_lo=-7.0, u_hi=-4.0)
    d = to_cuda(x)
    m = kda.chunk_transition(d["q"], d["k"], d["log_alpha"], d["beta"], cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    ref = _oracle_transition(x, cu=x["cu_seqlens"].numpy())
    assert rel_fro(m, ref) < 2e-2
    # an empty sequence's transition is the identity
    assert torch.equal(m[0].cpu(), torch.eye(128).expand(2, 128, 128))


def test_state_affine_exact():
    g = torch.Generator().manual_seed(971)
    M = torch.randn(3, 2, 128, 128, generator=g)
    B = torch.randn(3, 2, 128, 128, generator=g)
    S = torch.randn(3, 2, 128, 128, generator=g)
    ref = (M.double() @ S.double() + B.double())
    out = kda.state_affine(M.cuda(), B.cuda(), S.cuda())
    Bd = B.cuda()
    kda.state_affine(M.cuda(), Bd, S.cuda(), out=Bd)       # in place over B
    torch.cuda.synchronize()
    assert rel_fro(out, ref) < 1e-6
    assert torch.equal(Bd, out)


@pytest.mark.parametrize("world", [2, 3, 5])
def test_sequence_parallel_emulated_ranks(world):
    """The ranks of a sequence-parallel prefill run one after another here,
    the exchange a list: outputs and final state equal the oracle over all
    tokens (bf16 tolerance) and the unsplit kda_chunk_fwd."""
    x = inputs.prefill_inputs(1, 2000, 4, dtype=torch.bfloat16, seed=980 + world, init_std=0.1,
                              u_lo=-7.0, u_hi=-4.0)
    d = to_cuda(x)
    ops = sharding.cuda_range_ops(scale=x["scale"])
    ranges = [sharding.token_range(x["T"], world, r) for r in range(world)]
    sl = [{n: d[n][:, a:b].contiguous() for n in ("q", "k", "v", "log_alpha", "beta")}
          for a, b in ranges]
    first = [sharding.range_maps(s["q"], s["k"], s["v"], s["log_alpha"], s["beta"],
                                 d["initial_state"], r == 0, ops) for r, s in enumerate(sl)]
    gathered = [torch.stack([m, b]) for _, m, b in first]
    outs, fs = [first[0][0]], first[0][2]
    for r in range(1, world):
        s_in = sharding.entry_state([(g[0], g[1]) for g in gathered[:r]], ops)
        o, fs = ops.chunk_fwd(sl[r]["q"], sl[r]["k"], sl[r]["v"], sl[r]["log_alpha"],
                              sl[r]["beta"], s_in)
        outs.append(o)
    out = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], scale=x["scale"])
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2
    o_all, f_all = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                 initial_state=d["initial_state"], scale=x["scale"])
    torch.cuda.synchronize()
    assert rel_fro(out.float(), o_all.float()) < 1e-2
    assert rel_fro(fs, f_all) < 1e-2
    assert binding.device_error() == binding.KDA_OK
