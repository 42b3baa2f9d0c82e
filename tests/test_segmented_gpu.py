"""Segmented (sequence-parallel) bf16 prefill against the fp64 oracle.

The recurrence is affine in the state, so a run of whole chunks maps its
entry state to S_out = M S_in + B (M: the segments' state transition, the
product of the tokens' (I - beta k k^T) Diag(alpha) factors; B: its exit
state from zero).  The segmented kernel cuts every sequence into G segments,
computes M and B of the middle segments alongside segment 0, chains the
entry states and reruns segments 1 .. G-1 from them; the results must equal
the token recurrence within the bf16 tolerance for every G, including
segments that are empty, packed sequences of mixed lengths and the fused
L2Norm.  The automatic choice segments only when the chains are very few.
"""
import contextlib

import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from gated_delta_rule_103_b200.configs import make_prefill
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def segmented(G, first_pass="auto"):
    binding.set_prefill_kernel("segmented", segments=G, first_pass=first_pass)
    try:
        yield
    finally:
        binding.set_prefill_kernel("auto")


def _run(x, l2norm_qk=False):
    d = to_cuda(x)
    out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                            initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                            scale=d["scale"], l2norm_qk=l2norm_qk)
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    return out, fs


def _oracle(x, l2norm_qk=False):
    return oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                              initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                              scale=x["scale"], l2norm_qk=l2norm_qk)


@pytest.mark.parametrize("first_pass", ["separate", "shared"])
@pytest.mark.parametrize("G", [2, 3, 4, 7])
@pytest.mark.parametrize("T", [1000, 130])
def test_segmented_matches_oracle(G, T, first_pass):
    # T = 130: 3 chunks, so G = 4 and 7 leave segments empty; "shared" runs a
    # segment's zero-start and transition runs in one cluster (G >= 3)
    x = inputs.prefill_inputs(2, T, 2, dtype=torch.bfloat16, seed=900 + G + T, init_std=0.1)
    with segmented(G, first_pass):
        assert binding.prefill_kernel_choice(2, T, 2, 2) == "segmented"
        assert binding.prefill_segments(2, T, 2, 2) == G
        out, fs = _run(x)
    o_ref, f_ref = _oracle(x)
    assert rel_fro(out, o_ref) < 2e-2, rel_fro(out, o_ref)
    assert rel_fro(fs, f_ref) < 2e-2, rel_fro(fs, f_ref)


@pytest.mark.parametrize("first_pass", ["separate", "shared"])
@pytest.mark.parametrize("G", [3, 5])
def test_segmented_varlen(G, first_pass):
    lengths = [1, 700, 0, 130, 64, 1500, 17]
    x = inputs.prefill_inputs(1, 0, 3, dtype=torch.bfloat16, seed=910 + G, init_std=0.1,
                              lengths=lengths)
    with segmented(G, first_pass):
        out, fs = _run(x)
    o_ref, f_ref = _oracle(x)
    assert rel_fro(out, o_ref) < 2e-2, rel_fro(out, o_ref)
    assert rel_fro(fs, f_ref) < 2e-2, rel_fro(fs, f_ref)
    assert torch.equal(fs[2].cpu(), x["initial_state"][2])   # the empty sequence


def test_segmented_without_states_and_strong_decay():
    """No initial state (zeros) and a gate at the precondition (chunk sums at
    -79..-70 in half of the channels)."""
    x = inputs.prefill_inputs(1, 900, 3, dtype=torch.bfloat16, seed=920)
    gen = torch.Generator().manual_seed(921)
    g = x["log_alpha"].clone()
    g[..., :64] = -(70.0 + 9.0 * torch.rand(g[..., :64].shape, generator=gen)) / 64.0
    x["log_alpha"] = g
    with segmented(4):
        out, fs = _run(x)
    o_ref, f_ref = _oracle(x)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2


def test_segmented_l2norm():
    x = inputs.prefill_inputs(2, 600, 2, dtype=torch.bfloat16, seed=930, init_std=0.1,
                              normalize_qk=False)
    with segmented(3):
        out, fs = _run(x, l2norm_qk=True)
    o_ref, f_ref = _oracle(x, l2norm_qk=True)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2


def test_automatic_choice():
    # 32 chains fill the SMs with one cluster each: not segmented
    assert binding.prefill_kernel_choice(1, 131072, 32, 1) == "cluster"
    assert binding.prefill_segments(1, 131072, 32, 1) == 1
    # 8 chains of 2048 chunks leave most SMs idle: segmented
    assert binding.prefill_kernel_choice(1, 131072, 8, 1) == "segmented"
    assert binding.prefill_segments(1, 131072, 8, 1) >= 3
    # many chains: one CTA each
    assert binding.prefill_kernel_choice(4, 4096, 32, 4) == "cta"


def test_few_chains_long_context_sampled_heads():
    """The few-chain long-context case the automatic choice segments (B=1,
    H=8, T=131072) in the benchmark's launch configuration; two heads
    recomputed by the oracle over every token, all values against the
    unsegmented cluster kernel."""
    x = make_prefill("long", device="cuda", H=8)
    assert binding.prefill_kernel_choice(1, x["T"], 8, 1) == "segmented"
    out, fs = _run(x)
    binding.set_prefill_kernel("cluster")
    try:
        out_c, fs_c = _run(x)
    finally:
        binding.set_prefill_kernel("auto")
    heads = [1, 6]
    y = dict(x)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        y[n] = x[n][:, :, heads].cpu().contiguous()
    y["initial_state"] = None
    o_ref, f_ref = _oracle(y)
    assert rel_fro(out[:, :, heads], o_ref) < 2e-2
    assert rel_fro(fs[:, heads], f_ref) < 2e-2
    assert rel_fro(out.float(), out_c.float()) < 1e-2
    assert rel_fro(fs, fs_c) < 1e-2


@pytest.mark.parametrize("case", ["deltanet", "gdn"])
def test_segmented_slow_decay(case):
    """No decay (DeltaNet) or one gate per token-head (Gated DeltaNet): the
    segments' transitions stay far from zero, so the entry states depend on
    them, not only on the zero-start exit states."""
    x = inputs.prefill_inputs(2, 1200, 2, dtype=torch.bfloat16, seed=940, init_std=0.1)
    if case == "deltanet":
        x["log_alpha"] = torch.zeros_like(x["log_alpha"])
    else:
        x["log_alpha"] = (x["log_alpha"][..., :1] * 0.1).expand_as(x["log_alpha"]).contiguous()
    for first_pass in ("separate", "shared"):
        with segmented(5, first_pass):
            out, fs = _run(x)
        o_ref, f_ref = _oracle(x)
        assert rel_fro(out, o_ref) < 2e-2, rel_fro(out, o_ref)
        assert rel_fro(fs, f_ref) < 2e-2, rel_fro(fs, f_ref)


def test_one_million_tokens():
    """The pages' longest context: one sequence of 2^20 tokens with 2 heads,
    run as the automatic choice runs it (segmented), every token and the
    final state against the oracle."""
    x = make_prefill("long", device="cuda", H=2, T=1 << 20, seed=1007)
    assert binding.prefill_kernel_choice(1, x["T"], 2, 1) == "segmented"
    out, fs = _run(x)
    y = {n: (v.cpu() if isinstance(v, torch.Tensor) else v) for n, v in x.items()}
    o_ref, f_ref = _oracle(y)
    assert rel_fro(out, o_ref) < 2e-2, rel_fro(out, o_ref)
    assert rel_fro(fs, f_ref) < 2e-2, rel_fro(fs, f_ref)
    assert torch.isfinite(out).all()
