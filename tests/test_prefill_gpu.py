"""Chunked prefill (kda_chunk_fwd) against the fp64 oracle.

Small cases span several 64-token chunks and a ragged tail; the named
workloads run at full size in the benchmark's launch configuration and are
compared in full (fp32 and short) or on sampled heads (long and varlen).
"""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import inputs
from gated_delta_rule_103_b200.configs import WORKLOADS, make_prefill
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def run_gpu(x, **kw):
    d = to_cuda(x)
    out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                            initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                            scale=d["scale"], **kw)
    torch.cuda.synchronize()
    return out, fs


def run_oracle(x):
    return oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                              initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                              scale=x["scale"])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 512])
def test_prefill_small(T, dtype):
    x = inputs.prefill_inputs(2, T, 2, dtype=dtype, seed=T, init_std=0.1)
    out, fs = run_gpu(x)
    o_ref, f_ref = run_oracle(x)
    assert rel_fro(out, o_ref) < TOL[dtype]
    assert rel_fro(fs, f_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_prefill_varlen_small(dtype):
    lengths = [1, 63, 0, 130, 64, 17]
    x = inputs.prefill_inputs(1, 0, 3, dtype=dtype, seed=77, init_std=0.1, lengths=lengths)
    out, fs = run_gpu(x)
    o_ref, f_ref = run_oracle(x)
    assert rel_fro(out, o_ref) < TOL[dtype]
    assert rel_fro(fs, f_ref) < TOL[dtype]
    # the zero-length sequence passes its state through untouched
    assert torch.equal(fs[2].cpu(), x["initial_state"][2])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_prefill_state_in_place(dtype):
    """final_state may be the initial_state buffer."""
    x = inputs.prefill_inputs(1, 150, 2, dtype=dtype, seed=3, init_std=0.1)
    d = to_cuda(x)
    s = d["initial_state"].clone()
    out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                            initial_state=s, final_state=s, scale=x["scale"])
    torch.cuda.synchronize()
    o_ref, f_ref = run_oracle(x)
    assert fs.data_ptr() == s.data_ptr()
    assert rel_fro(s, f_ref) < TOL[dtype]
    assert rel_fro(out, o_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_prefill_then_decode_equals_longer_prefill(dtype):
    """prefill(T) followed by one decode step on token T+1 == prefill(T+1)."""
    x = inputs.prefill_inputs(2, 97, 2, dtype=dtype, seed=11, init_std=0.1)
    d = to_cuda(x)
    T = 96
    _, s = kda.chunk_fwd(d["q"][:, :T].contiguous(), d["k"][:, :T].contiguous(),
                         d["v"][:, :T].contiguous(), d["log_alpha"][:, :T].contiguous(),
                         d["beta"][:, :T].contiguous(), initial_state=d["initial_state"],
                         scale=x["scale"])
    o_step = kda.recurrent_step(d["q"][:, T].contiguous(), d["k"][:, T].contiguous(),
                                d["v"][:, T].contiguous(), d["log_alpha"][:, T].contiguous(),
                                d["beta"][:, T].contiguous(), s, scale=x["scale"])
    o_full, s_full = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                   initial_state=d["initial_state"], scale=x["scale"])
    torch.cuda.synchronize()
    assert rel_fro(o_step, o_full[:, T]) < TOL[dtype]
    assert rel_fro(s, s_full) < TOL[dtype]


def test_config_pr1_full():
    x = make_prefill("pr1")
    out, fs = run_gpu(x)
    o_ref, f_ref = run_oracle(x)
    assert out.dtype == torch.float32
    assert rel_fro(out, o_ref) < 1e-4
    assert rel_fro(fs, f_ref) < 1e-4


def test_config_short_full():
    x = make_prefill("short")
    out, fs = run_gpu(x)
    o_ref, f_ref = run_oracle(x)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2


def _sampled_heads(x, heads):
    y = dict(x)
    for n in ("q", "k", "v", "log_alpha", "beta"):
        y[n] = x[n][:, :, heads].cpu().contiguous()
    if x["initial_state"] is not None:
        y["initial_state"] = x["initial_state"][:, heads].cpu().contiguous()
    if x["cu_seqlens"] is not None:
        y["cu_seqlens"] = x["cu_seqlens"].cpu()
    return y


@pytest.mark.parametrize("name", ["long", "varlen"])
def test_config_full_size_sampled_heads(name):
    """Full-size long (128k) and varlen workloads on the device; the oracle
    recomputes two of the 32 heads over every token."""
    x = make_prefill(name, device="cuda")
    out, fs = run_gpu(x)
    heads = [0, 31]
    y = _sampled_heads(x, heads)
    o_ref, f_ref = run_oracle(y)
    assert rel_fro(out[:, :, heads], o_ref) < 2e-2
    assert rel_fro(fs[:, heads], f_ref) < 2e-2
    assert torch.isfinite(out).all() and torch.isfinite(fs).all()
    assert kda.binding.device_error() == kda.binding.KDA_OK
