"""Chunked prefill (kda_chunk_fwd) against the fp64 oracle.

Small cases span several 64-token chunks and a ragged tail; the named
workloads run at full size in the benchmark's launch configuration and are
compared in full (fp32 and short) or on sampled heads (long and varlen).
The bf16 cases run on both prefill kernels: one CTA per (sequence, head)
chain ("cta") and one thread-block cluster per chain ("cluster").
"""
import contextlib

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

# (dtype, bf16 prefill kernel); the fp32 path has a single kernel
CASES = [(torch.float32, "auto"), (torch.bfloat16, "cta"), (torch.bfloat16, "cluster")]
CASE_IDS = ["f32", "bf16-cta", "bf16-cluster"]


@contextlib.contextmanager
def prefill_kernel(kind):
    kda.binding.set_prefill_kernel(kind)
    try:
        yield
    finally:
        kda.binding.set_prefill_kernel("auto")


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


@pytest.mark.parametrize("dtype,kernel", CASES, ids=CASE_IDS)
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 512])
def test_prefill_small(T, dtype, kernel):
    x = inputs.prefill_inputs(2, T, 2, dtype=dtype, seed=T, init_std=0.1)
    with prefill_kernel(kernel):
        out, fs = run_gpu(x)
    o_ref, f_ref = run_oracle(x)
    assert rel_fro(out, o_ref) < TOL[dtype]
    assert rel_fro(fs, f_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype,kernel", CASES, ids=CASE_IDS)
def test_prefill_varlen_small(dtype, kernel):
    lengths = [1, 63, 0, 130, 64, 17]
    x = inputs.prefill_inputs(1, 0, 3, dtype=dtype, seed=77, init_std=0.1, lengths=lengths)
    with prefill_kernel(kernel):
        out, fs = run_gpu(x)
    o_ref, f_ref = run_oracle(x)
    assert rel_fro(out, o_ref) < TOL[dtype]
    assert rel_fro(fs, f_ref) < TOL[dtype]
    # the zero-length sequence passes its state through untouched
    assert torch.equal(fs[2].cpu(), x["initial_state"][2])


@pytest.mark.parametrize("dtype,kernel", CASES, ids=CASE_IDS)
def test_prefill_state_in_place(dtype, kernel):
    """final_state may be the initial_state buffer."""
    x = inputs.prefill_inputs(1, 150, 2, dtype=dtype, seed=3, init_std=0.1)
    d = to_cuda(x)
    s = d["initial_state"].clone()
    with prefill_kernel(kernel):
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=s, final_state=s, scale=x["scale"])
        torch.cuda.synchronize()
    o_ref, f_ref = run_oracle(x)
    assert fs.data_ptr() == s.data_ptr()
    assert rel_fro(s, f_ref) < TOL[dtype]
    assert rel_fro(out, o_ref) < TOL[dtype]


@pytest.mark.parametrize("dtype,kernel", CASES, ids=CASE_IDS)
def test_prefill_then_decode_equals_longer_prefill(dtype, kernel):
    """prefill(T) followed by one decode step on token T+1 == prefill(T+1)."""
    x = inputs.prefill_inputs(2, 97, 2, dtype=dtype, seed=11, init_std=0.1)
    d = to_cuda(x)
    T = 96
    with prefill_kernel(kernel):
        s, o_step, o_full, s_full = _prefill_then_decode(d, x, T)
    assert rel_fro(o_step, o_full[:, T]) < TOL[dtype]
    assert rel_fro(s, s_full) < TOL[dtype]


def _prefill_then_decode(d, x, T):
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
    return s, o_step, o_full, s_full


def test_config_pr1_full():
    x = make_prefill("pr1")
    out, fs = run_gpu(x)
    o_ref, f_ref = run_oracle(x)
    assert out.dtype == torch.float32
    assert rel_fro(out, o_ref) < 1e-4
    assert rel_fro(fs, f_ref) < 1e-4


@pytest.mark.parametrize("kernel", ["auto", "cluster"])
def test_config_short_full(kernel):
    x = make_prefill("short")
    with prefill_kernel(kernel):
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


@pytest.mark.parametrize("name,kernel", [("long", "cta"), ("varlen", "cluster")])
def test_config_full_size_other_kernel(name, kernel):
    """The full-size long and varlen workloads on the kernel that the
    automatic choice does not pick for them, sampled heads against the oracle
    and every value against the automatic choice."""
    x = make_prefill(name, device="cuda")
    out_a, fs_a = run_gpu(x)
    with prefill_kernel(kernel):
        out, fs = run_gpu(x)
    heads = [5, 17]
    y = _sampled_heads(x, heads)
    o_ref, f_ref = run_oracle(y)
    assert rel_fro(out[:, :, heads], o_ref) < 2e-2
    assert rel_fro(fs[:, heads], f_ref) < 2e-2
    # the two kernels round their bf16 operand tiles from gate sums taken in
    # different orders, so each carries its own few-1e-3 bf16 rounding noise
    # (the same size as its distance to the oracle), not a shared one
    assert rel_fro(out.float(), out_a.float()) < 1e-2
    assert rel_fro(fs, fs_a) < 1e-2
    assert kda.binding.device_error() == kda.binding.KDA_OK


def test_prefill_kernel_choice_rejects_unknown():
    with pytest.raises(ValueError):
        kda.binding.set_prefill_kernel("warp")


# ---------------------------------------------------------------- fused L2Norm of q, k
@pytest.mark.parametrize("dtype,kernel", CASES, ids=CASE_IDS)
@pytest.mark.parametrize("T", [65, 200])
def test_prefill_l2norm_qk(T, dtype, kernel):
    """Un-normalised q, k (Gaussian rows times per-row factors in [0.1, 10))
    with KDA_FLAG_L2NORM_QK against the oracle normalising in fp64."""
    x = inputs.prefill_inputs(2, T, 2, dtype=dtype, seed=300 + T, init_std=0.1,
                              normalize_qk=False)
    d = to_cuda(x)
    with prefill_kernel(kernel):
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=d["initial_state"], scale=x["scale"],
                                l2norm_qk=True)
        torch.cuda.synchronize()
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], scale=x["scale"],
                                      l2norm_qk=True)
    assert rel_fro(out, o_ref) < TOL[dtype]
    assert rel_fro(fs, f_ref) < TOL[dtype]


@pytest.mark.parametrize("kernel", ["cta", "cluster"])
def test_prefill_l2norm_qk_varlen(kernel):
    lengths = [1, 63, 0, 130, 64, 17]
    x = inputs.prefill_inputs(1, 0, 3, dtype=torch.bfloat16, seed=78, init_std=0.1,
                              lengths=lengths, normalize_qk=False)
    d = to_cuda(x)
    with prefill_kernel(kernel):
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                                scale=x["scale"], l2norm_qk=True)
        torch.cuda.synchronize()
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                                      scale=x["scale"], l2norm_qk=True)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2


def test_config_long_l2norm_qk_sampled_heads():
    """The long workload with un-normalised q, k and the fused L2Norm, in the
    benchmark's launch configuration; two heads recomputed by the oracle."""
    x = make_prefill("long", device="cuda", normalize_qk=False)
    out, fs = kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                            initial_state=x["initial_state"], scale=x["scale"], l2norm_qk=True)
    torch.cuda.synchronize()
    heads = [3, 28]
    y = _sampled_heads(x, heads)
    o_ref, f_ref = oracle.kda_forward(y["q"], y["k"], y["v"], y["log_alpha"], y["beta"],
                                      initial_state=y["initial_state"], scale=y["scale"],
                                      l2norm_qk=True)
    assert rel_fro(out[:, :, heads], o_ref) < 2e-2
    assert rel_fro(fs[:, heads], f_ref) < 2e-2
    assert kda.binding.device_error() == kda.binding.KDA_OK


# ---------------------------------------------------------------- output RMSNorm + gate
@pytest.mark.parametrize("dtype,kernel", CASES, ids=CASE_IDS)
def test_prefill_out_norm_gate(dtype, kernel):
    """KDA_FLAG_OUT_NORM_GATE: head-wise RMSNorm and sigmoid gate of every
    output row, against the oracle's fp64 epilogue; final_state unaffected."""
    x = inputs.prefill_inputs(2, 130, 3, dtype=dtype, seed=401, init_std=0.1)
    gate, weight = inputs.out_gate_inputs((2, 130, 3, 128), dtype, seed=401)
    d = to_cuda(x)
    with prefill_kernel(kernel):
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=d["initial_state"], scale=x["scale"],
                                out_gate=gate.cuda(), out_weight=weight.cuda(), out_eps=1e-6)
        torch.cuda.synchronize()
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], scale=x["scale"],
                                      out_gate=gate, out_weight=weight, out_eps=1e-6)
    assert rel_fro(out, o_ref) < TOL[dtype]
    assert rel_fro(fs, f_ref) < TOL[dtype]


def test_prefill_out_norm_gate_varlen_with_l2norm():
    """Both options together on packed sequences."""
    lengths = [1, 63, 0, 130, 64, 17]
    x = inputs.prefill_inputs(1, 0, 3, dtype=torch.bfloat16, seed=402, init_std=0.1,
                              lengths=lengths, normalize_qk=False)
    gate, weight = inputs.out_gate_inputs(tuple(x["v"].shape), torch.bfloat16, seed=402)
    d = to_cuda(x)
    out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                            initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                            scale=x["scale"], l2norm_qk=True, out_gate=gate.cuda(),
                            out_weight=weight.cuda())
    torch.cuda.synchronize()
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                                      scale=x["scale"], l2norm_qk=True, out_gate=gate,
                                      out_weight=weight)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2
