"""The output RMSNorm and sigmoid gate (KDA_FLAG_OUT_NORM_GATE) behind the
cluster and segmented prefills.

Checked against the oracle's fp64 epilogue on ragged chunks, packed
sequences, segmented runs and a longer sequence (no row past the sequence
written), and against the epilogue's formula applied to the plain output.
"""
import contextlib

import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def kernel(kind, **kw):
    binding.set_prefill_kernel(kind, **kw)
    try:
        yield
    finally:
        binding.set_prefill_kernel("auto")


def _fwd(d, gate=None, weight=None, eps=1e-6, l2norm_qk=False):
    kw = {} if gate is None else {"out_gate": gate.cuda(), "out_weight": weight.cuda(), "out_eps": eps}
    out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                            initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                            scale=d["scale"], l2norm_qk=l2norm_qk, **kw)
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    return out, fs


def _ref(x, gate, weight, eps=1e-6, l2norm_qk=False):
    return oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                              initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                              scale=x["scale"], l2norm_qk=l2norm_qk, out_gate=gate,
                              out_weight=weight, out_eps=eps)


def _separate_pass(o, gate, weight, eps):
    """The epilogue's formula on the plain bf16 output, in
    torch on the GPU for the comparison only: rows of dv, fp32."""
    x = o.float()
    inv = torch.rsqrt((x * x).mean(-1, keepdim=True) + eps)
    return (x * inv * weight.cuda() * torch.sigmoid(gate.cuda().float())).to(o.dtype)


@pytest.mark.parametrize("T", [64, 130, 1000])
def test_cluster_epilogue_ragged(T):
    x = inputs.prefill_inputs(2, T, 3, dtype=torch.bfloat16, seed=1100 + T, init_std=0.1)
    gate, weight = inputs.out_gate_inputs(tuple(x["v"].shape), torch.bfloat16, seed=1100 + T)
    d = to_cuda(x)
    with kernel("cluster"):
        assert binding.prefill_kernel_choice(x["B"], x["T"], x["H"], x["N"]) == "cluster"
        out, fs = _fwd(d, gate, weight)
        plain, fs0 = _fwd(d)
    o_ref, f_ref = _ref(x, gate, weight)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2
    assert torch.equal(fs, fs0)
    # against the epilogue's formula on the plain rows (torch's sigmoid and
    # rsqrt against the kernel's fast exponential and rsqrt)
    sep = _separate_pass(plain, gate, weight, 1e-6)
    assert rel_fro(out.float(), sep.float()) < 1e-2


def test_cluster_epilogue_varlen_l2norm():
    lengths = [1, 63, 0, 130, 64, 17, 300]
    x = inputs.prefill_inputs(1, 0, 2, dtype=torch.bfloat16, seed=1110, init_std=0.1,
                              lengths=lengths, normalize_qk=False)
    gate, weight = inputs.out_gate_inputs(tuple(x["v"].shape), torch.bfloat16, seed=1110)
    d = to_cuda(x)
    with kernel("cluster"):
        out, fs = _fwd(d, gate, weight, eps=1e-5, l2norm_qk=True)
    o_ref, f_ref = _ref(x, gate, weight, eps=1e-5, l2norm_qk=True)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2


@pytest.mark.parametrize("G", [2, 3])
def test_segmented_epilogue(G):
    x = inputs.prefill_inputs(1, 3000, 2, dtype=torch.bfloat16, seed=1120 + G, init_std=0.1,
                              u_lo=-7.0, u_hi=-4.0)
    gate, weight = inputs.out_gate_inputs(tuple(x["v"].shape), torch.bfloat16, seed=1120 + G)
    d = to_cuda(x)
    with kernel("segmented", segments=G):
        out, fs = _fwd(d, gate, weight)
    o_ref, f_ref = _ref(x, gate, weight)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2


def test_cluster_epilogue_long_sequence():
    """Two heads over 20k tokens (313 chunks, a ragged last one): every row
    normalised and gated, none past the sequence written."""
    x = inputs.prefill_inputs(1, 20000, 2, dtype=torch.bfloat16, seed=1130, init_std=0.1)
    gate, weight = inputs.out_gate_inputs(tuple(x["v"].shape), torch.bfloat16, seed=1130)
    d = to_cuda(x)
    out = torch.full((1, 20000 + 64, 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    fs = torch.empty(1, 2, 128, 128, device="cuda")
    with kernel("cluster"):
        kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                      initial_state=d["initial_state"], scale=d["scale"],
                      out=out[:, :20000], final_state=fs, out_gate=gate.cuda(),
                      out_weight=weight.cuda(), out_eps=1e-6)
        torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    o_ref, f_ref = _ref(x, gate, weight)
    assert rel_fro(out[:, :20000], o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2
    assert torch.all(out[:, 20000:] == 7.0)
