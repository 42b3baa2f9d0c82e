"""kda_chunk_fwd_noalloc against kda_chunk_fwd.

The no-allocation entry point runs the cluster prefill kernel with its
hand-off ring in the library's fixed device array.  Two calls in a row on
different inputs must each equal kda_chunk_fwd on the cluster kernel bit for
bit (the second call reuses the array the first one filled), stay within the
bf16 tolerance of the oracle, and leave the device's free memory unchanged.
This file is collected last; it passes on its own in a fresh process too.
"""
import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu


def _reference(d, kind):
    binding.set_prefill_kernel(kind)
    try:
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                                scale=d["scale"])
        torch.cuda.synchronize()
    finally:
        binding.set_prefill_kernel("auto")
    return out, fs


def _noalloc(d, out, fs):
    binding.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], out,
                              initial_state=d["initial_state"], final_state=fs,
                              cu_seqlens=d["cu_seqlens"], scale=d["scale"])


def _cases():
    # a batch with a ragged last chunk, then packed sequences of mixed lengths
    a = inputs.prefill_inputs(2, 1000, 4, dtype=torch.bfloat16, seed=41, init_std=0.1)
    b = inputs.prefill_inputs(1, 0, 8, dtype=torch.bfloat16, seed=42, init_std=0.1,
                              lengths=[700, 1, 0, 129, 64])
    return [a, b]


def test_two_calls_in_a_row_match_chunk_fwd():
    cases = _cases()
    devs = [to_cuda(x) for x in cases]
    outs = [torch.empty_like(d["v"]) for d in devs]
    fss = [torch.empty(x["N"], x["H"], 128, 128, dtype=torch.float32, device="cuda")
           for x in cases]
    for d, out, fs in zip(devs, outs, fss):
        _noalloc(d, out, fs)
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    for x, d, out, fs in zip(cases, devs, outs, fss):
        o_ref, f_ref = _reference(d, "cluster")
        assert torch.equal(out, o_ref)
        assert torch.equal(fs, f_ref)
        o64, f64 = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"],
                                      cu_seqlens=x["cu_seqlens"], scale=x["scale"])
        assert rel_fro(out, o64) < 2e-2
        assert rel_fro(fs, f64) < 2e-2


def test_calls_leave_free_memory_unchanged():
    d = to_cuda(_cases()[0])
    out = torch.empty_like(d["v"])
    fs = torch.empty(d["N"], d["H"], 128, 128, dtype=torch.float32, device="cuda")
    _noalloc(d, out, fs)          # first use loads the kernel's module
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        _noalloc(d, out, fs)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_rejects_more_chains_than_the_ring_holds():
    # 127 chains need more than the 16 MiB ring array
    x = inputs.prefill_inputs(1, 2, 127, dtype=torch.bfloat16, seed=5)
    d = to_cuda(x)
    out = torch.empty_like(d["v"])
    with pytest.raises(binding.KDAError) as e:
        _noalloc(d, out, None)
    assert e.value.status == binding.KDA_ERR_UNSUPPORTED
    # 126 chains fit
    x = inputs.prefill_inputs(1, 2, 126, dtype=torch.bfloat16, seed=5)
    d = to_cuda(x)
    out = torch.empty_like(d["v"])
    _noalloc(d, out, None)
    torch.cuda.synchronize()
    o_ref, _ = _reference(d, "cluster")
    assert torch.equal(out, o_ref)


def test_zero_tokens_pass_the_state_through():
    """T = 0 with an initial state, and packed sequences that are all empty:
    final_state equals initial_state and kda_chunk_fwd's result."""
    for x in (inputs.prefill_inputs(2, 0, 3, dtype=torch.bfloat16, seed=6, init_std=0.1),
              inputs.prefill_inputs(1, 0, 3, dtype=torch.bfloat16, seed=7, init_std=0.1,
                                    lengths=[0, 0, 0, 0])):
        d = to_cuda(x)
        out = torch.empty_like(d["v"])
        fs = torch.full((x["N"], x["H"], 128, 128), float("nan"), dtype=torch.float32,
                        device="cuda")
        _noalloc(d, out, fs)
        torch.cuda.synchronize()
        assert torch.equal(fs, d["initial_state"])
        _, f_ref = _reference(d, "auto")
        assert torch.equal(fs, f_ref)
