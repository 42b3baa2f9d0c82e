"""The failure path of the kernels' bounded waits, on a GPU, without a fault.

kda_selftest_wait_timeout runs the tensor-core kernels' wait routine on an
mbarrier that nothing arrives on, with a short limit: the wait must run out,
be reported once by kda_device_error as KDA_ERR_TIMEOUT, and leave the
context usable for the next prefill.
"""
import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_is_reported_once():
    assert binding.device_error() == binding.KDA_OK
    binding.selftest_wait_timeout(20000)      # 20 ms
    assert binding.device_error() == binding.KDA_ERR_TIMEOUT
    assert binding.device_error() == binding.KDA_OK


@pytest.mark.parametrize("kernel", ["cta", "cluster"])
def test_context_usable_after_a_run_out_wait(kernel):
    binding.selftest_wait_timeout(5000)
    assert binding.device_error() == binding.KDA_ERR_TIMEOUT
    x = inputs.prefill_inputs(1, 300, 2, dtype=torch.bfloat16, seed=21, init_std=0.1)
    d = to_cuda(x)
    binding.set_prefill_kernel(kernel)
    try:
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=d["initial_state"], scale=x["scale"])
        torch.cuda.synchronize()
    finally:
        binding.set_prefill_kernel("auto")
    assert binding.device_error() == binding.KDA_OK
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], scale=x["scale"])
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2
