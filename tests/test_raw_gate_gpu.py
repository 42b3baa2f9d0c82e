"""KDA_FLAG_RAW_GATE on every kernel, against the fp64 oracle.

The kernels take the gate's pre-activations z and use log alpha =
log sigmoid(z) (the reading of "深度解读报告" 3.2 recorded with the oracle's
``log_sigmoid``).  Two recipes: z = logit(alpha) of the workload's gate (the
same decays as the plain tests), and z ~ N(1, 1.5^2) as a projection's output
would be.  The fp32 path is held to 1e-4, the bf16 paths to 2e-2.
"""
import contextlib

import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
KERNELS = [(torch.float32, "auto"), (torch.bfloat16, "cta"), (torch.bfloat16, "cluster"),
           (torch.bfloat16, "segmented")]
KERNEL_IDS = ["f32", "bf16-cta", "bf16-cluster", "bf16-segmented"]


@contextlib.contextmanager
def prefill_kernel(kind):
    binding.set_prefill_kernel(kind, segments=3 if kind == "segmented" else 0)
    try:
        yield
    finally:
        binding.set_prefill_kernel("auto")


def _raw(x, recipe, seed):
    g = x["log_alpha"]
    if recipe == "logit":
        # z = log(alpha / (1 - alpha)) of the recipe's gate
        z = g - torch.log(-torch.expm1(g))
    else:
        gen = torch.Generator().manual_seed(seed)
        z = 1.0 + 1.5 * torch.randn(g.shape, generator=gen)
    return dict(x, log_alpha=z.contiguous())


@pytest.mark.parametrize("dtype,kernel", KERNELS, ids=KERNEL_IDS)
@pytest.mark.parametrize("recipe", ["logit", "normal"])
def test_prefill_raw_gate(recipe, dtype, kernel):
    x = _raw(inputs.prefill_inputs(2, 300, 2, dtype=dtype, seed=950, init_std=0.1), recipe, 951)
    d = to_cuda(x)
    with prefill_kernel(kernel):
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=d["initial_state"], scale=x["scale"], raw_gate=True)
        torch.cuda.synchronize()
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], scale=x["scale"],
                                      raw_gate=True)
    assert rel_fro(out, o_ref) < TOL[dtype], rel_fro(out, o_ref)
    assert rel_fro(fs, f_ref) < TOL[dtype], rel_fro(fs, f_ref)
    assert binding.device_error() == binding.KDA_OK


@pytest.mark.parametrize("kernel", ["cta", "cluster"])
def test_prefill_raw_gate_varlen_with_l2norm(kernel):
    """Packed sequences with ragged last chunks (the padded rows must keep no
    decay) and both input options together."""
    lengths = [1, 63, 0, 130, 64, 17]
    x = inputs.prefill_inputs(1, 0, 3, dtype=torch.bfloat16, seed=952, init_std=0.1,
                              lengths=lengths, normalize_qk=False)
    x = _raw(x, "normal", 953)
    d = to_cuda(x)
    with prefill_kernel(kernel):
        out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                                scale=x["scale"], l2norm_qk=True, raw_gate=True)
        torch.cuda.synchronize()
    o_ref, f_ref = oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                      initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                                      scale=x["scale"], l2norm_qk=True, raw_gate=True)
    assert rel_fro(out, o_ref) < 2e-2
    assert rel_fro(fs, f_ref) < 2e-2


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_raw_gate(dtype):
    N, H = 4, 3
    state = inputs.decode_state(N, H, seed=954, std=0.1).cuda()
    ref_state = state.cpu().double().numpy()
    for s in range(6):
        x = inputs.decode_inputs(N, H, dtype=dtype, seed=955, step=s)
        x = _raw(x, "normal", 956 + s)
        out = kda.recurrent_step(*(x[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")),
                                 state, scale=x["scale"], raw_gate=True)
        o_ref, ref_state = oracle.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"],
                                                  x["beta"], ref_state, scale=x["scale"],
                                                  raw_gate=True)
        assert rel_fro(out, o_ref) < TOL[dtype], f"step {s} out"
        assert rel_fro(state, ref_state) < TOL[dtype], f"step {s} state"
