"""Decode step (kda_recurrent_step) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import inputs
from gated_delta_rule_103_b200.configs import WORKLOADS
from helpers import rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,H", [(1, 1), (3, 2), (256, 32)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_steps_small(N, H, dtype):
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    state = inputs.decode_state(N, H, seed=5, std=0.1).cuda()
    ref_state = state.cpu().double().numpy()
    steps = 3 if N * H > 1000 else 12
    for s in range(steps):
        x = inputs.decode_inputs(N, H, dtype=dtype, seed=5, step=s)
        out = kda.recurrent_step(*(x[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")),
                                 state, scale=x["scale"])
        o_ref, ref_state = oracle.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"],
                                                  x["beta"], ref_state, scale=x["scale"])
        assert rel_fro(out, o_ref) < tol, f"step {s} out"
        assert rel_fro(state, ref_state) < tol, f"step {s} state"
    if dtype == torch.float32:
        assert rel_fro(state, ref_state) < 1e-5


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_l2norm_qk(dtype):
    """Un-normalised q, k with KDA_FLAG_L2NORM_QK against the oracle
    normalising in fp64, over several steps."""
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    N, H = 5, 3
    state = inputs.decode_state(N, H, seed=8, std=0.1).cuda()
    ref_state = state.cpu().double().numpy()
    for s in range(6):
        x = inputs.decode_inputs(N, H, dtype=dtype, seed=8, step=s, normalize_qk=False)
        out = kda.recurrent_step(*(x[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")),
                                 state, scale=x["scale"], l2norm_qk=True)
        o_ref, ref_state = oracle.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"],
                                                  x["beta"], ref_state, scale=x["scale"],
                                                  l2norm_qk=True)
        assert rel_fro(out, o_ref) < tol, f"step {s} out"
        assert rel_fro(state, ref_state) < tol, f"step {s} state"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_out_norm_gate(dtype):
    """KDA_FLAG_OUT_NORM_GATE fused into the decode step, against the
    oracle's fp64 epilogue; the state update is unaffected."""
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    N, H = 6, 4
    state = inputs.decode_state(N, H, seed=9, std=0.1).cuda()
    ref_state = state.cpu().double().numpy()
    for s in range(4):
        x = inputs.decode_inputs(N, H, dtype=dtype, seed=9, step=s)
        gate, weight = inputs.out_gate_inputs((N, H, 128), dtype, seed=9 + s)
        out = kda.recurrent_step(*(x[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")),
                                 state, scale=x["scale"], out_gate=gate.cuda(),
                                 out_weight=weight.cuda())
        o_ref, ref_state = oracle.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"],
                                                  x["beta"], ref_state, scale=x["scale"],
                                                  out_gate=gate, out_weight=weight)
        assert rel_fro(out, o_ref) < tol, f"step {s} out"
        assert rel_fro(state, ref_state) < tol, f"step {s} state"


def test_decode_config_1000_steps_sampled():
    """The batched-decode workload (256 requests x 32 heads, 1000 consecutive
    steps, state updated in place) in the launch configuration the benchmark
    times; the oracle follows 4 of the 256 requests (all 32 heads)."""
    w = WORKLOADS["decode"]
    N, H, steps = w["N"], w["H"], w["steps"]
    lo, hi = w["u_range"]
    dev = torch.device("cuda")
    state = inputs.decode_state(N, H, seed=w["seed"], std=w["state_std"], device=dev)
    sample = [0, 97, 200, 255]
    ref_state = state[sample].cpu().double().numpy()
    checks = {1, 10, 100, steps}
    for s in range(1, steps + 1):
        x = inputs.decode_inputs(N, H, dtype=w["dtype"], seed=w["seed"], step=s,
                                 u_lo=lo, u_hi=hi, device=dev)
        out = kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], state,
                                 scale=x["scale"])
        xs = {n: x[n][sample].cpu() for n in ("q", "k", "v", "log_alpha", "beta")}
        o_ref, ref_state = oracle.kda_decode_step(xs["q"], xs["k"], xs["v"], xs["log_alpha"],
                                                  xs["beta"], ref_state, scale=x["scale"])
        if s in checks:
            assert rel_fro(out[sample], o_ref) < w["tol"], f"out at step {s}"
    assert rel_fro(state[sample], ref_state) < w["tol"]
    assert torch.isfinite(state).all()
    assert kda.binding.device_error() == kda.binding.KDA_OK
