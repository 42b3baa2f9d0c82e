"""The method's special cases on every CUDA kernel, against the fp64 oracle.

The pages place DeltaNet (no decay), pure multiplicative decay (no delta
rule) and Gated DeltaNet (one scalar gate per head) in the same family as
KDA ("深度解读报告" 2.2-2.3; zhaixingw.cn ai-news/151, the Gated DeltaNet
formula).  Each is a choice of inputs here:

  deltanet     log_alpha = 0 (alpha = 1: nothing decays)
  pure_decay   beta = 0 with a non-zero initial state: the state only decays,
               S_t = Diag(exp G_t) S_0, o_t = scale S_t^T q_t (closed form
               checked as well)
  recall       beta = 1 and q = k: the written value is read back exactly,
               o_t = scale v_t for a unit key (checked as well)
  gdn          a gate that is constant over the channels of each token-head
  strong_decay the gate at the documented precondition: in half of the
               channels every 64-token chunk sums to between -79 and -70
               (the other half keeps the workload's gate), with a ragged
               last chunk, so e^{-G} reaches about 2e34 inside a chunk
  large        |v| about 100 and an initial state of standard deviation 10

Kernels: the fp32 FFMA prefill, both bf16 tensor-core prefills (one CTA or
one cluster per chain), the fused-L2Norm variants, the decode step and the
backward pass.  Tolerances are the operator's: 1e-4 relative Frobenius error
for fp32, 2e-2 for bf16 inputs with fp32 state; the backward's 1e-4.
"""
import contextlib

import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from helpers import rel_fro, to_cuda

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}
CASES = ["deltanet", "pure_decay", "recall", "gdn", "strong_decay", "large"]
KERNELS = [(torch.float32, "auto"), (torch.bfloat16, "cta"), (torch.bfloat16, "cluster")]
KERNEL_IDS = ["f32", "bf16-cta", "bf16-cluster"]


@contextlib.contextmanager
def prefill_kernel(kind):
    binding.set_prefill_kernel(kind)
    try:
        yield
    finally:
        binding.set_prefill_kernel("auto")


def _strong_gate(g: torch.Tensor, seed: int) -> torch.Tensor:
    """Channels 0-63: every run of 64 consecutive tokens sums to between -79
    and -70 (each token draws from [-79/64, -70/64]); channels 64-127 keep g."""
    gen = torch.Generator().manual_seed(seed + 991)
    u = torch.rand(g.shape[:-1] + (64,), generator=gen, dtype=torch.float32)
    out = g.clone()
    out[..., :64] = -(70.0 + 9.0 * u) / 64.0
    return out


def special(case: str, B: int, T: int, H: int, dtype, seed: int, lengths=None,
            normalize_qk: bool = True) -> dict:
    """Inputs of one special case, drawn with the workload recipe and then
    specialised (the specialisations only set or copy input values)."""
    init_std = 10.0 if case == "large" else 0.1
    x = inputs.prefill_inputs(B, T, H, dtype=dtype, seed=seed, init_std=init_std,
                              lengths=lengths, normalize_qk=normalize_qk)
    if case == "deltanet":
        x["log_alpha"] = torch.zeros_like(x["log_alpha"])
    elif case == "pure_decay":
        x["beta"] = torch.zeros_like(x["beta"])
    elif case == "recall":
        x["beta"] = torch.ones_like(x["beta"])
        x["q"] = x["k"].clone()
    elif case == "gdn":
        x["log_alpha"] = x["log_alpha"][..., :1].expand_as(x["log_alpha"]).contiguous()
    elif case == "strong_decay":
        x["log_alpha"] = _strong_gate(x["log_alpha"], seed)
    elif case == "large":
        x["v"] = (x["v"].float() * 100.0).to(dtype)
    else:
        raise ValueError(case)
    return x


def run_prefill(x, l2norm_qk=False):
    d = to_cuda(x)
    out, fs = kda.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                            initial_state=d["initial_state"], cu_seqlens=d["cu_seqlens"],
                            scale=d["scale"], l2norm_qk=l2norm_qk)
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    return out, fs


def run_oracle(x, l2norm_qk=False):
    return oracle.kda_forward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                              initial_state=x["initial_state"], cu_seqlens=x["cu_seqlens"],
                              scale=x["scale"], l2norm_qk=l2norm_qk)


def _f64(t):
    return t.detach().cpu().double().numpy()


def _closed_forms(case, x, out, fs):
    """The results the special case fixes without the oracle."""
    if case == "pure_decay":
        # S_t = Diag(exp G_t) S_0 per sequence; o_t = scale S_t^T q_t
        g, q, s0 = _f64(x["log_alpha"]), _f64(x["q"]), _f64(x["initial_state"])
        B, T, H, dk = q.shape
        o = np.zeros((B, T, H, s0.shape[-1]))
        fsr = np.zeros_like(s0)
        for b in range(B):
            G = np.cumsum(g[b], axis=0)                              # [T, H, dk]
            st = np.exp(G)[..., None] * s0[b][None]                   # [T, H, dk, dv]
            o[b] = x["scale"] * np.einsum("thkv,thk->thv", st, q[b])
            fsr[b] = st[-1]
        tol = 1e-4 if x["q"].dtype == torch.float32 else 2e-2
        assert rel_fro(out, o) < tol
        assert rel_fro(fs, fsr) < tol
    elif case == "recall":
        # a unit key written with beta = 1 is read back exactly: o_t = scale v_t
        k = _f64(x["k"])
        norm_dev = np.abs(np.linalg.norm(k, axis=-1) - 1.0).max()
        bound = 1e-4 if x["q"].dtype == torch.float32 else 2e-2
        assert norm_dev < bound / 4
        assert rel_fro(out, x["scale"] * _f64(x["v"])) < bound


@pytest.mark.parametrize("dtype,kernel", KERNELS, ids=KERNEL_IDS)
@pytest.mark.parametrize("case", CASES)
def test_prefill_special_case(case, dtype, kernel):
    x = special(case, 2, 200, 2, dtype, seed=700 + CASES.index(case))
    with prefill_kernel(kernel):
        out, fs = run_prefill(x)
    o_ref, f_ref = run_oracle(x)
    assert torch.isfinite(out).all() and torch.isfinite(fs).all()
    print(f"prefill {case} {kernel} {dtype} out {rel_fro(out, o_ref):.2e} "
          f"state {rel_fro(fs, f_ref):.2e}")
    assert rel_fro(out, o_ref) < TOL[dtype], rel_fro(out, o_ref)
    assert rel_fro(fs, f_ref) < TOL[dtype], rel_fro(fs, f_ref)
    _closed_forms(case, x, out, fs)


@pytest.mark.parametrize("dtype,kernel", KERNELS, ids=KERNEL_IDS)
@pytest.mark.parametrize("case", ["strong_decay", "large", "recall"])
def test_prefill_special_case_varlen(case, dtype, kernel):
    """Packed sequences (a zero-length, a one-token and ragged sequences):
    the chunks restart at every sequence start, so the gate's chunk sums
    stay at the precondition in every sequence."""
    x = special(case, 1, 0, 3, dtype, seed=720 + CASES.index(case),
                lengths=[1, 63, 0, 130, 64, 17, 200])
    with prefill_kernel(kernel):
        out, fs = run_prefill(x)
    o_ref, f_ref = run_oracle(x)
    assert rel_fro(out, o_ref) < TOL[dtype], rel_fro(out, o_ref)
    assert rel_fro(fs, f_ref) < TOL[dtype], rel_fro(fs, f_ref)


@pytest.mark.parametrize("kernel", ["cta", "cluster"])
@pytest.mark.parametrize("case", ["recall", "strong_decay", "large"])
def test_prefill_special_case_l2norm(case, kernel):
    """The fused L2Norm variant of both bf16 kernels on un-normalised q, k."""
    x = special(case, 2, 200, 2, torch.bfloat16, seed=740 + CASES.index(case),
                normalize_qk=False)
    with prefill_kernel(kernel):
        out, fs = run_prefill(x, l2norm_qk=True)
    o_ref, f_ref = run_oracle(x, l2norm_qk=True)
    assert rel_fro(out, o_ref) < 2e-2, rel_fro(out, o_ref)
    assert rel_fro(fs, f_ref) < 2e-2, rel_fro(fs, f_ref)
    if case == "recall":
        # normalised inside the kernel in fp32: o = scale v to bf16 rounding
        assert rel_fro(out, x["scale"] * _f64(x["v"])) < 2e-2


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("case", CASES)
def test_decode_special_case(case, dtype):
    """Eight consecutive decode steps, state in place, each token specialised
    like the prefill inputs (strong_decay: every token's gate in channels
    0-63 is in [-79/64, -70/64])."""
    N, H, steps = 3, 2, 8
    tol = TOL[dtype]
    std = 10.0 if case == "large" else 0.1
    state = inputs.decode_state(N, H, seed=760, std=std).cuda()
    ref_state = _f64(state)
    for s in range(steps):
        x = inputs.decode_inputs(N, H, dtype=dtype, seed=761 + CASES.index(case), step=s)
        if case == "deltanet":
            x["log_alpha"] = torch.zeros_like(x["log_alpha"])
        elif case == "pure_decay":
            x["beta"] = torch.zeros_like(x["beta"])
        elif case == "recall":
            x["beta"] = torch.ones_like(x["beta"])
            x["q"] = x["k"].clone()
        elif case == "gdn":
            x["log_alpha"] = x["log_alpha"][..., :1].expand_as(x["log_alpha"]).contiguous()
        elif case == "strong_decay":
            x["log_alpha"] = _strong_gate(x["log_alpha"], 762 + s)
        elif case == "large":
            x["v"] = (x["v"].float() * 100.0).to(dtype)
        out = kda.recurrent_step(*(x[n].cuda() for n in ("q", "k", "v", "log_alpha", "beta")),
                                 state, scale=x["scale"])
        o_ref, ref_state = oracle.kda_decode_step(x["q"], x["k"], x["v"], x["log_alpha"],
                                                  x["beta"], ref_state, scale=x["scale"])
        assert rel_fro(out, o_ref) < tol, f"step {s} out"
        assert rel_fro(state, ref_state) < tol, f"step {s} state"
        if s == steps - 1:
            print(f"decode {case} {dtype} out {rel_fro(out, o_ref):.2e} "
                  f"state {rel_fro(state, ref_state):.2e}")
        if case == "recall":
            assert rel_fro(out, x["scale"] * _f64(x["v"])) < (1e-4 if dtype == torch.float32 else 2e-2)
    assert binding.device_error() == binding.KDA_OK


NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "d_initial_state")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("case", CASES)
def test_backward_special_case(case, dtype):
    """kda_chunk_bwd on each special case (two sequences of 200 tokens, an
    initial state and a final-state adjoint), every gradient against the
    fp64 adjoint."""
    x = special(case, 2, 200, 2, dtype, seed=780 + CASES.index(case))
    d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), x["N"], x["H"], dtype=dtype,
                                          seed=781)
    d = to_cuda(x)
    got = kda.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d_out.cuda(),
                        initial_state=d["initial_state"], d_final_state=dfs.cuda(),
                        scale=d["scale"])
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK
    ref = oracle.kda_backward(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_out,
                              initial_state=x["initial_state"], d_final_state=dfs,
                              scale=x["scale"])
    for name, g, r in zip(NAMES, got, ref):
        assert torch.isfinite(g).all(), name
        if case == "recall" and name == "d_initial_state":
            # A unit key written with beta = 1 is read back exactly, so every
            # path from S_0 to an output cancels: the true gradient is the
            # rounding residual of ||k|| = 1 (about 1e-7 of the adjoints in
            # fp32, 1e-3 in bf16) and a relative error of it measures only
            # that cancellation.  Compared normwise instead, against the
            # adjoints that flow into it.
            scale_in = (np.linalg.norm(_f64(dfs).ravel())
                        + x["scale"] * np.linalg.norm(_f64(d_out).ravel()))
            err = float(np.linalg.norm((_f64(g) - r).ravel()) / scale_in)
        else:
            err = rel_fro(g, r)
        print(f"backward {case} {dtype} {name} {err:.2e}")
        assert err < 1e-4, f"{name}: {err:.3e}"
