"""Caller-owned workspace of kda_chunk_fwd and kda_chunk_bwd.

The caller owns every buffer, workspace included: the size queries are pure
functions of the sizes, a call with too small, misaligned or overlapping
workspace is rejected before anything is enqueued, results do not depend on
the workspace's previous contents, and calls with every buffer passed in
leave the device's free memory unchanged (the library allocates nothing).
"""
import ctypes

import pytest
import torch

import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, inputs
from helpers import to_cuda

pytestmark = pytest.mark.gpu


def test_forward_workspace_query():
    # few chains: the cluster kernel's ring; many chains or fp32: none
    assert binding.chunk_fwd_workspace_bytes(1, 4096, 32, 1) > 0
    assert binding.chunk_fwd_workspace_bytes(1, 4096, 32, 1, torch.float32) == 0
    assert binding.chunk_fwd_workspace_bytes(4, 4096, 32, 4) == 0
    assert binding.chunk_fwd_workspace_bytes(1, 0, 32, 1) == 0
    binding.set_prefill_kernel("cta")
    try:
        assert binding.chunk_fwd_workspace_bytes(1, 4096, 32, 1) == 0
    finally:
        binding.set_prefill_kernel("auto")
    # 133,120 bytes per preparing CTA and chain
    assert binding.chunk_fwd_workspace_bytes(1, 4096, 32, 1) % (32 * 133120) == 0


def test_backward_workspace_query():
    # 2 x 64 KiB per chunk slot and head, 512 B per token and head (each part
    # rounded up to 256 bytes)
    assert binding.chunk_bwd_workspace_bytes(2, 128, 3, 2, False) == 2 * 4 * 3 * 65536 + 2 * 128 * 3 * 512
    assert binding.chunk_bwd_workspace_bytes(1, 130, 1, 3, True) == 2 * (3 + 3) * 65536 + 130 * 512
    assert binding.chunk_bwd_workspace_bytes(1, 4, 0, 1, False) == 0


def _fwd_raw(lib, d, out, fs, ws, wsb):
    p = ctypes.c_void_p
    return lib.kda_chunk_fwd(p(d["q"].data_ptr()), p(d["k"].data_ptr()), p(d["v"].data_ptr()),
                             p(d["log_alpha"].data_ptr()), p(d["beta"].data_ptr()),
                             p(d["initial_state"].data_ptr()), None, ctypes.c_float(d["scale"]), 64,
                             p(out.data_ptr()), p(fs.data_ptr()), d["B"], d["T"], d["H"], 128, 128,
                             d["N"], binding.KDA_DTYPE_BF16, ws, wsb, None)


def test_forward_rejects_bad_workspace():
    lib = binding.load_library()
    x = to_cuda(inputs.prefill_inputs(1, 300, 2, dtype=torch.bfloat16, seed=810, init_std=0.1))
    need = binding.chunk_fwd_workspace_bytes(1, 300, 2, 1)
    assert need > 0
    out = torch.empty_like(x["v"])
    fs = torch.empty(1, 2, 128, 128, device="cuda")
    ws = torch.empty(need + 1024, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p
    assert _fwd_raw(lib, x, out, fs, None, 0) == binding.KDA_ERR_INVALID_ARG
    assert _fwd_raw(lib, x, out, fs, p(ws.data_ptr()), need - 1) == binding.KDA_ERR_INVALID_ARG
    assert _fwd_raw(lib, x, out, fs, p(ws.data_ptr() + 16), need) == binding.KDA_ERR_INVALID_ARG
    host = torch.empty(need, dtype=torch.uint8)
    assert _fwd_raw(lib, x, out, fs, p(host.data_ptr()), need) == binding.KDA_ERR_INVALID_ARG
    # a workspace overlapping an input (the initial state's buffer)
    big = torch.empty(need + (1 << 20), dtype=torch.uint8, device="cuda")
    s0 = big[:2 * 65536].view(torch.float32).view(1, 2, 128, 128)
    s0.copy_(x["initial_state"])
    y = dict(x, initial_state=s0)
    assert _fwd_raw(lib, y, out, fs, p(big.data_ptr()), need) == binding.KDA_ERR_INVALID_ARG
    assert _fwd_raw(lib, x, out, fs, p(ws.data_ptr()), need) == binding.KDA_OK
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK


def test_results_do_not_depend_on_workspace_contents():
    x = to_cuda(inputs.prefill_inputs(2, 700, 3, dtype=torch.bfloat16, seed=811, init_std=0.1))
    need = binding.chunk_fwd_workspace_bytes(2, 700, 3, 2)
    assert need > 0
    res = []
    for fill in (0, 255, 7):
        ws = torch.full((need,), fill, dtype=torch.uint8, device="cuda")
        res.append(kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                                 initial_state=x["initial_state"], scale=x["scale"], workspace=ws))
    torch.cuda.synchronize()
    for o, f in res[1:]:
        assert torch.equal(o, res[0][0]) and torch.equal(f, res[0][1])


def test_calls_allocate_nothing():
    """kda_chunk_fwd (cluster kernel, with its ring in the workspace) and
    kda_chunk_bwd with every buffer passed in: free device memory unchanged."""
    x = to_cuda(inputs.prefill_inputs(1, 1000, 4, dtype=torch.bfloat16, seed=812, init_std=0.1))
    d_out, dfs = inputs.backward_adjoints(tuple(x["v"].shape), 1, 4, seed=813, device="cuda")
    out = torch.empty_like(x["v"])
    fs = torch.empty(1, 4, 128, 128, device="cuda")
    wf = torch.empty(binding.chunk_fwd_workspace_bytes(1, 1000, 4, 1), dtype=torch.uint8,
                     device="cuda")
    wb = torch.empty(binding.chunk_bwd_workspace_bytes(1, 1000, 4, 1, False), dtype=torch.uint8,
                     device="cuda")
    assert wf.numel() > 0 and wb.numel() > 0
    f32 = dict(dtype=torch.float32, device="cuda")
    grads = (torch.empty(1, 1000, 4, 128, **f32), torch.empty(1, 1000, 4, 128, **f32),
             torch.empty(1, 1000, 4, 128, **f32), torch.empty(1, 1000, 4, 128, **f32),
             torch.empty(1, 1000, 4, **f32), torch.empty(1, 4, 128, 128, **f32))

    def step():
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"],
                      initial_state=x["initial_state"], scale=x["scale"], out=out,
                      final_state=fs, workspace=wf)
        kda.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], d_out,
                      initial_state=x["initial_state"], d_final_state=dfs, scale=x["scale"],
                      workspace=wb, grads=grads)

    step()                      # first use loads the kernels
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert binding.device_error() == binding.KDA_OK
