"""Host-side checks of the C ABI: the library builds, loads and exports every
symbol include/kda.h declares; size and dtype validation that happens before
any CUDA call; and (on a GPU) pointer validation and error statuses."""
import ctypes
import os
import re

import pytest
import torch

import gated_delta_rule_103_b200 as kda
from gated_delta_rule_103_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(kda_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) >= {"kda_chunk_fwd", "kda_recurrent_step", "kda_status_string"}
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    assert set(names) == set(binding.EXPORTED_SYMBOLS)


def test_status_strings_and_version(lib):
    for s in range(5):
        assert binding.status_string(s).startswith("KDA_")
    assert lib.kda_version() >= 10000


def _chunk_call(lib, **kw):
    a = dict(q=None, k=None, v=None, g=None, b=None, s0=None, cu=None, scale=0.1, chunk=64,
             out=None, fs=None, B=1, T=4, H=1, dk=128, dv=128, N=1, dt=1)
    a.update(kw)
    return lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["b"], a["s0"], a["cu"],
                             ctypes.c_float(a["scale"]), a["chunk"], a["out"], a["fs"],
                             a["B"], a["T"], a["H"], a["dk"], a["dv"], a["N"], a["dt"],
                             a.get("ws"), a.get("wsb", 0), None)


def test_size_validation_before_cuda(lib):
    """Unsupported sizes and inconsistent counts are rejected before any
    pointer is inspected (no CUDA call is made)."""
    assert _chunk_call(lib, chunk=32) == binding.KDA_ERR_UNSUPPORTED
    assert _chunk_call(lib, dk=64) == binding.KDA_ERR_UNSUPPORTED
    assert _chunk_call(lib, dv=256) == binding.KDA_ERR_UNSUPPORTED
    assert _chunk_call(lib, N=2) == binding.KDA_ERR_INVALID_ARG          # N != B
    assert _chunk_call(lib, H=0) == binding.KDA_ERR_INVALID_ARG
    assert _chunk_call(lib, T=-1) == binding.KDA_ERR_INVALID_ARG
    assert _chunk_call(lib, dt=7) == binding.KDA_ERR_INVALID_ARG
    assert _chunk_call(lib, scale=float("nan")) == binding.KDA_ERR_INVALID_ARG
    assert lib.kda_recurrent_step(None, None, None, None, None, None, None,
                                  1, 1, 64, 128, ctypes.c_float(1.0), 1, None) \
        == binding.KDA_ERR_UNSUPPORTED


def _bwd_call(lib, **kw):
    a = dict(scale=0.1, chunk=64, B=1, T=4, H=1, dk=128, dv=128, N=1, dt=1)
    a.update(kw)
    return lib.kda_chunk_bwd(None, None, None, None, None, None, None, None, None,
                             ctypes.c_float(a["scale"]), a["chunk"],
                             None, None, None, None, None, None,
                             a["B"], a["T"], a["H"], a["dk"], a["dv"], a["N"], a["dt"], None, 0,
                             None)


def test_backward_size_validation_before_cuda(lib):
    """kda_chunk_bwd rejects unsupported sizes and inconsistent counts
    before inspecting a pointer, and null pointers afterwards."""
    assert _bwd_call(lib, chunk=32) == binding.KDA_ERR_UNSUPPORTED
    assert _bwd_call(lib, dk=64) == binding.KDA_ERR_UNSUPPORTED
    assert _bwd_call(lib, dv=256) == binding.KDA_ERR_UNSUPPORTED
    assert _bwd_call(lib, N=2) == binding.KDA_ERR_INVALID_ARG           # N != B
    assert _bwd_call(lib, H=0) == binding.KDA_ERR_INVALID_ARG
    assert _bwd_call(lib, T=-1) == binding.KDA_ERR_INVALID_ARG
    assert _bwd_call(lib, dt=7) == binding.KDA_ERR_INVALID_ARG
    assert _bwd_call(lib, scale=float("nan")) == binding.KDA_ERR_INVALID_ARG
    assert _bwd_call(lib) == binding.KDA_ERR_INVALID_ARG                 # null tensors
    assert _bwd_call(lib, T=0, H=1, N=0, B=0) == binding.KDA_OK          # nothing to do


def test_binding_backward_refuses_cpu_tensors(lib):
    t = torch.zeros(1, 4, 1, 128)
    with pytest.raises((ValueError, RuntimeError)):
        kda.chunk_bwd(t, t, t, t, torch.zeros(1, 4, 1), t)


def test_unknown_flags_rejected_before_cuda(lib):
    assert lib.kda_chunk_fwd_ex(None, None, None, None, None, None, None, ctypes.c_float(1.0), 64,
                                None, None, 1, 64, 1, 128, 128, 1, 1, 8, None, None,
                                ctypes.c_float(0.0), None, 0, None) == binding.KDA_ERR_UNSUPPORTED
    assert lib.kda_recurrent_step_ex(None, None, None, None, None, None, None,
                                     1, 1, 128, 128, ctypes.c_float(1.0), 1, 8, None, None,
                                     ctypes.c_float(0.0), None) == binding.KDA_ERR_UNSUPPORTED
    # the output epilogue needs a positive eps, checked before any pointer
    assert lib.kda_chunk_fwd_ex(None, None, None, None, None, None, None, ctypes.c_float(1.0), 64,
                                None, None, 1, 64, 1, 128, 128, 1, 1, 2, None, None,
                                ctypes.c_float(0.0), None, 0, None) == binding.KDA_ERR_INVALID_ARG


def test_wait_selftest_limit_validated_before_cuda(lib):
    for bad in (0, -5, 1000001):
        assert lib.kda_selftest_wait_timeout(bad, None) == binding.KDA_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    x = torch.zeros(1, 4, 1, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        kda.chunk_fwd(x, x, x, torch.zeros(1, 4, 1, 128), torch.zeros(1, 4, 1))


@pytest.mark.gpu
def test_pointer_validation_gpu(lib):
    dev = torch.device("cuda")
    B, T, H = 1, 8, 2
    q = torch.randn(B, T, H, 128, device=dev, dtype=torch.bfloat16)
    g = -torch.rand(B, T, H, 128, device=dev)
    b = torch.rand(B, T, H, device=dev)
    out = torch.empty_like(q)
    host = torch.zeros(B, T, H, 128, dtype=torch.bfloat16)
    p = ctypes.c_void_p
    need = binding.chunk_fwd_workspace_bytes(B, T, H, B)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    ok = dict(q=p(q.data_ptr()), k=p(q.data_ptr()), v=p(q.data_ptr()), g=p(g.data_ptr()),
              b=p(b.data_ptr()), out=p(out.data_ptr()), B=B, T=T, H=H, N=B,
              ws=p(ws.data_ptr()), wsb=ws.numel())
    assert _chunk_call(lib, **ok) == binding.KDA_OK
    assert _chunk_call(lib, **{**ok, "q": p(host.data_ptr())}) == binding.KDA_ERR_INVALID_ARG
    assert _chunk_call(lib, **{**ok, "q": p(q.data_ptr() + 2)}) == binding.KDA_ERR_INVALID_ARG
    assert _chunk_call(lib, **{**ok, "out": p(q.data_ptr())}) == binding.KDA_ERR_INVALID_ARG
    assert _chunk_call(lib, **{**ok, "cu": p(0)}) == binding.KDA_OK  # NULL cu_seqlens
    torch.cuda.synchronize()
    assert binding.device_error() == binding.KDA_OK


@pytest.mark.gpu
def test_empty_calls_gpu(lib):
    dev = torch.device("cuda")
    q = torch.zeros(1, 0, 2, 128, device=dev, dtype=torch.bfloat16)
    s0 = torch.randn(1, 2, 128, 128, device=dev)
    out, fs = kda.chunk_fwd(q, q, q, torch.zeros(1, 0, 2, 128, device=dev),
                            torch.zeros(1, 0, 2, device=dev), initial_state=s0)
    torch.cuda.synchronize()
    assert torch.equal(fs, s0)
