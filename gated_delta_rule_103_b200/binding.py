"""Thin ctypes binding over the KDA C ABI (``include/kda.h``).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, then their ``data_ptr()`` and the current CUDA stream are passed to
the library, whose kernels do all of the work.  There is no CPU fallback: if
the library is missing or the tensors are not on a CUDA device, the calls
raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libkda_b200.so"

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(5)
KDA_DTYPE_F32, KDA_DTYPE_BF16 = 0, 1
KDA_FLAG_L2NORM_QK = 1
KDA_FLAG_OUT_NORM_GATE = 2
KDA_FLAG_RAW_GATE = 4

# Every symbol include/kda.h declares.
EXPORTED_SYMBOLS = ("kda_chunk_fwd", "kda_recurrent_step", "kda_status_string",
                    "kda_device_error", "kda_version", "kda_chunk_debug_stages",
                    "kda_chunk_debug_stage_floats", "kda_set_prefill_kernel",
                    "kda_prefill_kernel_choice", "kda_chunk_fwd_noalloc",
                    "kda_selftest_wait_timeout", "kda_chunk_fwd_ex", "kda_recurrent_step_ex",
                    "kda_chunk_bwd", "kda_chunk_fwd_workspace_bytes",
                    "kda_chunk_bwd_workspace_bytes", "kda_set_prefill_segments",
                    "kda_prefill_segments", "kda_chunk_transition",
                    "kda_chunk_transition_workspace_bytes", "kda_state_affine",
                    "kda_set_prefill_dual")

_lib = None


class KDAError(RuntimeError):
    """A KDA library call returned an error status."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        msg = status_string(status) if _lib is not None else f"status {status}"
        super().__init__(f"{where}: {msg}")


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load_library(path: Optional[str] = None):
    """Load (once) the compiled library.  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or library_path()
    if not os.path.exists(path):
        raise RuntimeError(
            f"KDA CUDA library not found at {path}; build it with "
            "`python -m gated_delta_rule_103_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    vp, fp, i32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    ci, cf = ctypes.c_int, ctypes.c_float
    sz = ctypes.c_size_t
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, i32p, cf, ci, vp, fp,
                                  ci, ci, ci, ci, ci, ci, ci, vp, sz, vp]
    lib.kda_chunk_fwd.restype = ci
    lib.kda_chunk_fwd_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
    lib.kda_chunk_fwd_workspace_bytes.restype = sz
    lib.kda_chunk_bwd_workspace_bytes.argtypes = [ci, ci, ci, ci, ci, ci]
    lib.kda_chunk_bwd_workspace_bytes.restype = sz
    lib.kda_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, vp,
                                       ci, ci, ci, ci, cf, ci, vp]
    lib.kda_recurrent_step.restype = ci
    lib.kda_status_string.argtypes = [ci]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_device_error.argtypes = [vp]
    lib.kda_device_error.restype = ci
    lib.kda_version.restype = ci
    lib.kda_chunk_debug_stages.argtypes = [vp, vp, vp, fp, fp, fp, cf, ci, vp, fp, fp, vp]
    lib.kda_chunk_debug_stages.restype = ci
    lib.kda_chunk_debug_stage_floats.restype = ci
    lib.kda_set_prefill_kernel.argtypes = [ci]
    lib.kda_set_prefill_kernel.restype = ci
    lib.kda_prefill_kernel_choice.argtypes = [ci, ci, ci, ci]
    lib.kda_prefill_kernel_choice.restype = ci
    lib.kda_prefill_segments.argtypes = [ci, ci, ci, ci]
    lib.kda_prefill_segments.restype = ci
    lib.kda_set_prefill_segments.argtypes = [ci]
    lib.kda_set_prefill_segments.restype = ci
    lib.kda_set_prefill_dual.argtypes = [ci]
    lib.kda_set_prefill_dual.restype = ci
    lib.kda_chunk_fwd_ex.argtypes = lib.kda_chunk_fwd.argtypes[:-3] + [ctypes.c_uint, vp, fp, cf,
                                                                        vp, sz, vp]
    lib.kda_chunk_fwd_ex.restype = ci
    lib.kda_recurrent_step_ex.argtypes = lib.kda_recurrent_step.argtypes[:-1] + [ctypes.c_uint, vp, fp,
                                                                                  cf, vp]
    lib.kda_recurrent_step_ex.restype = ci
    lib.kda_chunk_fwd_noalloc.argtypes = lib.kda_chunk_fwd.argtypes[:-3] + [vp]
    lib.kda_chunk_fwd_noalloc.restype = ci
    lib.kda_selftest_wait_timeout.argtypes = [ci, vp]
    lib.kda_selftest_wait_timeout.restype = ci
    lib.kda_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, i32p, vp, fp, cf, ci,
                                  fp, fp, fp, fp, fp, fp, ci, ci, ci, ci, ci, ci, ci, vp, sz, vp]
    lib.kda_chunk_bwd.restype = ci
    lib.kda_chunk_transition.argtypes = [vp, vp, fp, fp, i32p, fp, ci, ci, ci, ci, ci, ci,
                                         ctypes.c_uint, vp, sz, vp]
    lib.kda_chunk_transition.restype = ci
    lib.kda_chunk_transition_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
    lib.kda_chunk_transition_workspace_bytes.restype = sz
    lib.kda_state_affine.argtypes = [fp, fp, fp, fp, ci, ci, ci, ci, vp]
    lib.kda_state_affine.restype = ci
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().kda_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != KDA_OK:
        raise KDAError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_DTYPE_BF16
    if t.dtype == torch.float32:
        return KDA_DTYPE_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("KDA tensors must be on a CUDA device (no CPU fallback)")


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _workspace(need: int, workspace: Optional[torch.Tensor], device):
    """The (pointer, bytes) of the caller's workspace for a call that needs
    ``need`` bytes: the given uint8 tensor, or a new one (torch's allocator,
    so the memory is the caller's, not the library's)."""
    if need == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    _need_cuda(workspace)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous() \
            or workspace.numel() < need:
        raise ValueError(f"workspace must be a contiguous uint8 tensor of >= {need} bytes")
    return ctypes.c_void_p(workspace.data_ptr()), workspace.numel()


def chunk_fwd_workspace_bytes(B: int, T: int, H: int, N: int, dtype=torch.bfloat16) -> int:
    """``kda_chunk_fwd_workspace_bytes``: device workspace a chunk_fwd call of
    these sizes needs on the current device (0: none)."""
    dt = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_F32
    return int(load_library().kda_chunk_fwd_workspace_bytes(B, T, H, N, dt))


def chunk_bwd_workspace_bytes(B: int, T: int, H: int, N: int, packed: bool,
                              dtype=torch.bfloat16) -> int:
    """``kda_chunk_bwd_workspace_bytes`` (``packed``: cu_seqlens is passed)."""
    dt = KDA_DTYPE_BF16 if dtype == torch.bfloat16 else KDA_DTYPE_F32
    return int(load_library().kda_chunk_bwd_workspace_bytes(B, T, H, N, int(packed), dt))


def chunk_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
              log_alpha: torch.Tensor, beta: torch.Tensor,
              initial_state: Optional[torch.Tensor] = None,
              cu_seqlens: Optional[torch.Tensor] = None,
              scale: Optional[float] = None, chunk: int = 64,
              output_final_state: bool = True,
              out: Optional[torch.Tensor] = None,
              final_state: Optional[torch.Tensor] = None,
              stream=None, l2norm_qk: bool = False,
              out_gate: Optional[torch.Tensor] = None,
              out_weight: Optional[torch.Tensor] = None,
              out_eps: float = 1e-6,
              workspace: Optional[torch.Tensor] = None,
              raw_gate: bool = False) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked KDA prefill (``kda_chunk_fwd``; ``kda_chunk_fwd_ex`` when
    ``l2norm_qk`` (KDA_FLAG_L2NORM_QK: q and k rows L2-normalised inside the
    kernels) or ``out_gate`` is given (KDA_FLAG_OUT_NORM_GATE: out becomes
    RMSNorm(out) * out_weight * sigmoid(out_gate) per (token, head) row;
    out_gate shaped and typed like out, out_weight [dv] fp32)).  ``workspace``:
    a uint8 device tensor of at least ``chunk_fwd_workspace_bytes(...)`` bytes
    (allocated here with torch when None and needed).  ``raw_gate``
    (KDA_FLAG_RAW_GATE): ``log_alpha`` holds the gate's pre-activations z and
    the kernels use log sigmoid(z).

    q, k [B,T,H,dk], v [B,T,H,dv] in bf16 or fp32; log_alpha [B,T,H,dk] and
    beta [B,T,H] fp32; initial_state [N,H,dk,dv] fp32 or None; cu_seqlens
    [N+1] int32 (B must be 1) or None.  Returns ``(out, final_state)``;
    ``final_state`` may be passed equal to ``initial_state`` to update it in
    place.
    """
    lib = load_library()
    _need_cuda(q, k, v, log_alpha, beta, initial_state, cu_seqlens, out, final_state)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k and v must share a dtype")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("log_alpha and beta must be float32")
    if k.shape != q.shape or log_alpha.shape != q.shape or tuple(v.shape[:3]) != (B, T, H) \
            or tuple(beta.shape) != (B, T, H):
        raise ValueError("inconsistent shapes")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise TypeError("cu_seqlens must be a 1-D int32 tensor")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    for t in (q, k, v, log_alpha, beta, initial_state, cu_seqlens):
        if t is not None and not t.is_contiguous():
            raise ValueError("KDA tensors must be contiguous")
    if initial_state is not None:
        if initial_state.dtype != torch.float32 or tuple(initial_state.shape) != (N, H, dk, dv):
            raise ValueError("initial_state must be float32 [N,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
            _ptr(initial_state), _ptr(cu_seqlens), float(scale), int(chunk),
            _ptr(out), _ptr(final_state), B, T, H, dk, dv, N, dt)
    flags, extra = _options(l2norm_qk, out_gate, out_weight, out_eps, out, dv)
    flags |= KDA_FLAG_RAW_GATE if raw_gate else 0
    ws = _workspace(int(lib.kda_chunk_fwd_workspace_bytes(B, T, H, N, dt)), workspace, q.device)
    if flags:
        _check(lib.kda_chunk_fwd_ex(*args, flags, *extra, *ws, _stream(stream)), "kda_chunk_fwd_ex")
    else:
        _check(lib.kda_chunk_fwd(*args, *ws, _stream(stream)), "kda_chunk_fwd")
    return out, final_state


def chunk_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
              log_alpha: torch.Tensor, beta: torch.Tensor, d_out: torch.Tensor,
              initial_state: Optional[torch.Tensor] = None,
              d_final_state: Optional[torch.Tensor] = None,
              cu_seqlens: Optional[torch.Tensor] = None,
              scale: Optional[float] = None, chunk: int = 64,
              need_initial_state_grad: bool = True, stream=None,
              workspace: Optional[torch.Tensor] = None, grads=None):
    """Backward pass of ``chunk_fwd`` (``kda_chunk_bwd``).

    Inputs as for ``chunk_fwd`` plus ``d_out`` (shaped and typed like out) and
    ``d_final_state`` [N,H,dk,dv] fp32 or None (zero).  Returns fp32
    ``(dq, dk, dv, dlog_alpha, dbeta, d_initial_state)``; the last is None
    when ``need_initial_state_grad`` is false.  ``grads``: the caller's six
    output tensors (the last may be None) instead of new ones; ``workspace``
    as for ``chunk_fwd`` (``chunk_bwd_workspace_bytes``).
    """
    lib = load_library()
    _need_cuda(q, k, v, log_alpha, beta, d_out, initial_state, d_final_state, cu_seqlens)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or d_out.dtype != q.dtype:
        raise TypeError("q, k, v and d_out must share a dtype")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("log_alpha and beta must be float32")
    if k.shape != q.shape or log_alpha.shape != q.shape or tuple(v.shape[:3]) != (B, T, H) \
            or tuple(beta.shape) != (B, T, H) or d_out.shape != v.shape:
        raise ValueError("inconsistent shapes")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise TypeError("cu_seqlens must be a 1-D int32 tensor")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    for t in (q, k, v, log_alpha, beta, d_out, initial_state, d_final_state, cu_seqlens):
        if t is not None and not t.is_contiguous():
            raise ValueError("KDA tensors must be contiguous")
    for t in (initial_state, d_final_state):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (N, H, dk, dv)):
            raise ValueError("states must be float32 [N,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    f32 = dict(dtype=torch.float32, device=q.device)
    if grads is None:
        dq = torch.empty((B, T, H, dk), **f32)
        dkk = torch.empty((B, T, H, dk), **f32)
        dvv = torch.empty((B, T, H, dv), **f32)
        dg = torch.empty((B, T, H, dk), **f32)
        db = torch.empty((B, T, H), **f32)
        ds0 = torch.empty((N, H, dk, dv), **f32) if need_initial_state_grad else None
    else:
        dq, dkk, dvv, dg, db, ds0 = grads
        shapes = [(B, T, H, dk), (B, T, H, dk), (B, T, H, dv), (B, T, H, dk), (B, T, H),
                  (N, H, dk, dv)]
        for t, shp in zip(grads, shapes):
            if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != shp
                                  or not t.is_contiguous() or not t.is_cuda):
                raise ValueError("grads must be contiguous fp32 CUDA tensors of the input shapes")
    ws = _workspace(int(lib.kda_chunk_bwd_workspace_bytes(B, T, H, N, int(cu_seqlens is not None),
                                                          dt)), workspace, q.device)
    _check(lib.kda_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                             _ptr(initial_state), _ptr(cu_seqlens), _ptr(d_out),
                             _ptr(d_final_state), float(scale), int(chunk),
                             _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(db), _ptr(ds0),
                             B, T, H, dk, dv, N, dt, *ws, _stream(stream)), "kda_chunk_bwd")
    return dq, dkk, dvv, dg, db, ds0


def chunk_transition(q: torch.Tensor, k: torch.Tensor, log_alpha: torch.Tensor,
                     beta: torch.Tensor, cu_seqlens: Optional[torch.Tensor] = None,
                     l2norm_qk: bool = False, raw_gate: bool = False,
                     out: Optional[torch.Tensor] = None, stream=None,
                     workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``kda_chunk_transition``: the state transition M [N,H,dk,dk] fp32 of
    every (sequence, head), so that chunk_fwd's final state from an initial
    state S0 is M S0 + (its final state from zeros).  q, k [B,T,H,dk] bf16,
    log_alpha [B,T,H,dk] and beta [B,T,H] fp32, as for chunk_fwd."""
    lib = load_library()
    _need_cuda(q, k, log_alpha, beta, cu_seqlens, out)
    B, T, H, dk = k.shape
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16:
        raise TypeError("q and k must be bfloat16")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("log_alpha and beta must be float32")
    if q.shape != k.shape or log_alpha.shape != k.shape or tuple(beta.shape) != (B, T, H):
        raise ValueError("inconsistent shapes")
    N = cu_seqlens.numel() - 1 if cu_seqlens is not None else B
    for t in (q, k, log_alpha, beta, cu_seqlens):
        if t is not None and not t.is_contiguous():
            raise ValueError("KDA tensors must be contiguous")
    if out is None:
        out = torch.empty((N, H, dk, dk), dtype=torch.float32, device=k.device)
    flags = (KDA_FLAG_L2NORM_QK if l2norm_qk else 0) | (KDA_FLAG_RAW_GATE if raw_gate else 0)
    ws = _workspace(int(lib.kda_chunk_transition_workspace_bytes(B, T, H, N, KDA_DTYPE_BF16)),
                    workspace, k.device)
    _check(lib.kda_chunk_transition(_ptr(q), _ptr(k), _ptr(log_alpha), _ptr(beta),
                                    _ptr(cu_seqlens), _ptr(out), B, T, H, dk, N,
                                    KDA_DTYPE_BF16, flags, *ws, _stream(stream)),
           "kda_chunk_transition")
    return out


def state_affine(M: torch.Tensor, B: torch.Tensor, S_in: torch.Tensor,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """``kda_state_affine``: M S_in + B per (sequence, head) in fp32 (M
    [N,H,dk,dk], B and S_in [N,H,dk,dv]); ``out`` may be B."""
    lib = load_library()
    _need_cuda(M, B, S_in, out)
    N, H, dk, dv = B.shape
    for t in (M, B, S_in):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("states must be contiguous float32")
    if tuple(M.shape) != (N, H, dk, dk) or S_in.shape != B.shape:
        raise ValueError("inconsistent shapes")
    if out is None:
        out = torch.empty_like(B)
    _check(lib.kda_state_affine(_ptr(M), _ptr(B), _ptr(S_in), _ptr(out), N, H, dk, dv,
                                _stream(stream)), "kda_state_affine")
    return out


def _options(l2norm_qk, out_gate, out_weight, out_eps, out, dv):
    """The _ex entry points' flags and (out_gate, out_weight, out_eps)."""
    flags = KDA_FLAG_L2NORM_QK if l2norm_qk else 0
    if out_gate is None:
        if out_weight is not None:
            raise ValueError("out_weight needs out_gate")
        return flags, (None, None, 0.0)
    _need_cuda(out_gate, out_weight)
    if out_weight is None or out_weight.dtype != torch.float32 or tuple(out_weight.shape) != (dv,):
        raise ValueError("out_weight must be float32 [dv]")
    if out_gate.dtype != out.dtype or out_gate.shape != out.shape:
        raise ValueError("out_gate must match out in shape and dtype")
    if not (out_gate.is_contiguous() and out_weight.is_contiguous()):
        raise ValueError("KDA tensors must be contiguous")
    return flags | KDA_FLAG_OUT_NORM_GATE, (_ptr(out_gate), _ptr(out_weight), float(out_eps))


def recurrent_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                   log_alpha: torch.Tensor, beta: torch.Tensor, state: torch.Tensor,
                   scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                   stream=None, l2norm_qk: bool = False,
                   out_gate: Optional[torch.Tensor] = None,
                   out_weight: Optional[torch.Tensor] = None,
                   out_eps: float = 1e-6, raw_gate: bool = False) -> torch.Tensor:
    """One batched decode step (``kda_recurrent_step``, or
    ``kda_recurrent_step_ex`` with KDA_FLAG_L2NORM_QK when ``l2norm_qk``,
    KDA_FLAG_RAW_GATE when ``raw_gate``);
    ``state`` [N,H,dk,dv] fp32 is updated in place.  q, k [N,H,dk], v
    [N,H,dv]; log_alpha [N,H,dk], beta [N,H] fp32.  Returns out [N,H,dv]."""
    lib = load_library()
    _need_cuda(q, k, v, log_alpha, beta, state, out)
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k and v must share a dtype")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32 \
            or state.dtype != torch.float32:
        raise TypeError("log_alpha, beta and state must be float32")
    if tuple(state.shape) != (N, H, dk, dv) or tuple(beta.shape) != (N, H):
        raise ValueError("inconsistent shapes")
    for t in (q, k, v, log_alpha, beta, state):
        if not t.is_contiguous():
            raise ValueError("KDA tensors must be contiguous")
    if scale is None:
        scale = dk ** -0.5
    if out is None:
        out = torch.empty((N, H, dv), dtype=q.dtype, device=q.device)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
            _ptr(state), _ptr(out), N, H, dk, dv, float(scale), dt)
    flags, extra = _options(l2norm_qk, out_gate, out_weight, out_eps, out, dv)
    flags |= KDA_FLAG_RAW_GATE if raw_gate else 0
    if flags:
        _check(lib.kda_recurrent_step_ex(*args, flags, *extra, _stream(stream)),
               "kda_recurrent_step_ex")
    else:
        _check(lib.kda_recurrent_step(*args, _stream(stream)), "kda_recurrent_step")
    return out


def chunk_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      log_alpha: torch.Tensor, beta: torch.Tensor, out: torch.Tensor,
                      initial_state: Optional[torch.Tensor] = None,
                      final_state: Optional[torch.Tensor] = None,
                      cu_seqlens: Optional[torch.Tensor] = None,
                      scale: Optional[float] = None, stream=None) -> None:
    """``kda_chunk_fwd_noalloc``: the bf16 chunked prefill for callers that
    must not allocate device memory during the call.  Nothing here allocates
    either: ``out`` [B,T,H,dv] bf16 (and ``final_state`` [N,H,dk,dv] fp32, or
    None) are the caller's.  N * H must be at most 126; calls whose
    executions overlap in time race on the library's fixed ring array."""
    lib = load_library()
    _need_cuda(q, k, v, log_alpha, beta, out, initial_state, final_state, cu_seqlens)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype != torch.bfloat16 or k.dtype != q.dtype or v.dtype != q.dtype \
            or out.dtype != q.dtype:
        raise TypeError("q, k, v and out must be bfloat16")
    if log_alpha.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("log_alpha and beta must be float32")
    if k.shape != q.shape or log_alpha.shape != q.shape or tuple(v.shape[:3]) != (B, T, H) \
            or tuple(beta.shape) != (B, T, H) or tuple(out.shape) != (B, T, H, dv):
        raise ValueError("inconsistent shapes")
    if cu_seqlens is not None:
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise TypeError("cu_seqlens must be a 1-D int32 tensor")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    for t in (q, k, v, log_alpha, beta, out, initial_state, final_state, cu_seqlens):
        if t is not None and not t.is_contiguous():
            raise ValueError("KDA tensors must be contiguous")
    for t in (initial_state, final_state):
        if t is not None and (t.dtype != torch.float32 or tuple(t.shape) != (N, H, dk, dv)):
            raise ValueError("states must be float32 [N,H,dk,dv]")
    if scale is None:
        scale = dk ** -0.5
    st = lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                   _ptr(initial_state), _ptr(cu_seqlens), float(scale), 64,
                                   _ptr(out), _ptr(final_state), B, T, H, dk, dv, N,
                                   KDA_DTYPE_BF16, _stream(stream))
    _check(st, "kda_chunk_fwd_noalloc")


def selftest_wait_timeout(limit_us: int = 10000, stream=None) -> None:
    """Enqueues the library's bounded-wait self-test: one CTA waits on an
    mbarrier that nothing arrives on until ``limit_us`` runs out, and records
    the timeout; read it with ``device_error()``."""
    _check(load_library().kda_selftest_wait_timeout(int(limit_us), _stream(stream)),
           "kda_selftest_wait_timeout")


PREFILL_KERNELS = {"auto": 0, "cta": 1, "cluster": 2, "segmented": 3}


PREFILL_DUAL = {"auto": 0, "separate": 1, "shared": 2}


def set_prefill_kernel(kind: str = "auto", segments: int = 0, first_pass: str = "auto") -> None:
    """Selects the bf16 prefill kernel process-wide: "auto" (default; one
    thread-block cluster per (sequence, head) chain when the chains are few,
    segmented clusters when they are very few, else one CTA per chain),
    "cta", "cluster" or "segmented" (``segments``: the segment count, 0 by the
    cost model; ``first_pass``: "separate" or "shared" clusters for a
    segment's zero-start and transition runs, "auto" by the cost model)."""
    if kind not in PREFILL_KERNELS:
        raise ValueError(f"kind must be one of {sorted(PREFILL_KERNELS)}")
    if first_pass not in PREFILL_DUAL:
        raise ValueError(f"first_pass must be one of {sorted(PREFILL_DUAL)}")
    lib = load_library()
    _check(lib.kda_set_prefill_kernel(PREFILL_KERNELS[kind]), "kda_set_prefill_kernel")
    _check(lib.kda_set_prefill_segments(int(segments)), "kda_set_prefill_segments")
    _check(lib.kda_set_prefill_dual(PREFILL_DUAL[first_pass]), "kda_set_prefill_dual")


def prefill_kernel_choice(B: int, T: int, H: int, N: int) -> str:
    """The bf16 prefill kernel ("cta", "cluster" or "segmented") a call of
    these sizes would use on the current device under the current setting."""
    r = load_library().kda_prefill_kernel_choice(B, T, H, N)
    if r not in (1, 2, 3):
        raise ValueError("invalid sizes")
    return {1: "cta", 2: "cluster", 3: "segmented"}[r]


def prefill_segments(B: int, T: int, H: int, N: int) -> int:
    """Segments per sequence such a call would use (1: not segmented)."""
    r = load_library().kda_prefill_segments(B, T, H, N)
    if r < 1:
        raise ValueError("invalid sizes")
    return int(r)


def device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(load_library().kda_device_error(_stream(stream)))


# Offsets (in floats) of the intermediates kda_chunk_debug_stages writes.
DEBUG_STAGES = {
    "AP": (0, (128, 64)), "T": (8192, (64, 64)), "WT": (12288, (128, 64)),
    "UpT": (20480, (128, 64)), "O1T": (28672, (128, 64)), "UT": (36864, (128, 64)),
    "DT": (45056, (128, 128)), "OT": (61440, (128, 64)), "ST": (69632, (128, 128)),
}


def chunk_debug_stages(q, k, v, log_alpha, beta, initial_state=None, scale=None, stream=None):
    """One chunk (T <= 64) of one head through the bf16 tensor-core kernel;
    returns (out [T, dv], final_state [dk, dv], dict of intermediate tiles).
    q, k [T, dk], v [T, dv] bf16; log_alpha [T, dk], beta [T] fp32."""
    lib = load_library()
    _need_cuda(q, k, v, log_alpha, beta, initial_state)
    T, dk = q.shape
    if scale is None:
        scale = dk ** -0.5
    out = torch.empty((T, v.shape[-1]), dtype=q.dtype, device=q.device)
    fs = torch.empty((dk, v.shape[-1]), dtype=torch.float32, device=q.device)
    n = lib.kda_chunk_debug_stage_floats()
    stages = torch.full((n,), float("nan"), dtype=torch.float32, device=q.device)
    st = lib.kda_chunk_debug_stages(_ptr(q.contiguous()), _ptr(k.contiguous()), _ptr(v.contiguous()),
                                    _ptr(log_alpha.contiguous()), _ptr(beta.contiguous()),
                                    _ptr(initial_state), float(scale), T, _ptr(out), _ptr(fs),
                                    _ptr(stages), _stream(stream))
    _check(st, "kda_chunk_debug_stages")
    torch.cuda.synchronize()
    d = {name: stages[o:o + r * c].view(r, c) for name, (o, (r, c)) in DEBUG_STAGES.items()}
    return out, fs, d
