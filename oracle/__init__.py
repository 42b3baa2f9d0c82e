"""KDA oracle -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct CPU evaluations of the Kimi Delta Attention
operator, used to check the CUDA library.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  It shares no code with the CUDA path and never imports it.

Contents
--------
``kda_forward``      fp64 token-by-token recurrence (C, OpenMP over
                     sequence x head), built from ``kda_oracle.c``; options
                     for the layer's adjacent steps: the L2Norm of q and k
                     (``l2norm_rows``), the gate from its pre-activation
                     (``log_sigmoid``), the output norm and gate
                     (``out_norm_gate``).
``kda_backward``     fp64 reverse-mode adjoint of the same recurrence (C):
                     the gradients of out and final_state with respect to
                     q, k, v, log_alpha, beta and initial_state.
``chunked``          fp64 restatement of the chunkwise algorithm (numpy), with
                     its intermediates, used to pin the chunk algebra; and
                     of its adjoint (``chunked_backward``).

Every function here is pinned by ``tests/test_oracle.py`` against special
cases, closed forms and brute force; see that file for which pin covers what.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        d = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.kda_oracle_forward.argtypes = [d, d, d, d, d, d, i64p,
                                           i64, i64, i64, i64, i64, i64,
                                           ctypes.c_double, d, d, ctypes.c_int]
        lib.kda_oracle_forward.restype = ctypes.c_int
        lib.kda_oracle_backward.argtypes = [d, d, d, d, d, d, i64p, d, d,
                                            i64, i64, i64, i64, i64, i64,
                                            ctypes.c_double, d, d, d, d, d, d, ctypes.c_int]
        lib.kda_oracle_backward.restype = ctypes.c_int
        lib.kda_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _f64(x):
    """Exact fp64 copy of a torch tensor (any float dtype) or array."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, ctype=ctypes.c_double):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctype))


def l2norm_rows(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """x / max(||x||_2, eps) over the last axis, in fp64: the L2Norm the layer
    applies to q and k before the recurrence ("深度解读报告" 3.2)."""
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def out_norm_gate(o: np.ndarray, gate, weight, eps: float) -> np.ndarray:
    """The layer's output side in fp64 ("深度解读报告" 3.2: head-wise RMSNorm
    and a data-dependent sigmoid output gate): every [dv] row o becomes
    o / sqrt(mean(o^2) + eps) * weight * sigmoid(gate)."""
    g = _f64(gate)
    w = _f64(weight)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + eps) * w / (1.0 + np.exp(-g))


def log_sigmoid(z: np.ndarray) -> np.ndarray:
    """log sigmoid(z) = -log(1 + e^-z) in fp64, without overflow: the log of
    the forget gate alpha = sigmoid(z) from its pre-activation z (the reading
    taken of "深度解读报告" 3.2, which obtains the gate from a low-rank
    projection and prints no activation)."""
    return -np.logaddexp(0.0, -z)


def kda_forward(q, k, v, log_alpha, beta, initial_state=None, cu_seqlens=None,
                scale=None, nthreads: int = 0, l2norm_qk: bool = False,
                out_gate=None, out_weight=None, out_eps: float = 1e-6,
                raw_gate: bool = False):
    """fp64 token-by-token KDA forward.

    Shapes: q, k, log_alpha [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H];
    initial_state [N,H,dk,dv] or None; cu_seqlens [N+1] or None (then N = B).
    Returns ``(out [B,T,H,dv], final_state [N,H,dk,dv])`` as fp64 numpy arrays.
    ``scale`` defaults to dk ** -0.5.  ``l2norm_qk``: the q and k rows are
    first L2-normalised (``l2norm_rows``), as the operator's fused option does.
    ``out_gate`` (shaped like out) and ``out_weight`` [dv]: the output rows
    then go through ``out_norm_gate``; final_state is unaffected.
    ``raw_gate``: ``log_alpha`` holds the gate's pre-activations z and the
    recurrence uses ``log_sigmoid(z)``.
    """
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    if raw_gate:
        g = log_sigmoid(g)
    if l2norm_qk:
        q, k = l2norm_rows(q), l2norm_rows(k)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != (B, T, H) \
            or b.shape != (B, T, H):
        raise ValueError("inconsistent shapes")
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int64))
        N = cu.shape[0] - 1
    else:
        cu = None
        N = B
    s0 = _f64(initial_state)
    if s0 is not None and s0.shape != (N, H, dk, dv):
        raise ValueError("initial_state shape")
    if scale is None:
        scale = dk ** -0.5
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    fs = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(s0),
        _ptr(cu, ctypes.c_int64), B, T, H, dk, dv, N, float(scale),
        _ptr(out), _ptr(fs), int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_forward failed with code {rc}")
    if out_gate is not None:
        out = out_norm_gate(out, out_gate, out_weight, out_eps)
    return out, fs


def kda_backward(q, k, v, log_alpha, beta, d_out, initial_state=None, d_final_state=None,
                 cu_seqlens=None, scale=None, nthreads: int = 0):
    """fp64 backward pass of ``kda_forward`` (without its L2Norm and output
    options): given the adjoints ``d_out`` [B,T,H,dv] of the outputs and
    ``d_final_state`` [N,H,dk,dv] (None = zeros) of the final state, returns
    ``(dq, dk, dv, dlog_alpha, dbeta, d_initial_state)`` as fp64 arrays shaped
    like q, k, v, log_alpha, beta and the initial state [N,H,dk,dv]."""
    q, k, v, g, b, do = (_f64(x) for x in (q, k, v, log_alpha, beta, d_out))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != (B, T, H) \
            or b.shape != (B, T, H) or do.shape != v.shape:
        raise ValueError("inconsistent shapes")
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
            dtype=np.int64))
        N = cu.shape[0] - 1
    else:
        cu = None
        N = B
    s0 = _f64(initial_state)
    dfs = _f64(d_final_state)
    for a in (s0, dfs):
        if a is not None and a.shape != (N, H, dk, dv):
            raise ValueError("state shape")
    if scale is None:
        scale = dk ** -0.5
    dq = np.zeros_like(q)
    dkk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dg = np.zeros_like(g)
    db = np.zeros_like(b)
    ds0 = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(s0), _ptr(cu, ctypes.c_int64),
        _ptr(do), _ptr(dfs), B, T, H, dk, dv, N, float(scale),
        _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(db), _ptr(ds0), int(nthreads))
    if rc != 0:
        raise ValueError(f"kda_oracle_backward failed with code {rc}")
    return dq, dkk, dvv, dg, db, ds0


def kda_decode_step(q, k, v, log_alpha, beta, state, scale=None, nthreads: int = 0,
                    l2norm_qk: bool = False, out_gate=None, out_weight=None,
                    out_eps: float = 1e-6, raw_gate: bool = False):
    """One decode step for N requests: the recurrence applied to a single
    token per (request, head).  Shapes: q, k, log_alpha [N,H,dk]; v [N,H,dv];
    beta [N,H]; state [N,H,dk,dv].  Returns ``(out [N,H,dv], new_state)``."""
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    out, fs = kda_forward(q[:, None], k[:, None], v[:, None], g[:, None], b[:, None],
                          initial_state=state, scale=scale, nthreads=nthreads,
                          l2norm_qk=l2norm_qk, raw_gate=raw_gate)
    out = out[:, 0]
    if out_gate is not None:
        out = out_norm_gate(out, out_gate, out_weight, out_eps)
    return out, fs
