"""B200-native Kimi Delta Attention (KDA) operator.

``chunk_fwd`` (chunked prefill), ``chunk_bwd`` (its backward pass) and
``recurrent_step`` (batched decode) run
hand-written sm_100a CUDA kernels through the library's C ABI
(``include/kda.h``).  The binding only marshals arguments; there is no CPU
fallback: on a machine without the built library or a CUDA device the calls
raise.
"""
from .binding import (  # noqa: F401
    KDAError,
    chunk_bwd,
    chunk_bwd_workspace_bytes,
    chunk_fwd,
    chunk_fwd_workspace_bytes,
    chunk_transition,
    state_affine,
    recurrent_step,
    load_library,
    library_path,
)

__all__ = ["chunk_fwd", "chunk_bwd", "recurrent_step", "chunk_transition", "state_affine",
           "chunk_fwd_workspace_bytes",
           "chunk_bwd_workspace_bytes", "KDAError", "load_library", "library_path"]
