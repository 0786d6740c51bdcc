"""B200-native FlashSwin windowed-RoPE attention (forward and backward).

The compute lives in ``libfswin.so`` (hand-written CUDA for sm_100a, C ABI in
``include/fswin.h``); this package only marshals arguments to it.
"""
from ._lib import FswinError, Shape, load, make_shape, status_string  # noqa: F401
from .ops import (WindowAttentionRoPE, alloc_workspace, bwd_workspace_bytes, window_attention,  # noqa: F401
                  winattn_bwd, winattn_fwd)

__all__ = ["FswinError", "Shape", "load", "make_shape", "status_string", "WindowAttentionRoPE", "alloc_workspace",
           "bwd_workspace_bytes", "window_attention", "winattn_bwd", "winattn_fwd"]
