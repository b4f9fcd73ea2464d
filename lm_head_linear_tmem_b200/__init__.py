"""B200-native fused linear cross-entropy (FLCE).

The hot path is a C-ABI CUDA library (`include/flce.h`, sources in `csrc/`)
with hand-written sm_100a kernels: tcgen05/TMEM bf16 GEMM tiles fed by TMA
with the softcap, an online fp32 logsumexp and the label gather fused into the
forward epilogue, and a backward that recomputes logit tiles, forms dZ in
registers and feeds two more tensor-core GEMMs (dHidden, split-K dWeight).
This package is its thin PyTorch binding.
"""
from .flce import (  # noqa: F401
    FlceForward, FusedLinearCrossEntropy, alloc_workspace, backward, forward,
    fused_linear_cross_entropy, status, workspace_bytes,
)
from ._native import FlceError, get_option, load, options, set_option  # noqa: F401

__all__ = [
    "FlceForward", "FusedLinearCrossEntropy", "FlceError", "alloc_workspace", "backward",
    "forward", "fused_linear_cross_entropy", "get_option", "load", "options", "set_option",
    "status", "workspace_bytes",
]
