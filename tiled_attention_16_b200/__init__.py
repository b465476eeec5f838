"""Exact tiled (flash) attention for NVIDIA B200 (sm_100a).

The compute lives in ``libfa_sm100.so`` (C ABI declared in include/fa.h);
``attention`` is its thin Python binding.  The shared library is loaded on
first use, so importing this package (for example for the seeded workloads
in ``workloads``) needs no GPU.
"""
from .attention import (  # noqa: F401
    FA_ERR_CUDA,
    FA_ERR_INVALID_ARG,
    FA_ERR_TIMEOUT,
    FA_ERR_UNSUPPORTED,
    FA_OK,
    FAError,
    bwd,
    device_status,
    fwd,
    workspace_bytes,
)
