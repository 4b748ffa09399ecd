"""Sketch Attention (SA, FlashSA) and STCA for NVIDIA B200 (sm_100a).

The compute path is libska.so (hand-written tcgen05/TMA kernels behind a C ABI, declared in
include/sketch_attn.h); this package is a thin ctypes binding plus the seeded workload
generators and the FLOP accounting. There is no CPU fallback: calling the API without the
built library or without a CUDA device raises.
"""
from ._lib import SkaError, LIB_PATH  # noqa: F401


def __getattr__(name):
    if name in ("sa_forward", "sa_desc", "sa_forward_workspace_size", "read_device_status",
                "set_debug", "sa_backward", "stca_forward", "stca_desc", "stca_forward_workspace_size",
                "set_timing_events"):
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
