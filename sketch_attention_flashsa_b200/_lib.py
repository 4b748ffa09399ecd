"""ctypes view of libska.so (include/sketch_attn.h). Argument marshalling only."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libska.so")

SKA_OK = 0
SKA_ERR_INVALID_VALUE = 1
SKA_ERR_UNSUPPORTED = 2
SKA_ERR_WORKSPACE_TOO_SMALL = 3
SKA_ERR_CUDA = 4
SKA_ERR_DEVICE_TIMEOUT = 5
SKA_ERR_RANGE = 6

SKA_BF16 = 0
SKA_F32 = 1
SKA_NORM_PROTO = 0
SKA_NORM_TOKEN = 1

EXPORTED = ("sa_forward_workspace_size", "sa_forward", "sa_backward_workspace_size", "sa_backward",
            "stca_forward_workspace_size", "stca_forward", "ska_status_string",
            "ska_read_device_status", "ska_set_debug", "ska_set_timing_events",
            "sa_forward_noalloc", "sa_forward_noalloc_scratch_bytes", "sa_forward_noalloc_read_status",
            "ska_last_error_string", "sa_refine_workspace_size", "sa_refine", "sa_project_queries",
            "stca_backward_workspace_size", "stca_backward", "sa_forward_diag", "sa_weight_histogram",
            "sa_cache_bytes", "sa_cache_init", "sa_cache_put", "sa_cache_get")


class SaDesc(ctypes.Structure):
    _fields_ = [("num_users", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("num_protos", ctypes.c_int32),
                ("total_tokens", ctypes.c_int64), ("max_seqlen", ctypes.c_int32),
                ("scale", ctypes.c_float), ("norm", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
                ("q_per_user", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class StcaDesc(ctypes.Structure):
    _fields_ = [("num_users", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("num_sketch", ctypes.c_int32),
                ("total_targets", ctypes.c_int64), ("total_hist", ctypes.c_int64),
                ("max_targets", ctypes.c_int32), ("max_hist", ctypes.c_int32),
                ("scale", ctypes.c_float), ("reserved", ctypes.c_int32)]


class RefineDesc(ctypes.Structure):
    _fields_ = [("num_users", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("num_protos", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ffn_dim", ctypes.c_int32), ("eps", ctypes.c_float), ("x_tilde_shared", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class CacheKey(ctypes.Structure):
    _fields_ = [("user_id", ctypes.c_uint64), ("model_version", ctypes.c_uint32), ("sketch_config", ctypes.c_uint32),
                ("history_timestamp", ctypes.c_int64)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_sets", ctypes.c_int32), ("ways", ctypes.c_int32), ("row_floats", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("ttl", ctypes.c_int64)]


class SkaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        detail = ""
        if code == SKA_ERR_CUDA and _lib is not None:
            detail = " [" + _lib.ska_last_error_string().decode() + "]"
        super().__init__(f"{what}: {status_string(code)} ({code}){detail}")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libska.so; raise loudly if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sketch_attention_flashsa_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    vp, sz, i32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
    L.sa_forward_workspace_size.argtypes = [ctypes.POINTER(SaDesc)]
    L.sa_forward_workspace_size.restype = sz
    L.sa_forward.argtypes = [ctypes.POINTER(SaDesc), vp, vp, vp, i32p, i32p, vp, vp, vp, vp, sz, vp]
    L.sa_forward.restype = ctypes.c_int
    L.sa_backward_workspace_size.argtypes = [ctypes.POINTER(SaDesc)]
    L.sa_backward_workspace_size.restype = sz
    L.sa_backward.argtypes = [ctypes.POINTER(SaDesc), vp, vp, vp, i32p, i32p, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.sa_backward.restype = ctypes.c_int
    L.stca_forward_workspace_size.argtypes = [ctypes.POINTER(StcaDesc)]
    L.stca_forward_workspace_size.restype = sz
    L.stca_forward.argtypes = [ctypes.POINTER(StcaDesc), vp, i32p, vp, vp, i32p, i32p, vp, vp, vp, vp, vp, sz, vp]
    L.stca_forward.restype = ctypes.c_int
    L.ska_last_error_string.argtypes = []
    L.ska_last_error_string.restype = ctypes.c_char_p
    L.ska_status_string.argtypes = [ctypes.c_int]
    L.ska_status_string.restype = ctypes.c_char_p
    L.ska_read_device_status.argtypes = [vp, vp]
    L.ska_read_device_status.restype = ctypes.c_int
    L.ska_set_debug.argtypes = [ctypes.c_uint64, ctypes.c_uint32]
    L.ska_set_debug.restype = None
    L.sa_forward_noalloc.argtypes = [ctypes.POINTER(SaDesc), vp, vp, vp, i32p, i32p, vp, vp, vp, vp]
    L.sa_forward_noalloc.restype = ctypes.c_int
    L.sa_forward_noalloc_scratch_bytes.argtypes = []
    L.sa_forward_noalloc_scratch_bytes.restype = sz
    L.sa_forward_noalloc_read_status.argtypes = [vp]
    L.sa_forward_noalloc_read_status.restype = ctypes.c_int
    L.sa_cache_bytes.argtypes = [ctypes.POINTER(CacheDesc)]
    L.sa_cache_bytes.restype = sz
    L.sa_cache_init.argtypes = [ctypes.POINTER(CacheDesc), vp, sz, vp]
    L.sa_cache_init.restype = ctypes.c_int
    L.sa_cache_put.argtypes = [ctypes.POINTER(CacheDesc), vp, sz, vp, vp, ctypes.c_int32, ctypes.c_int64, vp, vp]
    L.sa_cache_put.restype = ctypes.c_int
    L.sa_cache_get.argtypes = [ctypes.POINTER(CacheDesc), vp, sz, vp, ctypes.c_int32, ctypes.c_int64, vp, vp, vp]
    L.sa_cache_get.restype = ctypes.c_int
    L.sa_forward_diag.argtypes = [ctypes.POINTER(SaDesc), vp, vp, vp, i32p, i32p, vp, vp, vp, vp, ctypes.c_int32,
                                  vp, sz, vp]
    L.sa_forward_diag.restype = ctypes.c_int
    L.sa_weight_histogram.argtypes = [vp, ctypes.c_int64, ctypes.c_int32, vp, vp]
    L.sa_weight_histogram.restype = ctypes.c_int
    L.stca_backward_workspace_size.argtypes = [ctypes.POINTER(StcaDesc)]
    L.stca_backward_workspace_size.restype = sz
    L.stca_backward.argtypes = [ctypes.POINTER(StcaDesc)] + [vp] * 17 + [sz, vp]
    L.stca_backward.restype = ctypes.c_int
    L.sa_refine_workspace_size.argtypes = [ctypes.POINTER(RefineDesc)]
    L.sa_refine_workspace_size.restype = sz
    L.sa_refine.argtypes = [ctypes.POINTER(RefineDesc)] + [vp] * 15 + [sz, vp]
    L.sa_refine.restype = ctypes.c_int
    L.sa_project_queries.argtypes = [ctypes.c_int32] * 4 + [vp] * 4 + [sz, vp]
    L.sa_project_queries.restype = ctypes.c_int
    L.ska_set_timing_events.argtypes = [vp, vp]
    L.ska_set_timing_events.restype = None
    _lib = L
    return L


def status_string(code: int) -> str:
    return lib().ska_status_string(code).decode()
