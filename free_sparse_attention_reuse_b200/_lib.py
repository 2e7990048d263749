"""ctypes binding of libmcs.so (the C ABI in include/mcs.h).

Argument marshalling only: torch tensors are checked for device/dtype/contiguity and passed
as raw device pointers with torch's current CUDA stream.  Every step of the computation runs
in the library's CUDA kernels; there is no CPU or PyTorch fallback, and a missing library
raises at load time.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmcs.so")

EXPORTS = (
    "mcs_abi_version",
    "mcs_status_string",
    "mcs_workspace_size",
    "mcs_dense_attn",
    "mcs_group",
    "mcs_select",
    "mcs_select_noalloc",
    "mcs_sparse_attn",
    "mcs_residual",
    "mcs_anchor",
    "mcs_sync_status",
    "mcs_select_blocks",
    "mcs_perquery_workspace_size",
    "mcs_perquery_attn",
    "mcs_host_staging_size",
    "mcs_sparse_attn_host",
    "mcs_set_attn_wait_limit",
    "mcs_kmeans_workspace_size",
    "mcs_group_kmeans",
)

STATUS_NAMES = {
    0: "MCS_OK",
    1: "MCS_ERR_INVALID_ARG",
    2: "MCS_ERR_SHAPE",
    3: "MCS_ERR_DTYPE_ALIGN",
    4: "MCS_ERR_UNSUPPORTED_ARCH",
    5: "MCS_ERR_CUDA",
    6: "MCS_ERR_BAD_INDEX",
    7: "MCS_ERR_TIMEOUT",
    8: "MCS_ERR_WORKSPACE",
}


class MCSError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int), ("d", ctypes.c_int),
                ("scale", ctypes.c_float)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmcs.so once; raises if it is missing (build it with build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libmcs.so not found at {path}: run free_sparse_attention_reuse_b200/build.py")
    lib = ctypes.CDLL(path)
    vp, i32p = ctypes.c_void_p, ctypes.c_void_p
    lib.mcs_abi_version.restype = ctypes.c_int
    lib.mcs_abi_version.argtypes = []
    lib.mcs_status_string.restype = ctypes.c_char_p
    lib.mcs_status_string.argtypes = [ctypes.c_int]
    lib.mcs_workspace_size.restype = ctypes.c_size_t
    lib.mcs_workspace_size.argtypes = [Shape, ctypes.c_int, ctypes.c_int]
    lib.mcs_dense_attn.restype = ctypes.c_int
    lib.mcs_dense_attn.argtypes = [Shape, vp, vp, vp, vp, vp, vp]
    lib.mcs_group.restype = ctypes.c_int
    lib.mcs_group.argtypes = [Shape, vp, ctypes.c_int, i32p, vp, ctypes.c_size_t, vp]
    lib.mcs_select.restype = ctypes.c_int
    lib.mcs_select.argtypes = [Shape, vp, vp, i32p, ctypes.c_int, ctypes.c_int, vp, i32p, vp, ctypes.c_size_t, vp]
    lib.mcs_select_noalloc.restype = ctypes.c_int
    lib.mcs_select_noalloc.argtypes = [Shape, vp, vp, i32p, ctypes.c_int, ctypes.c_int, vp, i32p, vp]
    lib.mcs_sparse_attn.restype = ctypes.c_int
    lib.mcs_sparse_attn.argtypes = [Shape, vp, vp, vp, i32p, ctypes.c_int, i32p, ctypes.c_int, vp, vp, vp]
    lib.mcs_residual.restype = ctypes.c_int
    lib.mcs_residual.argtypes = [Shape, vp, vp, vp, i32p, ctypes.c_int, i32p, ctypes.c_int, vp, vp, vp]
    lib.mcs_anchor.restype = ctypes.c_int
    lib.mcs_anchor.argtypes = [Shape, vp, vp, vp, ctypes.c_int, ctypes.c_int, vp, i32p, i32p, vp, vp,
                               ctypes.c_size_t, vp]
    lib.mcs_sync_status.restype = ctypes.c_int
    lib.mcs_sync_status.argtypes = [vp]
    lib.mcs_select_blocks.restype = ctypes.c_int
    lib.mcs_select_blocks.argtypes = [Shape, vp, vp, i32p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp,
                                      i32p, vp, ctypes.c_size_t, vp]
    lib.mcs_perquery_workspace_size.restype = ctypes.c_size_t
    lib.mcs_perquery_workspace_size.argtypes = [Shape]
    lib.mcs_perquery_attn.restype = ctypes.c_int
    lib.mcs_perquery_attn.argtypes = [Shape, vp, vp, vp, ctypes.c_int, vp, vp, ctypes.c_size_t, vp]
    lib.mcs_host_staging_size.restype = ctypes.c_size_t
    lib.mcs_host_staging_size.argtypes = [Shape, ctypes.c_int]
    lib.mcs_sparse_attn_host.restype = ctypes.c_int
    lib.mcs_sparse_attn_host.argtypes = [Shape, vp, vp, vp, i32p, ctypes.c_int, i32p, ctypes.c_int, vp, vp,
                                         ctypes.c_int, vp, ctypes.c_size_t, vp]
    lib.mcs_kmeans_workspace_size.restype = ctypes.c_size_t
    lib.mcs_kmeans_workspace_size.argtypes = [Shape, ctypes.c_int]
    lib.mcs_group_kmeans.restype = ctypes.c_int
    lib.mcs_group_kmeans.argtypes = [Shape, vp, ctypes.c_int, ctypes.c_int, i32p, vp, ctypes.c_size_t, vp]
    lib.mcs_set_attn_wait_limit.restype = ctypes.c_uint64
    lib.mcs_set_attn_wait_limit.argtypes = [ctypes.c_uint64, vp]
    _lib = lib
    return lib


def check(status: int, what: str):
    if status != 0:
        raise MCSError(status, f"{what}: {load().mcs_status_string(status).decode()}")


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def stream_ptr():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
