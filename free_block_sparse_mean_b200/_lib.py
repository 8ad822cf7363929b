"""ctypes loader for the C ABI in include/sparse_attn.h (libsparse_attn.so).

No fallback: if the library is missing the import of the calls fails loudly."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsparse_attn.so")

SA_OK = 0
SA_ERR_DEVICE_CHECK = 5
SA_FILTER_LAMBDA = 0
SA_FILTER_RECALL = 1
SA_HOST_FP8_SCORES = 1
SA_HOST_INT8_SCORES = 2
STATUS_NAMES = {
    0: "SA_OK",
    1: "SA_ERR_INVALID_ARG",
    2: "SA_ERR_UNSUPPORTED",
    3: "SA_ERR_WORKSPACE",
    4: "SA_ERR_CUDA",
    5: "SA_ERR_DEVICE_CHECK",
}

# Every symbol include/sparse_attn.h declares.
EXPORTS = (
    "sparse_attn_plan_workspace_size",
    "sparse_attn_num_tiles",
    "sparse_attn_plan",
    "sparse_attn_plan_heads",
    "sparse_attn_fwd",
    "sparse_attn_status_string",
    "sparse_attn_device_error",
    "sparse_attn_plan_noalloc",
    "sparse_attn_plan_q8",
    "sparse_attn_fwd_q8",
    "sparse_attn_plan_i8",
    "sparse_attn_fwd_i8",
    "sparse_attn_fwd_recall",
    "sparse_attn_fwd_decisions",
    "sparse_attn_host_workspace_size",
    "sparse_attn_host",
    "sparse_attn_cluster_workspace_size",
    "sparse_attn_cluster",
    "sparse_attn_permute_rows",
    "sparse_attn_selftest_wait_timeout",
)


class SaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("block", ctypes.c_int32)]


class SparseAttnError(RuntimeError):
    def __init__(self, call: str, status: int, lib=None):
        msg = STATUS_NAMES.get(status, f"status {status}")
        if lib is not None:
            try:
                msg = lib.sparse_attn_status_string(status).decode()
            except Exception:  # pragma: no cover - message only
                pass
        super().__init__(f"{call} failed: {msg}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH):
    """Load the shared library once and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"CUDA library not built: {path} is missing (run __graft_entry__.build() or "
            "python -m free_block_sparse_mean_b200.build)")
    lib = ctypes.CDLL(path)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    lib.sparse_attn_plan_workspace_size.argtypes = [SaShape]
    lib.sparse_attn_plan_workspace_size.restype = sz
    lib.sparse_attn_num_tiles.argtypes = [SaShape]
    lib.sparse_attn_num_tiles.restype = ctypes.c_int64
    lib.sparse_attn_plan.argtypes = [vp, vp, SaShape, f32, f32, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.sparse_attn_plan.restype = i32
    lib.sparse_attn_plan_heads.argtypes = [vp, vp, SaShape, vp, f32, i32, vp, vp, vp, vp, vp, sz, vp]
    lib.sparse_attn_plan_heads.restype = i32
    lib.sparse_attn_fwd.argtypes = [vp, vp, vp, SaShape, vp, vp, f32, f32, i32, vp, vp, vp]
    lib.sparse_attn_fwd.restype = i32
    lib.sparse_attn_status_string.argtypes = [i32]
    lib.sparse_attn_status_string.restype = ctypes.c_char_p
    lib.sparse_attn_device_error.argtypes = [vp, ctypes.POINTER(i32)]
    lib.sparse_attn_device_error.restype = i32
    lib.sparse_attn_plan_noalloc.argtypes = [vp, vp, SaShape, f32, f32, i32, vp, vp, vp, vp, vp]
    lib.sparse_attn_plan_noalloc.restype = i32
    lib.sparse_attn_plan_q8.argtypes = [vp, vp, SaShape, f32, f32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sparse_attn_plan_q8.restype = i32
    lib.sparse_attn_fwd_q8.argtypes = [vp, vp, vp, vp, vp, SaShape, vp, vp, f32, f32, i32, vp, vp, vp]
    lib.sparse_attn_fwd_q8.restype = i32
    lib.sparse_attn_plan_i8.argtypes = lib.sparse_attn_plan_q8.argtypes
    lib.sparse_attn_plan_i8.restype = i32
    lib.sparse_attn_fwd_i8.argtypes = lib.sparse_attn_fwd_q8.argtypes
    lib.sparse_attn_fwd_i8.restype = i32
    lib.sparse_attn_fwd_recall.argtypes = [vp, vp, vp, SaShape, vp, vp, f32, f32, i32, vp, vp, vp]
    lib.sparse_attn_fwd_recall.restype = i32
    lib.sparse_attn_fwd_decisions.argtypes = [vp, vp, vp, SaShape, vp, vp, i32, f32, f32, i32, vp, vp, vp, vp]
    lib.sparse_attn_fwd_decisions.restype = i32
    lib.sparse_attn_host_workspace_size.argtypes = [SaShape, i32, i32]
    lib.sparse_attn_host_workspace_size.restype = sz
    lib.sparse_attn_host.argtypes = [vp, vp, vp, SaShape, f32, vp, i32, f32, f32, i32, i32, vp, vp, sz, i32, vp, vp, vp]
    lib.sparse_attn_host.restype = i32
    lib.sparse_attn_cluster_workspace_size.argtypes = [SaShape]
    lib.sparse_attn_cluster_workspace_size.restype = sz
    lib.sparse_attn_cluster.argtypes = [vp, vp, SaShape, i32, vp, vp, vp, vp, sz, vp]
    lib.sparse_attn_cluster.restype = i32
    lib.sparse_attn_permute_rows.argtypes = [vp, vp, SaShape, i32, vp, vp]
    lib.sparse_attn_permute_rows.restype = i32
    lib.sparse_attn_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
    lib.sparse_attn_selftest_wait_timeout.restype = i32
    _lib = lib
    return lib
