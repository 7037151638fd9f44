"""ctypes binding of ``libmoe_b200.so`` (the C ABI in ``include/moe.h``).

Argument marshalling only: every step of the forward pass runs in the
library's CUDA kernels. torch is used for device memory and the current
stream. There is no fallback: if the library or a GPU is missing, the calls
raise.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_WORKSPACE = 0, 1, 2, 3, 6
MOE_DEV_TIMEOUT, MOE_DEV_NONFINITE, MOE_DEV_INTERNAL = 0x1, 0x2, 0x4
MOE_F32, MOE_BF16 = 0, 1

STATUS_NAMES = {
    MOE_OK: "MOE_OK",
    MOE_ERR_INVALID_ARG: "MOE_ERR_INVALID_ARG",
    MOE_ERR_UNSUPPORTED: "MOE_ERR_UNSUPPORTED",
    MOE_ERR_CUDA: "MOE_ERR_CUDA",
    MOE_ERR_WORKSPACE: "MOE_ERR_WORKSPACE",
}

EXPORTED = ("moe_workspace_size", "moe_forward", "moe_forward_events", "moe_kernel_name", "moe_get_permutation",
            "moe_last_error_detail", "moe_forward_noalloc", "moe_selftest_wait_timeout", "moe_workspace_size_ex",
            "moe_forward_ex", "moe_launch_plan", "moe_pipeline_create", "moe_pipeline_submit",
            "moe_pipeline_synchronize", "moe_pipeline_stream", "moe_pipeline_destroy")
MOE_NORM_NONE, MOE_NORM_RMS, MOE_NORM_RMS_EPS_OUTSIDE = 0, 1, 2
MOE_MAX_SHARED = 8
MOE_NOALLOC_SCRATCH_BYTES = 16 << 20
MOE_NUM_KERNELS = 6
MOE_PLAN_FUSED_COMBINE, MOE_PLAN_FUSED_GEMMS, MOE_PLAN_ROUTER_WEIGHT_SPLIT, MOE_PLAN_FUSED_SCAN = 1, 2, 4, 8
MOE_PLAN_PERMUTE_SCAN = 16


class moe_options(ctypes.Structure):
    """The C struct ``moe_options`` of include/moe.h (same field order and types)."""

    _fields_ = [
        ("struct_bytes", ctypes.c_size_t),
        ("norm_form", ctypes.c_int),
        ("norm_eps", ctypes.c_float),
        ("norm_weight", ctypes.c_void_p),
        ("n_shared", ctypes.c_int),
        ("shared_gate", ctypes.c_void_p),
        ("shared_up", ctypes.c_void_p),
        ("shared_down", ctypes.c_void_p),
        ("capacity_factor", ctypes.c_double),
        ("dropped", ctypes.c_void_p),
        ("z_loss", ctypes.c_void_p),
        ("fold_combine", ctypes.c_int),
    ]


MOE_PIPELINE_COPY_IN, MOE_PIPELINE_COMPUTE, MOE_PIPELINE_COPY_OUT = 0, 1, 2


class moe_layer_desc(ctypes.Structure):
    """The C struct ``moe_layer_desc`` of include/moe.h (same field order and types)."""

    _fields_ = [
        ("struct_bytes", ctypes.c_size_t),
        ("w_router", ctypes.c_void_p),
        ("b_router", ctypes.c_void_p),
        ("w_gate", ctypes.c_void_p),
        ("w_up", ctypes.c_void_p),
        ("w_down", ctypes.c_void_p),
        ("T", ctypes.c_int), ("d", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int), ("I", ctypes.c_int),
        ("renorm", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("opt", ctypes.POINTER(moe_options)),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
        ("topk_idx", ctypes.c_void_p),
        ("topk_gate", ctypes.c_void_p),
        ("counts", ctypes.c_void_p),
        ("status_dev", ctypes.c_void_p),
        ("x_dev", ctypes.c_void_p * 2),
        ("out_dev", ctypes.c_void_p * 2),
        ("aux_dev", ctypes.c_void_p * 2),
    ]


class MoEError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {detail}")
        self.status = status
        self.detail = detail


_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load the CUDA library (once). Raises if it has not been built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"{p} is missing: build it with `python -m sparse_mixture_experts_renorm_b200.build` "
            "(there is no non-CUDA fallback)"
        )
    lib = ctypes.CDLL(p)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.moe_workspace_size.argtypes = [I32, I32, I32, I32, I32, I32]
    lib.moe_workspace_size.restype = SZ
    lib.moe_forward.argtypes = [P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, P, P, P, P, P, P, SZ, P, P]
    lib.moe_forward.restype = I32
    lib.moe_forward_events.argtypes = lib.moe_forward.argtypes + [ctypes.POINTER(ctypes.c_void_p), I32]
    lib.moe_forward_events.restype = I32
    OPT = ctypes.POINTER(moe_options)
    lib.moe_workspace_size_ex.argtypes = [I32, I32, I32, I32, I32, I32, OPT]
    lib.moe_workspace_size_ex.restype = SZ
    lib.moe_forward_ex.argtypes = ([P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, OPT, P, P, P, P, P, P, SZ, P,
                                    P, ctypes.POINTER(ctypes.c_void_p), I32])
    lib.moe_forward_ex.restype = I32
    lib.moe_launch_plan.argtypes = [I32, I32, I32, I32, I32, I32, OPT]
    lib.moe_launch_plan.restype = I32
    lib.moe_pipeline_create.argtypes = [ctypes.POINTER(moe_layer_desc), P, ctypes.POINTER(ctypes.c_void_p)]
    lib.moe_pipeline_create.restype = I32
    lib.moe_pipeline_submit.argtypes = [P, P, P, P]
    lib.moe_pipeline_submit.restype = I32
    lib.moe_pipeline_synchronize.argtypes = [P]
    lib.moe_pipeline_synchronize.restype = I32
    lib.moe_pipeline_stream.argtypes = [P, I32]
    lib.moe_pipeline_stream.restype = P
    lib.moe_pipeline_destroy.argtypes = [P]
    lib.moe_pipeline_destroy.restype = I32
    lib.moe_kernel_name.argtypes = [I32]
    lib.moe_kernel_name.restype = ctypes.c_char_p
    lib.moe_forward_noalloc.argtypes = [P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, P, P, P, P, P, P, P]
    lib.moe_forward_noalloc.restype = I32
    lib.moe_selftest_wait_timeout.argtypes = [P, ctypes.c_longlong, P]
    lib.moe_selftest_wait_timeout.restype = I32
    lib.moe_get_permutation.argtypes = [P, SZ, I32, I32, I32, I32, I32, I32, P, P, P, P]
    lib.moe_get_permutation.restype = I32
    lib.moe_last_error_detail.argtypes = [ctypes.c_char_p, SZ]
    lib.moe_last_error_detail.restype = SZ
    if path is None:
        _lib = lib
    return lib


def last_error_detail(lib=None) -> str:
    lib = lib or load_library()
    buf = ctypes.create_string_buffer(1024)
    lib.moe_last_error_detail(buf, len(buf))
    return buf.value.decode()


def kernel_names(lib=None) -> list[str]:
    lib = lib or load_library()
    return [lib.moe_kernel_name(i).decode() for i in range(MOE_NUM_KERNELS)]


def check(status: int, lib=None) -> None:
    if status != MOE_OK:
        raise MoEError(status, last_error_detail(lib))
