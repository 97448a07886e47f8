"""ctypes loader for the in-tree CUDA library ``libasp.so`` (C ABI in
include/as_partition.h).  There is no fallback: if the library is missing or
fails to load, importing the binding raises."""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
# ASP_DEBUG=1 selects the checked build (device-side index checks)
CHECKED = os.environ.get("ASP_DEBUG", "0") == "1"
LIB_PATH = os.path.join(PKG, "libasp_debug.so" if CHECKED else "libasp.so")

AS_MAX_P = 64
AS_OK, AS_ERR_INVALID_ARG, AS_ERR_UNSUPPORTED, AS_ERR_CACHE_MISS, AS_ERR_CUDA, AS_ERR_TIMEOUT, AS_ERR_BOUNDS = range(7)
AS_F32, AS_BF16 = 0, 1
AS_PLAN_REUSE, AS_PLAN_FRESH, AS_PLAN_FRESH_STORE = 0, 1, 2

STATUS_NAMES = {
    AS_OK: "AS_OK", AS_ERR_INVALID_ARG: "AS_ERR_INVALID_ARG", AS_ERR_UNSUPPORTED: "AS_ERR_UNSUPPORTED",
    AS_ERR_CACHE_MISS: "AS_ERR_CACHE_MISS", AS_ERR_CUDA: "AS_ERR_CUDA", AS_ERR_TIMEOUT: "AS_ERR_TIMEOUT",
    AS_ERR_BOUNDS: "AS_ERR_BOUNDS",
}

# every entry point declared in include/as_partition.h
EXPORTS = ("as_last_error", "as_version", "as_partition_attn", "as_compose", "as_cache_bytes",
           "as_cache_init", "as_plan_resolve", "as_step", "as_device_status", "as_debug_timeout_probe",
           "as_debug_exp2", "as_planner_init", "as_planner_scratch_bytes", "as_local_states", "as_plan_drift",
           "as_plan_select", "as_planner_next", "as_planner_commit_anchor", "as_plan_drift_static",
           "as_cache_group_bytes", "as_cache_group_init", "as_planner_group_init", "as_plan_select_grouped",
           "as_step_local", "as_cache_cp_bytes", "as_cache_cp_init", "as_step_cp", "as_residual_encode",
           "as_residual_decode", "as_debug_bounds_probe")


class AsCacheStruct(ctypes.Structure):
    _fields_ = [
        ("magic", ctypes.c_uint32),
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("S", ctypes.c_int), ("d", ctypes.c_int), ("P", ctypes.c_int),
        ("cache_dt", ctypes.c_int),
        ("out_planes", ctypes.c_void_p),
        ("lse_planes", ctypes.c_void_p),
        ("t_c", ctypes.c_int32 * (AS_MAX_P * AS_MAX_P)),
        ("g", ctypes.c_int), ("n_groups", ctypes.c_int),
        ("member", ctypes.c_uint64 * (AS_MAX_P * AS_MAX_P)),
        ("q_first", ctypes.c_int), ("q_count", ctypes.c_int),
    ]


class AsPlannerStruct(ctypes.Structure):
    _fields_ = [
        ("magic", ctypes.c_uint32),
        ("P", ctypes.c_int), ("window", ctypes.c_int),
        ("reuse_ratio", ctypes.c_double), ("eps_local", ctypes.c_double),
        ("has_anchor", ctypes.c_int),
        ("w", ctypes.c_double * (AS_MAX_P * AS_MAX_P)),
        ("alpha", ctypes.c_double * (AS_MAX_P * AS_MAX_P)),
        ("drift", ctypes.c_double * AS_MAX_P),
        ("rel_drift", ctypes.c_double * AS_MAX_P),
        ("g", ctypes.c_int),
    ]


class AsError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m attention_state_reuse_partition_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    c_int, c_float, vp = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
    i64, u32, sz = ctypes.c_int64, ctypes.c_uint32, ctypes.c_size_t
    lib.as_last_error.restype = ctypes.c_char_p
    lib.as_last_error.argtypes = []
    lib.as_version.restype = ctypes.c_char_p
    lib.as_version.argtypes = []
    lib.as_partition_attn.restype = c_int
    lib.as_partition_attn.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, c_float,
                                      c_int, ctypes.POINTER(ctypes.c_int32), c_int, c_int, vp, vp, vp]
    lib.as_compose.restype = c_int
    lib.as_compose.argtypes = [vp, vp, c_int, i64, c_int, i64, i64, vp, vp, vp]
    lib.as_cache_bytes.restype = sz
    lib.as_cache_bytes.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int]
    lib.as_cache_init.restype = c_int
    lib.as_cache_init.argtypes = [ctypes.POINTER(AsCacheStruct), vp, sz, c_int, c_int, c_int, c_int, c_int, c_int]
    lib.as_cache_group_bytes.restype = sz
    lib.as_cache_group_bytes.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int, c_int]
    lib.as_cache_group_init.restype = c_int
    lib.as_cache_group_init.argtypes = [ctypes.POINTER(AsCacheStruct), vp, sz, c_int, c_int, c_int, c_int, c_int,
                                        c_int, c_int]
    lib.as_plan_resolve.restype = c_int
    lib.as_plan_resolve.argtypes = [ctypes.POINTER(AsCacheStruct), vp, c_int, vp, vp]
    lib.as_step.restype = c_int
    lib.as_step.argtypes = [ctypes.POINTER(AsCacheStruct), vp, vp, vp, c_int, c_float, vp, c_int, vp, vp,
                            vp, vp, vp]
    lib.as_step_local.restype = c_int
    lib.as_step_local.argtypes = [ctypes.POINTER(AsCacheStruct), vp, vp, vp, c_int, c_float, vp, c_int, vp, vp,
                                  vp, vp, vp, vp, vp]
    lib.as_cache_cp_bytes.restype = sz
    lib.as_cache_cp_bytes.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_int]
    lib.as_cache_cp_init.restype = c_int
    lib.as_cache_cp_init.argtypes = [ctypes.POINTER(AsCacheStruct), vp, sz, c_int, c_int, c_int, c_int, c_int,
                                     c_int, c_int, c_int, c_int]
    lib.as_debug_bounds_probe.restype = c_int
    lib.as_debug_bounds_probe.argtypes = [vp, ctypes.c_int64, vp]
    lib.as_residual_encode.restype = c_int
    lib.as_residual_encode.argtypes = [vp, vp, vp, vp, ctypes.c_int64, c_int, vp]
    lib.as_residual_decode.restype = c_int
    lib.as_residual_decode.argtypes = [vp, vp, vp, ctypes.c_int64, c_int, vp]
    lib.as_step_cp.restype = c_int
    lib.as_step_cp.argtypes = [ctypes.POINTER(AsCacheStruct), vp, vp, vp, c_int, vp, c_int, c_float, vp, c_int,
                               vp, vp, vp, vp, vp]
    lib.as_device_status.restype = c_int
    lib.as_device_status.argtypes = [vp, ctypes.POINTER(u32)]
    lib.as_debug_timeout_probe.restype = c_int
    lib.as_debug_timeout_probe.argtypes = [u32, u32, vp]
    dbl = ctypes.c_double
    lib.as_planner_init.restype = c_int
    lib.as_planner_init.argtypes = [ctypes.POINTER(AsPlannerStruct), c_int, c_int, dbl, dbl]
    lib.as_planner_group_init.restype = c_int
    lib.as_planner_group_init.argtypes = [ctypes.POINTER(AsPlannerStruct), c_int, c_int, c_int, dbl, dbl]
    lib.as_plan_select_grouped.restype = c_int
    lib.as_plan_select_grouped.argtypes = [vp, c_int, c_int, c_int, dbl, vp]
    lib.as_planner_scratch_bytes.restype = sz
    lib.as_planner_scratch_bytes.argtypes = [c_int, c_int, c_int]
    lib.as_local_states.restype = c_int
    lib.as_local_states.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, ctypes.c_float, vp, vp, vp]
    lib.as_plan_drift.restype = c_int
    lib.as_plan_drift.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, vp, sz, vp, vp, vp]
    lib.as_plan_drift_static.restype = c_int
    lib.as_plan_drift_static.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp, vp]
    lib.as_plan_select.restype = c_int
    lib.as_plan_select.argtypes = [vp, c_int, c_int, dbl, vp]
    lib.as_planner_next.restype = c_int
    lib.as_planner_next.argtypes = [ctypes.POINTER(AsPlannerStruct), vp, vp, c_int, c_int, c_int, c_int, vp, sz, vp,
                                    ctypes.POINTER(c_int), vp, vp]
    lib.as_planner_commit_anchor.restype = c_int
    lib.as_planner_commit_anchor.argtypes = [ctypes.POINTER(AsPlannerStruct), ctypes.POINTER(AsCacheStruct), vp, vp,
                                             vp, vp, sz, vp]
    lib.as_debug_exp2.restype = c_int
    lib.as_debug_exp2.argtypes = [vp, vp, i64, c_int, vp]
    return lib


LIB = _load()


def check(status: int) -> None:
    if status != AS_OK:
        raise AsError(status, LIB.as_last_error().decode())
