"""ctypes view of the C ABI declared in include/gla.h (libgla_b200.so).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels. If the library is missing this module raises at import; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgla_b200.so")

GLA_OK, GLA_ERR_INVALID_ARG, GLA_ERR_UNSUPPORTED, GLA_ERR_WORKSPACE, GLA_ERR_CUDA, GLA_ERR_TIMEOUT, GLA_ERR_RANGE = range(7)
GLA_F32, GLA_BF16 = 0, 1
GLA_GATE_NONE, GLA_GATE_PER_KEY, GLA_GATE_PER_HEAD = 0, 1, 2
GLA_PLAN_AUTO, GLA_PLAN_SIMT, GLA_PLAN_TC = 0, 1, 2

# Every symbol include/gla.h declares (checked by tests/test_abi_symbols.py).
EXPORTED = ("gla_workspace_bytes", "gla_fwd", "gla_bwd", "gla_status_string",
            "gla_check_device_status", "gla_version", "gla_launch_count", "gla_profiler_enable",
            "gla_profiler_read", "gla_fwd_static_scratch", "gla_last_error_detail", "gla_plan_info",
            "gla_saved_states_bytes", "gla_fwd_save", "gla_bwd_saved", "gla_debug_wait_timeout",
            "gla_decode", "gla_shard_state", "gla_state_fold", "gla_shard_state_grad", "gla_deltanet_fwd",
            "gla_deltanet_bwd_workspace_bytes", "gla_deltanet_bwd", "gla_mlstm_workspace_bytes", "gla_mlstm_fwd",
            "gla_mlstm_bwd", "gla_shard_workspace_bytes", "gla_deltanet_saved_bytes", "gla_deltanet_fwd_save",
            "gla_deltanet_bwd_saved", "gla_mlstm_saved_bytes", "gla_mlstm_fwd_save", "gla_mlstm_bwd_saved")


class GlaProblem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int),
                ("Dk", ctypes.c_int), ("Dv", ctypes.c_int), ("chunk", ctypes.c_int),
                ("scale", ctypes.c_float), ("io", ctypes.c_int), ("gate", ctypes.c_int),
                ("plan", ctypes.c_int)]


class GlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status == GLA_ERR_CUDA:
            try:
                detail = " -- " + lib.gla_last_error_detail().decode()
            except Exception:
                pass
        super().__init__(f"{where}: {status_string(status)} (status {status}){detail}")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"CUDA library {LIB_PATH} is missing; build it with `python -m linear_rnn_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, fp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
    pp = ctypes.POINTER(GlaProblem)
    lib.gla_workspace_bytes.argtypes = [pp, ctypes.c_int]
    lib.gla_workspace_bytes.restype = sz
    lib.gla_fwd.argtypes = [pp, vp, vp, vp, fp, fp, fp, vp, fp, vp, sz, vp]
    lib.gla_fwd.restype = ctypes.c_int
    lib.gla_bwd.argtypes = [pp, vp, vp, vp, fp, fp, fp, vp, fp, vp, vp, vp, fp, fp, fp, vp, sz, vp]
    lib.gla_bwd.restype = ctypes.c_int
    lib.gla_saved_states_bytes.argtypes = [pp]
    lib.gla_saved_states_bytes.restype = sz
    lib.gla_fwd_save.argtypes = [pp, vp, vp, vp, fp, fp, fp, vp, fp, fp, vp, sz, vp]
    lib.gla_fwd_save.restype = ctypes.c_int
    lib.gla_bwd_saved.argtypes = [pp, vp, vp, vp, fp, fp, fp, vp, fp, fp, vp, vp, vp, fp, fp, fp, vp, sz, vp]
    lib.gla_bwd_saved.restype = ctypes.c_int
    lib.gla_status_string.argtypes = [ctypes.c_int]
    lib.gla_status_string.restype = ctypes.c_char_p
    lib.gla_check_device_status.argtypes = [vp, vp]
    lib.gla_check_device_status.restype = ctypes.c_int
    lib.gla_version.argtypes = []
    lib.gla_version.restype = ctypes.c_int
    lib.gla_last_error_detail.argtypes = []
    lib.gla_last_error_detail.restype = ctypes.c_char_p
    lib.gla_fwd_static_scratch.argtypes = [pp, vp, vp, vp, fp, fp, fp, vp, fp, vp]
    lib.gla_fwd_static_scratch.restype = ctypes.c_int
    ip = ctypes.POINTER(ctypes.c_int)
    lib.gla_plan_info.argtypes = [pp, ctypes.c_int, ip, ip, ip]
    lib.gla_plan_info.restype = ctypes.c_int
    lib.gla_shard_workspace_bytes.argtypes = [pp]
    lib.gla_shard_workspace_bytes.restype = ctypes.c_size_t
    lib.gla_shard_state.argtypes = [pp] + [ctypes.c_void_p] * 7 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_shard_state.restype = ctypes.c_int
    lib.gla_shard_state_grad.argtypes = [pp] + [ctypes.c_void_p] * 6 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_shard_state_grad.restype = ctypes.c_int
    lib.gla_deltanet_fwd.argtypes = [pp] + [ctypes.c_void_p] * 8
    lib.gla_deltanet_fwd.restype = ctypes.c_int
    lib.gla_deltanet_bwd_workspace_bytes.argtypes = [pp]
    lib.gla_deltanet_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.gla_deltanet_bwd.argtypes = [pp] + [ctypes.c_void_p] * 13 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_deltanet_bwd.restype = ctypes.c_int
    lib.gla_deltanet_saved_bytes.argtypes = [pp]
    lib.gla_deltanet_saved_bytes.restype = ctypes.c_size_t
    lib.gla_deltanet_fwd_save.argtypes = [pp] + [ctypes.c_void_p] * 9
    lib.gla_deltanet_fwd_save.restype = ctypes.c_int
    lib.gla_deltanet_bwd_saved.argtypes = [pp] + [ctypes.c_void_p] * 14 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_deltanet_bwd_saved.restype = ctypes.c_int
    lib.gla_mlstm_workspace_bytes.argtypes = [pp, ctypes.c_int]
    lib.gla_mlstm_workspace_bytes.restype = ctypes.c_size_t
    lib.gla_mlstm_fwd.argtypes = [pp] + [ctypes.c_void_p] * 7 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_mlstm_fwd.restype = ctypes.c_int
    lib.gla_mlstm_bwd.argtypes = [pp] + [ctypes.c_void_p] * 12 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_mlstm_bwd.restype = ctypes.c_int
    lib.gla_mlstm_saved_bytes.argtypes = [pp]
    lib.gla_mlstm_saved_bytes.restype = ctypes.c_size_t
    lib.gla_mlstm_fwd_save.argtypes = [pp] + [ctypes.c_void_p] * 8 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_mlstm_fwd_save.restype = ctypes.c_int
    lib.gla_mlstm_bwd_saved.argtypes = [pp] + [ctypes.c_void_p] * 13 + [ctypes.c_size_t, ctypes.c_void_p]
    lib.gla_mlstm_bwd_saved.restype = ctypes.c_int
    lib.gla_state_fold.argtypes = [pp, ctypes.c_int] + [ctypes.c_void_p] * 5
    lib.gla_state_fold.restype = ctypes.c_int
    lib.gla_decode.argtypes = [pp] + [ctypes.c_void_p] * 8
    lib.gla_decode.restype = ctypes.c_int
    lib.gla_debug_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_uint, ctypes.c_void_p]
    lib.gla_debug_wait_timeout.restype = ctypes.c_int
    lib.gla_launch_count.argtypes = []
    lib.gla_launch_count.restype = ctypes.c_ulonglong
    lib.gla_profiler_enable.argtypes = [ctypes.c_int]
    lib.gla_profiler_enable.restype = ctypes.c_int
    lib.gla_profiler_read.argtypes = [ctypes.c_char_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                      ctypes.POINTER(ctypes.c_double), ctypes.c_int]
    lib.gla_profiler_read.restype = ctypes.c_int
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.gla_status_string(int(status)).decode()


def profiler_enable(on: bool) -> None:
    lib.gla_profiler_enable(int(on))


def profiler_read(max_kernels: int = 64):
    """{kernel name: (launches, total_ms)} of the events recorded since the last read."""
    stride = 64
    names = ctypes.create_string_buffer(stride * max_kernels)
    cnt = (ctypes.c_int * max_kernels)()
    ms = (ctypes.c_double * max_kernels)()
    n = lib.gla_profiler_read(names, stride, cnt, ms, max_kernels)
    if n < 0:
        raise RuntimeError("gla_profiler_read failed")
    return {names.raw[i * stride:(i + 1) * stride].split(b"\0")[0].decode(): (cnt[i], ms[i])
            for i in range(min(n, max_kernels))}


def launch_count() -> int:
    return int(lib.gla_launch_count())


def plan_info(problem: GlaProblem, for_backward: bool):
    """(plan, nseg, tiles_per_seg) that gla_fwd / gla_bwd would use; GlaError if invalid."""
    plan, nseg, tiles = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    st = lib.gla_plan_info(ctypes.byref(problem), int(for_backward), ctypes.byref(plan), ctypes.byref(nseg),
                           ctypes.byref(tiles))
    if st != GLA_OK:
        raise GlaError(st, "gla_plan_info")
    return plan.value, nseg.value, tiles.value
