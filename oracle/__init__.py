"""Float64 CPU oracle for gated linear attention -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this
package. The CUDA library and its Python binding never import it.

It wraps the plain C recurrence in gla_oracle.c (token-by-token forward, and
back-propagation through time for the backward) through ctypes. Every array is
converted to float64 (bf16/fp32 inputs convert exactly), so comparisons measure the
kernel's error, not input rounding.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

from . import build as _build

GATE_NONE, GATE_PER_KEY, GATE_PER_HEAD = 0, 1, 2

_lib = None


def _load():
    global _lib
    if _lib is None:
        # ORACLE_LIB_OVERRIDE lets tests/test_oracle_mutants.py load a planted-mistake
        # build; everything else uses the oracle as stated.
        path = os.environ.get("ORACLE_LIB_OVERRIDE") or _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_gla_fwd.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int] + [dp] * 8 + [ctypes.c_int]
        lib.oracle_gla_fwd.restype = ctypes.c_int
        lib.oracle_gla_bwd.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double, ctypes.c_int] + [dp] * 14 + [ctypes.c_int]
        lib.oracle_gla_bwd.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return _load().oracle_num_threads()


def _f64(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _gate_mode(g, Dk_shape_len: int) -> int:
    if g is None:
        return GATE_NONE
    return GATE_PER_KEY if g.ndim == Dk_shape_len else GATE_PER_HEAD


def gla_fwd(q, k, v, g=None, igate=None, h0=None, scale: float = 1.0,
            nthreads: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """o [B,H,L,Dv], hT [B,H,Dk,Dv] in float64 by the token recurrence.
    g: None (alpha = 1), [B,H,L,Dk] (per key dim) or [B,H,L] (per head)."""
    q, k, v, g, igate, h0 = map(_f64, (q, k, v, g, igate, h0))
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    mode = _gate_mode(g, 4)
    o = np.empty((B, H, L, Dv), np.float64)
    hT = np.empty((B, H, Dk, Dv), np.float64)
    rc = _load().oracle_gla_fwd(B, H, L, Dk, Dv, float(scale), mode, _ptr(q), _ptr(k), _ptr(v),
                                _ptr(g), _ptr(igate), _ptr(h0), _ptr(o), _ptr(hT), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_gla_fwd rejected its arguments")
    return o, hT


def gla_bwd(q, k, v, g=None, igate=None, h0=None, dO=None, dhT=None, scale: float = 1.0,
            nthreads: int = 0):
    """Gradients by back-propagation through time, float64.
    Returns dict dq, dk, dv, dg (None if ungated), di (None without input gate), dh0."""
    q, k, v, g, igate, h0, dO, dhT = map(_f64, (q, k, v, g, igate, h0, dO, dhT))
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    mode = _gate_mode(g, 4)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    dg = np.empty_like(g) if g is not None else None
    di = np.empty((B, H, L), np.float64) if igate is not None else None
    dh0 = np.empty((B, H, Dk, Dv), np.float64)
    rc = _load().oracle_gla_bwd(B, H, L, Dk, Dv, float(scale), mode, _ptr(q), _ptr(k), _ptr(v),
                                _ptr(g), _ptr(igate), _ptr(h0), _ptr(dO), _ptr(dhT), _ptr(dq),
                                _ptr(dk), _ptr(dv), _ptr(dg), _ptr(di), _ptr(dh0), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_gla_bwd rejected its arguments")
    return {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "di": di, "dh0": dh0}


def run_workload_inputs(inputs, scale: float, backward: bool, nthreads: int = 0):
    """Convenience: forward (and backward) of an inputs dict from linear_rnn_b200.inputs."""
    o, hT = gla_fwd(inputs["q"], inputs["k"], inputs["v"], inputs["g"], inputs["igate"],
                    inputs["h0"], scale, nthreads)
    out = {"o": o, "hT": hT}
    if backward:
        out.update(gla_bwd(inputs["q"], inputs["k"], inputs["v"], inputs["g"], inputs["igate"],
                           inputs["h0"], inputs["dO"], inputs.get("dhT"), scale, nthreads))
    return out
