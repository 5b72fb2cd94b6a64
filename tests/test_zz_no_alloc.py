"""The forward entry point that allocates nothing (gla_fwd_static_scratch).

Some callers cannot allocate device memory themselves (a host whose device memory is all
owned by another allocator, or code that must not call cudaMalloc because it
synchronises the device); this entry point takes its scratch from a fixed array inside
the library. The test calls it through the C ABI twice in a row and checks each result
against the ordinary gla_fwd (CUDA-core plan) within the parity tolerances, and that a
problem whose scratch would not fit is rejected. This file is collected last so that a
stop-at-first-failure run has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from linear_rnn_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _err(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_static_scratch_forward_matches_gla_fwd_twice(dtype):
    from linear_rnn_b200 import _lib, ops
    w = I.WORKLOADS["c3"].replace(B=1, H=2, L=300, Dk=64, Dv=128, dtype=dtype, h0_std=0.5)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        x = {k: (None if v is None else v.cuda()) for k, v in I.make_inputs(w, seed=20 + call).items()}
        o_ref, hT_ref = ops.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], scale=w.scale,
                                    chunk=w.chunk, plan="simt")
        p = ops.make_problem(x["q"], x["v"], x["g"], scale=w.scale, chunk=w.chunk, plan="simt")
        o = torch.full_like(o_ref, float("nan"))
        hT = torch.full_like(hT_ref, float("nan"))
        st = _lib.lib.gla_fwd_static_scratch(ctypes.byref(p), _ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]),
                                             _ptr(x["g"]), _ptr(x["igate"]), _ptr(x["h0"]), _ptr(o), _ptr(hT),
                                             stream)
        assert st == _lib.GLA_OK, _lib.status_string(st)
        torch.cuda.synchronize()
        assert _err(o, o_ref) <= TOL[dtype], call
        assert _err(hT, hT_ref) <= TOL[dtype], call


def test_static_scratch_rejects_oversized_problem():
    from linear_rnn_b200 import _lib, ops
    q = torch.zeros(2, 8, 8192, 128, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(2, 8, 8192, 256, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(2, 8, 8192, 128, device="cuda")
    o = torch.empty_like(v)
    p = ops.make_problem(q, v, g, scale=1.0, chunk=64, plan="simt")
    st = _lib.lib.gla_fwd_static_scratch(ctypes.byref(p), _ptr(q), _ptr(q), _ptr(v), _ptr(g), None, None, _ptr(o),
                                         None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.GLA_ERR_WORKSPACE
