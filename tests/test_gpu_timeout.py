"""Failure detection on the GPU without a fault: a bounded mbarrier wait that nothing
completes gives up after its poll limit and sets the device status word, which
gla_check_device_status reports as GLA_ERR_TIMEOUT; the context stays usable afterwards."""
import ctypes

import pytest
import torch

from linear_rnn_b200 import _lib
from linear_rnn_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_bounded_wait_times_out_and_the_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert _lib.lib.gla_debug_wait_timeout(ptr(ws), 2000, stream()) == _lib.GLA_OK
    assert _lib.lib.gla_check_device_status(ptr(ws), stream()) == _lib.GLA_ERR_TIMEOUT
    # a normal call on the same context runs and leaves a clean status
    from linear_rnn_b200 import ops
    w = I.small(I.WORKLOADS["c3"])
    x = {k: (None if v is None else v.cuda()) for k, v in I.make_inputs(w, seed=3).items()}
    prob = ops.make_problem(x["q"], x["v"], x["g"], scale=w.scale, chunk=w.chunk, plan="tc")
    wsb = torch.empty(ops.gla_workspace_bytes(prob, False), dtype=torch.uint8, device="cuda")
    o, _ = ops.gla_fwd(x["q"], x["k"], x["v"], x["g"], scale=w.scale, chunk=w.chunk, plan="tc", workspace=wsb)
    assert ops.gla_check_device_status(wsb) == _lib.GLA_OK
    assert torch.isfinite(o.float()).all()
