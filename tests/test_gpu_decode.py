"""GPU parity of the recurrent single-token step (gla_decode) against the float64 oracle.

One step from a given state is the token recurrence over L = 1 with h0 = the state: the
oracle's forward on that token gives o and the new state. Same bound as the chunkwise path:
max|x - x_ref| / max|x_ref| <= 1e-2 for bf16 I/O, 1e-4 for fp32 I/O.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def err(got, ref):
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def step_case(w, seed):
    from linear_rnn_b200 import ops
    x = I.make_inputs(w.replace(L=1), seed=seed)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    state = xd["h0"].clone()
    o = ops.gla_decode(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], state, scale=w.scale)
    ro, rS = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], w.scale)
    return err(f64(o), ro), err(f64(state), rS)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 256), (256, 128), (256, 256), (64, 256)])
@pytest.mark.parametrize("gate,ig", [(I.GATE_PER_KEY, False), (I.GATE_PER_HEAD, True), (I.GATE_NONE, False)])
def test_decode_step_matches_oracle(dtype, Dk, Dv, gate, ig):
    w = I.WORKLOADS["c3"].replace(B=2, H=3, Dk=Dk, Dv=Dv, dtype=dtype, gate=gate, input_gate=ig, h0_std=0.5,
                                  gate_mean=3.0 if gate == I.GATE_PER_HEAD else 0.0,
                                  gate_div=1.0 if gate == I.GATE_PER_HEAD else 16.0)
    eo, es = step_case(w, 31)
    assert eo <= TOL[dtype] and es <= TOL[dtype], (eo, es)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_steps_equal_the_chunkwise_forward(dtype):
    """L single-token steps from h0 reproduce the chunkwise forward over the L tokens."""
    from linear_rnn_b200 import ops
    L = 37
    w = I.WORKLOADS["c3"].replace(B=1, H=2, L=L, Dk=128, Dv=128, dtype=dtype, input_gate=True, h0_std=0.5)
    x = I.make_inputs(w, seed=32)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    ro, rS = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], w.scale)
    state = xd["h0"].clone()
    outs = []
    for t in range(L):
        sl = lambda a: None if a is None else a[:, :, t:t + 1].contiguous()
        outs.append(ops.gla_decode(sl(xd["q"]), sl(xd["k"]), sl(xd["v"]), sl(xd["g"]), sl(xd["igate"]), state,
                                   scale=w.scale))
    o = torch.cat(outs, dim=2)
    assert err(f64(o), ro) <= TOL[dtype]
    assert err(f64(state), rS) <= TOL[dtype]
    fo, fS = ops.gla_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], scale=w.scale)
    assert err(f64(o), f64(fo)) <= TOL[dtype] and err(f64(state), f64(fS)) <= TOL[dtype]


def test_decode_at_serving_batch_sampled_heads():
    """The measured decode workload (1024 heads, state 128 MiB): whole batch on the GPU,
    two heads recomputed by the oracle."""
    from linear_rnn_b200 import ops
    w = I.DECODE
    x = I.make_inputs(w, seed=0)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    state = xd["h0"].clone()
    o = ops.gla_decode(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], state, scale=w.scale)
    for flat in (5, 1000):
        b, h = divmod(flat, w.H)
        pick = lambda a: None if a is None else a[b:b + 1, h:h + 1].contiguous()
        ro, rS = oracle.gla_fwd(pick(x["q"]), pick(x["k"]), pick(x["v"]), pick(x["g"]), pick(x["igate"]),
                                pick(x["h0"]), w.scale)
        assert err(f64(o[b:b + 1, h:h + 1]), ro) <= TOL[w.dtype]
        assert err(f64(state[b:b + 1, h:h + 1]), rS) <= TOL[w.dtype]


def test_decode_empty_batch_and_rejects_multi_token():
    from linear_rnn_b200 import ops
    from linear_rnn_b200._lib import GlaError
    q = torch.zeros(0, 2, 1, 64, device="cuda")
    state = torch.zeros(0, 2, 64, 64, device="cuda")
    assert ops.gla_decode(q, q, q, None, None, state).shape == (0, 2, 1, 64)
    q2 = torch.zeros(1, 1, 2, 64, device="cuda")
    with pytest.raises(ValueError):
        ops.gla_decode(q2, q2, q2, None, None, torch.zeros(1, 1, 64, 64, device="cuda"))
