"""GPU parity of the tensor-core (tcgen05) plan against the float64 oracle.

Covers the single-pass plan (enough (batch*head, Dv tile) pairs to fill the GPU) and
the segmented plan (few heads: segment states, scan, output pass), ragged tails, head
dims, gate modes, the input gate, initial and final states. bf16 I/O, bound 1e-2 on the
max-normalised error of every output.
"""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def f64(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def err(got, ref):
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30))


def run_tc_fwd(w, seed, plan="tc"):
    from linear_rnn_b200 import ops
    x = I.make_inputs(w, seed=seed)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    o, hT = ops.gla_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], scale=w.scale, chunk=w.chunk,
                        plan=plan)
    ro, rhT = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], w.scale)
    return err(f64(o), ro), err(f64(hT), rhT)


def base(**kw):
    w = I.WORKLOADS["c3"].replace(dtype="bf16", backward=False, chunk=64)
    return w.replace(**kw)


@pytest.mark.parametrize("L", [1, 40, 64, 65, 200, 1000])
def test_tc_segmented_ragged(L):
    w = base(B=1, H=2, L=L, Dk=128, Dv=128, h0_std=0.5)
    eo, eh = run_tc_fwd(w, 11)
    assert eo <= TOL and eh <= TOL, (eo, eh)


@pytest.mark.parametrize("L", [64, 130, 700])
def test_tc_single_pass(L):
    # 4*32 heads x 1 Dv tile = 128 CTAs: one pass per (head, Dv tile)
    w = base(B=4, H=32, L=L, Dk=64, Dv=64, h0_std=0.3)
    eo, eh = run_tc_fwd(w, 12)
    assert eo <= TOL and eh <= TOL, (eo, eh)


@pytest.mark.parametrize("Dk,Dv", [(64, 64), (64, 128), (128, 64), (128, 128), (128, 256), (256, 64), (256, 256),
                                   (64, 256)])
def test_tc_head_dims(Dk, Dv):
    w = base(B=1, H=3, L=333, Dk=Dk, Dv=Dv, h0_std=0.2)
    eo, eh = run_tc_fwd(w, 13)
    assert eo <= TOL and eh <= TOL, (eo, eh)


@pytest.mark.parametrize("gate,ig", [(I.GATE_NONE, False), (I.GATE_PER_HEAD, False), (I.GATE_PER_HEAD, True),
                                     (I.GATE_PER_KEY, True), (I.GATE_NONE, True)])
def test_tc_gate_modes(gate, ig):
    w = base(B=2, H=2, L=300, Dk=128, Dv=128, gate=gate, input_gate=ig, h0_std=0.4,
             gate_mean=3.0 if gate == I.GATE_PER_HEAD else 0.0, gate_div=1.0 if gate == I.GATE_PER_HEAD else 16.0)
    eo, eh = run_tc_fwd(w, 14)
    assert eo <= TOL and eh <= TOL, (eo, eh)


@pytest.mark.parametrize("chunk", [64, 128, 256, 1024])
def test_tc_chunk_sizes(chunk):
    w = base(B=1, H=2, L=2500, Dk=128, Dv=128, chunk=chunk, h0_std=0.3)
    eo, eh = run_tc_fwd(w, 15)
    assert eo <= TOL and eh <= TOL, (eo, eh)


def test_tc_rejects_fp32_and_odd_chunks():
    from linear_rnn_b200 import ops
    from linear_rnn_b200._lib import GlaError
    q = torch.zeros(1, 1, 64, 64, device="cuda")
    with pytest.raises(GlaError):
        ops.gla_fwd(q, q, q, None, scale=1.0, chunk=64, plan="tc")
    qb = q.bfloat16()
    with pytest.raises(GlaError):
        ops.gla_fwd(qb, qb, qb, None, scale=1.0, chunk=48, plan="tc")


def test_tc_matches_simt_plan():
    """Both GPU plans against each other (bf16 outputs; they round differently)."""
    from linear_rnn_b200 import ops
    w = base(B=2, H=4, L=513, Dk=128, Dv=128, h0_std=0.2)
    x = {k: (None if v is None else v.cuda()) for k, v in I.make_inputs(w, seed=16).items()}
    a = ops.gla_fwd(x["q"], x["k"], x["v"], x["g"], None, x["h0"], scale=w.scale, plan="tc")
    b = ops.gla_fwd(x["q"], x["k"], x["v"], x["g"], None, x["h0"], scale=w.scale, plan="simt")
    assert err(f64(a[0]), f64(b[0])) < 1e-2
    assert err(f64(a[1]), f64(b[1])) < 1e-2


def test_tc_deterministic():
    from linear_rnn_b200 import ops
    w = base(B=1, H=2, L=900, Dk=128, Dv=128)
    x = {k: (None if v is None else v.cuda()) for k, v in I.make_inputs(w, seed=17).items()}
    a = ops.gla_fwd(x["q"], x["k"], x["v"], x["g"], scale=w.scale, plan="tc")
    b = ops.gla_fwd(x["q"], x["k"], x["v"], x["g"], scale=w.scale, plan="tc")
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


# ------------------------------------------------------------- backward, Dk = 256
# The key dims split over a cluster of two CTAs; dv (and di, a per-head dg) combine the two
# blocks' partial sums through distributed shared memory.

def run_tc_bwd(w, seed, plan="tc", dhT=True):
    from linear_rnn_b200 import ops
    x = I.make_inputs(w, seed=seed)
    if dhT:
        x["dhT"] = I.make_dhT(w, seed)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    r = ops.gla_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], xd["dO"], xd.get("dhT"),
                    scale=w.scale, chunk=w.chunk, plan=plan)
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], x["dO"], x.get("dhT"), w.scale)
    errs = {}
    for n in ("dq", "dk", "dv", "dg", "di", "dh0"):
        if ref[n] is None:
            assert r[n] is None, n
            continue
        errs[n] = err(f64(r[n]), ref[n])
    return errs


@pytest.mark.parametrize("gate,ig", [(I.GATE_NONE, False), (I.GATE_PER_HEAD, True), (I.GATE_PER_HEAD, False),
                                     (I.GATE_PER_KEY, True), (I.GATE_PER_KEY, False)])
@pytest.mark.parametrize("Dv", [128, 256])
def test_tc_bwd_dk256_gate_modes(gate, ig, Dv):
    w = base(B=1, H=2, L=333, Dk=256, Dv=Dv, gate=gate, input_gate=ig, h0_std=0.3, backward=True,
             gate_mean=3.0 if gate == I.GATE_PER_HEAD else 0.0, gate_div=1.0 if gate == I.GATE_PER_HEAD else 16.0)
    errs = run_tc_bwd(w, 21)
    assert all(e <= TOL for e in errs.values()), errs


@pytest.mark.parametrize("L", [1, 64, 65, 1500])
def test_tc_bwd_dk256_lengths(L):
    # c5's variant (per-head forget gate, input gate); L = 1500 runs several segments
    w = I.WORKLOADS["c5"].replace(B=1, H=2, L=L, h0_std=0.2)
    errs = run_tc_bwd(w, 22)
    assert all(e <= TOL for e in errs.values()), errs


def test_tc_bwd_dk256_deterministic_and_matches_simt():
    """Two partial sums per dv element add the same way every call; the CUDA-core plan agrees."""
    from linear_rnn_b200 import ops
    w = I.WORKLOADS["c5"].replace(B=1, H=3, L=700)
    x = {k: (None if v is None else v.cuda()) for k, v in I.make_inputs(w, seed=23).items()}
    args = (x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], x["dO"], None)
    a = ops.gla_bwd(*args, scale=w.scale, chunk=w.chunk, plan="tc")
    b = ops.gla_bwd(*args, scale=w.scale, chunk=w.chunk, plan="tc")
    c = ops.gla_bwd(*args, scale=w.scale, chunk=w.chunk, plan="simt")
    for n in ("dq", "dk", "dv", "dg", "di"):
        assert torch.equal(a[n], b[n]), n
        assert err(f64(a[n]), f64(c[n])) < 1e-2, n


# ---------------------------------------------- forward state pass in finer sub-segments
# With few (head, Dv tile) pairs the forward's state pass runs R sub-segments per output
# segment (here R = 4 or 16) and the output pass starts from every R-th scanned state.

@pytest.mark.parametrize("Dk,Dv,chunk,gate,ig", [(256, 256, 256, I.GATE_PER_HEAD, True),
                                                 (256, 256, 256, I.GATE_PER_KEY, False),
                                                 (128, 128, 1024, I.GATE_PER_KEY, True),
                                                 (256, 128, 256, I.GATE_NONE, False)])
def test_tc_fwd_state_subsegments(Dk, Dv, chunk, gate, ig):
    w = base(B=1, H=1, L=2000 if chunk == 256 else 5000, Dk=Dk, Dv=Dv, chunk=chunk, gate=gate, input_gate=ig,
             h0_std=0.3, gate_mean=3.0 if gate == I.GATE_PER_HEAD else 0.0,
             gate_div=1.0 if gate == I.GATE_PER_HEAD else 16.0)
    eo, eh = run_tc_fwd(w, 24)
    assert eo <= TOL and eh <= TOL, (eo, eh)


# ------------------------------------------------- backward on the second stream
# The state-gradient pass and its reverse scan run on a library-owned second stream beside the
# dq kernel (one stream while the launch profiler is on); the results must not depend on that.

def _bwd_inputs(seed):
    w = I.WORKLOADS["c3"].replace(B=1, H=4, L=1500)
    x = {k: (None if v is None else v.cuda()) for k, v in I.make_inputs(w, seed=seed).items()}
    return w, x


def test_tc_bwd_second_stream_bitwise_equal_to_one_stream():
    from linear_rnn_b200 import _lib, ops
    w, x = _bwd_inputs(41)
    args = (x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], x["dO"], None)
    assert _lib.plan_info(ops.make_problem(x["q"], x["v"], x["g"], scale=w.scale, chunk=w.chunk, plan="tc"),
                          True)[1] > 1   # segmented: the second stream is used
    a = ops.gla_bwd(*args, scale=w.scale, chunk=w.chunk, plan="tc")
    _lib.profiler_enable(True)
    try:
        b = ops.gla_bwd(*args, scale=w.scale, chunk=w.chunk, plan="tc")
        torch.cuda.synchronize()
    finally:
        _lib.profiler_enable(False)
        _lib.profiler_read()
    for n in ("dq", "dk", "dv", "dg", "dh0"):
        assert torch.equal(a[n], b[n]), n


def test_tc_bwd_concurrent_calls_on_two_streams():
    """Two backward calls on two streams (distinct workspaces) share the library's second
    stream; each matches its own result computed alone."""
    from linear_rnn_b200 import ops
    w, x1 = _bwd_inputs(42)
    _, x2 = _bwd_inputs(43)
    args = lambda x: (x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], x["dO"], None)
    ref1 = ops.gla_bwd(*args(x1), scale=w.scale, chunk=w.chunk, plan="tc")
    ref2 = ops.gla_bwd(*args(x2), scale=w.scale, chunk=w.chunk, plan="tc")
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for _ in range(3):
        with torch.cuda.stream(s1):
            r1 = ops.gla_bwd(*args(x1), scale=w.scale, chunk=w.chunk, plan="tc")
        with torch.cuda.stream(s2):
            r2 = ops.gla_bwd(*args(x2), scale=w.scale, chunk=w.chunk, plan="tc")
        outs.append((r1, r2))
    torch.cuda.synchronize()
    for r1, r2 in outs:
        for n in ("dq", "dk", "dv", "dg", "dh0"):
            assert torch.equal(r1[n], ref1[n]), n
            assert torch.equal(r2[n], ref2[n]), n


@pytest.mark.parametrize("Dk,Dv", [(128, 256), (128, 128), (64, 256)])
@pytest.mark.parametrize("gate,ig", [(I.GATE_PER_KEY, True), (I.GATE_PER_HEAD, True), (I.GATE_NONE, False)])
def test_tc_bwd_single_stage_ring(Dk, Dv, gate, ig):
    """Backward shapes whose kernels hold one tile at a time and issue the next tile's loads as
    each slot's last reader finishes: 16 heads cut into segments of several tiles each, a
    ragged last tile, initial state and final-state gradient; two heads against the oracle."""
    from test_gpu_parity import check_bwd, with_dhT
    w = I.WORKLOADS["c3"].replace(B=2, H=8, L=1765, Dk=Dk, Dv=Dv, dtype="bf16", gate=gate, input_gate=ig,
                                  h0_std=0.3, backward=True,
                                  gate_mean=3.0 if gate == I.GATE_PER_HEAD else 0.0,
                                  gate_div=1.0 if gate == I.GATE_PER_HEAD else 16.0)
    x = with_dhT(I.make_inputs(w, seed=16), w)
    check_bwd(x, w, plan="tc", heads=[3, 12])
