"""Parity of the chunkwise DeltaNet forward (gla_deltanet_fwd) and backward (gla_deltanet_bwd)
with the float64 delta-rule oracle (oracle/deltanet.py: the recurrence and its back-propagation
through time, pinned in test_oracle_deltanet.py), element by element, on seeded inputs: unit-norm keys, beta = sigmoid(N(0,1)). Cases span several 64-token chunks and a ragged
tail, both key widths, several 64-column value slices, with and without h0, and the edge
lengths L = 0, 1 and 64. Bound: the max-normalised error, 1e-4 for fp32 I/O and 1e-2 for bf16
(fp32 I/O runs the CUDA-core forward, rounding only; bf16 I/O runs the tensor-core forward, whose
bf16 operands T, R, X and the state copy add their rounding to the output's)."""
import numpy as np
import pytest
import torch

from linear_rnn_b200 import inputs as I
from oracle import deltanet as DN

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


def record(case, errs):
    """Measured errors of a case, appended to the report file GLA_PARITY_REPORT names (if set)."""
    import json
    import os
    path = os.environ.get("GLA_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, "errors": errs}) + "\n")


def heads_of(t, heads):
    if t is None or heads is None:
        return t
    B, H = t.shape[0], t.shape[1]
    return t.reshape((B * H,) + tuple(t.shape[2:]))[heads][None]


def check(B, H, L, Dk, Dv, dtype, h0_std, seed=0, heads=None, case=None):
    from linear_rnn_b200 import ops
    x = I.make_deltanet_inputs(B, H, L, Dk, Dv, dtype, seed=seed, h0_std=h0_std)
    xd = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    scale = Dk ** -0.5
    o, hT = ops.gla_deltanet_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], scale=scale)
    torch.cuda.synchronize()
    xs = {n: heads_of(t, heads) for n, t in x.items()}
    ro, rS = DN.deltanet_fwd(xs["q"], xs["k"], xs["v"], xs["beta"], xs["h0"], scale)
    errs = {"hT": err(f64(heads_of(hT, heads)), rS)}
    if L:
        errs["o"] = err(f64(heads_of(o, heads)), ro)
    if case:
        record(case, errs)
    assert all(e <= TOL[dtype] for e in errs.values()), errs
    return o, hT


@pytest.mark.parametrize("B,H,L,Dk,Dv,dtype,h0_std", [
    (1, 2, 150, 64, 64, "f32", 0.5),
    (2, 1, 300, 128, 128, "bf16", 0.5),
    (1, 3, 200, 128, 256, "bf16", 0.0),
    (1, 2, 333, 128, 64, "f32", 1.0),
    (2, 2, 64, 64, 192, "bf16", 0.5),
])
def test_parity(B, H, L, Dk, Dv, dtype, h0_std):
    check(B, H, L, Dk, Dv, dtype, h0_std)


@pytest.mark.parametrize("L", [1, 63, 65])
def test_edge_lengths(L):
    check(1, 2, L, 64, 64, "f32", 0.5, seed=3)


@pytest.mark.parametrize("Dk", [64, 128])
@pytest.mark.parametrize("L", [1, 63, 64, 65, 129])
def test_tensor_core_edge_lengths(Dk, L):
    """bf16 I/O (the tensor-core forward) at chunk edges: a ragged last chunk reads zero rows past
    the end and stores none."""
    check(1, 2, L, Dk, 128, "bf16", 0.5, seed=11)


def test_tensor_core_full_size():
    """The DeltaNet workload (B=4 H=16 L=4096 Dk=Dv=128, bf16) on the tensor cores; two heads
    against the oracle."""
    c = I.DELTANET
    check(c["B"], c["H"], c["L"], c["Dk"], c["Dv"], c["dtype"], 0.5, seed=0, heads=[5, 50],
          case="deltanet full size heads=[5, 50]")


def test_empty_sequence_returns_h0():
    from linear_rnn_b200 import ops
    q = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(1, 2, 0, 128, dtype=torch.bfloat16, device="cuda")
    beta = torch.zeros(1, 2, 0, device="cuda")
    h0 = torch.randn(1, 2, 64, 128, device="cuda")
    o, hT = ops.gla_deltanet_fwd(q, q, v, beta, h0)
    assert o.shape == (1, 2, 0, 128) and torch.equal(hT, h0)
    _, hz = ops.gla_deltanet_fwd(q, q, v, beta, None)
    assert not torch.any(hz)


def test_long_sequence():
    # 32 chunks: the state hand-off between chunks over a long walk
    check(2, 4, 2048, 128, 128, "bf16", 0.5, seed=5)


def test_deterministic_and_host_round_trip():
    from linear_rnn_b200 import ops
    x = I.make_deltanet_inputs(1, 2, 257, 128, 128, "bf16", seed=9, h0_std=0.5)
    xd = {n: t.cuda() for n, t in x.items()}
    o1, h1 = ops.gla_deltanet_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"])
    o2, h2 = ops.gla_deltanet_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"])
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
    oh, hh = ops.gla_deltanet_fwd(x["q"], x["k"], x["v"], x["beta"], x["h0"])
    assert oh.device.type == "cpu" and torch.equal(oh, o1.cpu()) and torch.equal(hh, h1.cpu())


def check_bwd(B, H, L, Dk, Dv, dtype, h0_std, with_dhT, seed=0, case=None):
    from linear_rnn_b200 import ops
    x = I.make_deltanet_inputs(B, H, L, Dk, Dv, dtype, seed=seed, h0_std=h0_std)
    gen = torch.Generator().manual_seed(100 + seed)
    dO = torch.randn(B, H, L, Dv, generator=gen).to(x["q"].dtype)
    dhT = torch.randn(B, H, Dk, Dv, generator=gen) if with_dhT else None
    xd = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    scale = Dk ** -0.5
    r = ops.gla_deltanet_bwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], dO.cuda(),
                             None if dhT is None else dhT.cuda(), scale=scale)
    torch.cuda.synchronize()
    ref = DN.deltanet_bwd(x["q"], x["k"], x["v"], x["beta"], x["h0"], dO, dhT, scale)
    errs = {name: err(f64(r[name]), ref[name]) for name in ("dq", "dk", "dv", "dbeta", "dh0") if ref[name].size}
    if case:
        record(case, errs)
    assert all(e <= TOL[dtype] for e in errs.values()), errs
    return r


@pytest.mark.parametrize("B,H,L,Dk,Dv,dtype,h0_std,with_dhT", [
    (1, 2, 150, 64, 64, "f32", 0.5, True),
    (2, 1, 300, 128, 128, "bf16", 0.5, True),
    (1, 3, 200, 128, 256, "bf16", 0.0, False),
    (1, 2, 333, 128, 64, "f32", 1.0, False),
    (2, 2, 64, 64, 192, "bf16", 0.5, True),
])
def test_backward_parity(B, H, L, Dk, Dv, dtype, h0_std, with_dhT):
    check_bwd(B, H, L, Dk, Dv, dtype, h0_std, with_dhT)


@pytest.mark.parametrize("L", [0, 1, 63, 65])
def test_backward_edge_lengths(L):
    r = check_bwd(1, 2, L, 64, 64, "f32", 0.5, True, seed=7)
    assert r["dq"].shape == (1, 2, L, 64)


def test_backward_full_size():
    """The DeltaNet workload's backward (B=4 H=16 L=4096 Dk=Dv=128, bf16: the tensor-core state
    and reverse walks); two heads against the oracle's back-propagation through time."""
    from linear_rnn_b200 import ops
    c = I.DELTANET
    B, H, L, Dk, Dv = c["B"], c["H"], c["L"], c["Dk"], c["Dv"]
    x = I.make_deltanet_inputs(B, H, L, Dk, Dv, c["dtype"], seed=0, h0_std=0.5)
    gen = torch.Generator().manual_seed(100)
    dO = torch.randn(B, H, L, Dv, generator=gen).to(x["q"].dtype)
    xd = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    r = ops.gla_deltanet_bwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], dO.cuda(), None, scale=Dk ** -0.5)
    torch.cuda.synchronize()
    heads = [5, 50]
    xs = {n: heads_of(t, heads) for n, t in x.items()}
    ref = DN.deltanet_bwd(xs["q"], xs["k"], xs["v"], xs["beta"], xs["h0"], heads_of(dO, heads), None, Dk ** -0.5)
    errs = {n: err(f64(heads_of(r[n], heads)), ref[n]) for n in ("dq", "dk", "dv", "dbeta", "dh0")}
    record("deltanet backward full size heads=[5, 50]", errs)
    assert all(e <= TOL["bf16"] for e in errs.values()), errs


def test_backward_long_sequence():
    check_bwd(1, 2, 2048, 128, 128, "bf16", 0.5, True, seed=8, case="deltanet backward L=2048")


@pytest.mark.parametrize("L", [1, 64, 65])
def test_backward_tensor_core_recompute_edges(L):
    """bf16 I/O: the backward's chunk start states come from the tensor-core state walk."""
    check_bwd(1, 2, L, 128, 128, "bf16", 0.5, True, seed=12)


@pytest.mark.parametrize("B,H,L,Dk,Dv,dtype", [
    (2, 1, 300, 128, 128, "bf16"),
    (1, 2, 65, 64, 192, "bf16"),
    (1, 2, 150, 64, 64, "f32"),
    (1, 1, 1, 128, 64, "f32"),
])
def test_training_pair_saved_states(B, H, L, Dk, Dv, dtype):
    """gla_deltanet_fwd_save -> gla_deltanet_bwd_saved: the forward leaves the chunk start states
    and the backward reads them instead of walking the recurrence again. The states are the ones
    the backward's own walk writes, so every gradient is bit-identical to the recomputing
    backward's; both stay within the bound of the oracle."""
    from linear_rnn_b200 import ops
    x = I.make_deltanet_inputs(B, H, L, Dk, Dv, dtype, seed=21, h0_std=0.5)
    gen = torch.Generator().manual_seed(121)
    dO = torch.randn(B, H, L, Dv, generator=gen).to(x["q"].dtype)
    dhT = torch.randn(B, H, Dk, Dv, generator=gen)
    xd = {n: t.cuda() for n, t in x.items()}
    scale = Dk ** -0.5
    prob = ops.make_problem(xd["q"], xd["v"], None, scale=scale, chunk=64, plan="auto")
    nbytes = ops.gla_deltanet_saved_bytes(prob)
    esize = 2 if dtype == "bf16" else 4
    assert nbytes == B * H * ((L + 63) // 64) * Dk * Dv * esize
    saved = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")   # NaN pattern until written
    o1, h1 = ops.gla_deltanet_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], scale=scale, saved_states=saved)
    o0, h0 = ops.gla_deltanet_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], scale=scale)
    assert torch.equal(o1, o0) and torch.equal(h1, h0)
    args = (xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], dO.cuda(), dhT.cuda())
    ra = ops.gla_deltanet_bwd(*args, scale=scale, saved_states=saved)
    rb = ops.gla_deltanet_bwd(*args, scale=scale)
    for n in ("dq", "dk", "dv", "dbeta", "dh0"):
        assert torch.equal(ra[n], rb[n]), n
    ref = DN.deltanet_bwd(x["q"], x["k"], x["v"], x["beta"], x["h0"], dO, dhT, scale)
    errs = {n: err(f64(ra[n]), ref[n]) for n in ("dq", "dk", "dv", "dbeta", "dh0")}
    assert all(e <= TOL[dtype] for e in errs.values()), errs


def test_training_pair_rejects_short_saved_buffer():
    from linear_rnn_b200 import ops
    from linear_rnn_b200._lib import GlaError
    x = I.make_deltanet_inputs(1, 1, 128, 64, 64, "bf16", seed=3, h0_std=0.0)
    xd = {n: (None if t is None else t.cuda()) for n, t in x.items()}
    short = torch.empty(2 * 64 * 64 * 2 - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(GlaError):
        ops.gla_deltanet_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], None, saved_states=short)
