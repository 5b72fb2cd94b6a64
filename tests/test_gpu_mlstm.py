"""GPU parity of the mLSTM cell (gla_mlstm_fwd / gla_mlstm_bwd) against the float64 oracle
(oracle/mlstm.py: the stabilised token recurrence and its gradients), on the same seeded
inputs. Metric per output tensor: max|x - x_ref| / max|x_ref|; bound 1e-2 for bf16 I/O, 1e-4
for fp32 I/O. The normaliser is always the fp32 recurrence; the value pass runs in fp32 on the
CUDA cores (automatic plan, "simt") or in bf16 on the tensor cores ("tc")."""
import numpy as np
import pytest
import torch

import oracle
from linear_rnn_b200 import inputs as I
from oracle import mlstm as ML

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def err(got, ref):
    """max|got - ref| / max|ref|; where the reference is identically zero (dg of a single token),
    the absolute error instead."""
    scale = np.abs(ref).max() if ref.size else 0.0
    return float(np.abs(got - ref).max() / scale) if scale > 0 else float(np.abs(got).max(initial=0.0))


def heads_of(t, heads):
    if heads is None:
        return t
    B, H = t.shape[0], t.shape[1]
    return t.reshape((B * H,) + tuple(t.shape[2:]))[heads][None]


def run(w, seed=0, itil_shift=0.0, backward=True, heads=None, plan="auto"):
    from linear_rnn_b200 import ops
    x = I.make_mlstm_inputs(w, seed=seed, itil_shift=itil_shift)
    xd = {k: v.cuda() for k, v in x.items() if v is not None}
    h = ops.gla_mlstm_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["itil"], scale=w.scale, chunk=w.chunk, plan=plan)
    xs = {k: heads_of(v, heads) for k, v in x.items() if v is not None}
    rh, _ = ML.mlstm_fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["itil"], w.scale)
    errs = {"h": err(heads_of(f64(h), heads), rh)}
    if backward:
        r = ops.gla_mlstm_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["itil"], xd["dh"], scale=w.scale, chunk=w.chunk,
                              plan=plan)
        ref = ML.mlstm_bwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["itil"], xs["dh"], w.scale)
        for n in ("dq", "dk", "dv", "dg", "ditil"):
            errs[n] = err(heads_of(f64(r[n]), heads), ref[n])
    tol = TOL[w.dtype]
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, (bad, errs)
    return errs


def record(case, errs):
    """Measured errors of a case, appended to the report file GLA_PARITY_REPORT names (if set)."""
    import json
    import os
    path = os.environ.get("GLA_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, "errors": errs}) + "\n")


def small(**kw):
    return I.MLSTM.replace(B=1, H=2, L=300, **kw)


@pytest.mark.parametrize("Dk,Dv", [(64, 64), (128, 128), (128, 256), (256, 256), (64, 256)])
def test_head_dims_bf16(Dk, Dv):
    run(small(Dk=Dk, Dv=Dv, scale=Dk ** -0.5), seed=1)


@pytest.mark.parametrize("L", [1, 63, 64, 65, 200])
def test_ragged_lengths(L):
    run(I.MLSTM.replace(B=2, H=1, L=L, Dk=128, Dv=128, scale=128 ** -0.5), seed=2)


def test_fp32_cuda_core_plan():
    run(small(Dk=64, Dv=128, dtype="f32", scale=64 ** -0.5), seed=3)


@pytest.mark.parametrize("Dk,Dv", [(64, 128), (256, 256)])
def test_bf16_cuda_core_value_pass(Dk, Dv):
    """plan="simt" on bf16 I/O (the automatic plan's path): the value pass on fp32 copies of the
    inputs, gradients cast back."""
    run(small(Dk=Dk, Dv=Dv, scale=Dk ** -0.5), seed=8, plan="simt")


def test_tensor_core_value_pass_full_size():
    """plan="tc" on the mLSTM workload (B=2 H=8 L=8192 Dk=Dv=256, bf16): the value pass on the
    tensor cores, the normaliser recurrence in fp32; two heads against the oracle."""
    errs = run(I.MLSTM, seed=0, heads=[1, 14], plan="tc")
    record("mlstm tc plan full size heads=[1, 14]", errs)


@pytest.mark.parametrize("L", [64, 300, 1000])
def test_tensor_core_value_pass_c5_shape(L):
    """plan="tc" at the head dims of the mLSTM workload (Dk=Dv=256) over shorter sequences."""
    errs = run(I.MLSTM.replace(B=1, H=2, L=L), seed=10, plan="tc")
    record(f"mlstm tc plan L={L}", errs)


@pytest.mark.parametrize("L", [31, 32, 33, 97, 600])
def test_normaliser_segment_edges(L):
    """Sequences that end inside, at and just past a 32-token segment of the normaliser recurrence
    (600 tokens: 19 segments, past a group of 16 in the scans over segments)."""
    run(I.MLSTM.replace(B=1, H=3, L=L, Dk=64, Dv=64, scale=0.125), seed=9)


@pytest.mark.parametrize("L", [1, 33, 257, 1500])
def test_normaliser_segment_edges_fp32(L):
    """fp32 I/O (both sums on the CUDA cores in fp32) at 1e-4, across segment edges and the
    segment scans (1500 tokens: 47 segments, groups of 16, 16 and 15 in the two-level scans)."""
    run(I.MLSTM.replace(B=2, H=1, L=L, Dk=128, Dv=64, dtype="f32", scale=128 ** -0.5), seed=13)


@pytest.mark.parametrize("shift", [60.0, -20.0])
def test_input_gates_far_from_zero(shift):
    """exp(i~) far outside [e^-20, e^60]: the per-head shift keeps the gates in range and h equals
    the stabilised recurrence."""
    run(small(Dk=128, Dv=128, scale=128 ** -0.5), seed=4, itil_shift=shift)


def test_normaliser_bound_active():
    """A small scale puts |den| below 1 for many tokens (the bound 1 is the divisor there)."""
    w = small(Dk=128, Dv=128, scale=0.002)
    x = I.make_mlstm_inputs(w, seed=5)
    den, _ = oracle.gla_fwd(x["q"], x["k"], np.ones(tuple(x["v"].shape[:-1]) + (1,)), x["g"], np.exp(f64(x["itil"])),
                            None, w.scale)
    frac = float((np.abs(den) < 1).mean())
    assert 0.2 < frac < 1.0, frac
    run(w, seed=5)


def test_full_size_workload():
    """The mLSTM workload (B=2 H=8 L=8192 Dk=Dv=256, bf16) on the GPU; two heads against the
    oracle."""
    errs = run(I.MLSTM, seed=0, heads=[1, 14])
    record("mlstm automatic plan full size heads=[1, 14]", errs)


def test_empty_and_deterministic():
    from linear_rnn_b200 import ops
    w = small(Dk=128, Dv=128, scale=128 ** -0.5)
    x = {k: v.cuda() for k, v in I.make_mlstm_inputs(w, seed=6).items()}
    a = ops.gla_mlstm_bwd(x["q"], x["k"], x["v"], x["g"], x["itil"], x["dh"], scale=w.scale)
    b = ops.gla_mlstm_bwd(x["q"], x["k"], x["v"], x["g"], x["itil"], x["dh"], scale=w.scale)
    for n in a:
        assert torch.equal(a[n], b[n]), n
    e = {k: v[:, :, :0].contiguous() for k, v in x.items()}
    h = ops.gla_mlstm_fwd(e["q"], e["k"], e["v"], e["g"], e["itil"], scale=w.scale)
    assert h.shape == (1, 2, 0, 128)


def test_tensor_core_value_pass_other_dims():
    """plan="tc" at head dims other than the workload's: finite results, and h within the bf16
    bound (the gradients' error there is the bf16 pass's, amplified where the numerator's and the
    normaliser's parts cancel; it is recorded, not bounded)."""
    from linear_rnn_b200 import ops
    for Dk, Dv in ((64, 64), (128, 128), (128, 256)):
        w = small(Dk=Dk, Dv=Dv, scale=Dk ** -0.5)
        x = I.make_mlstm_inputs(w, seed=7)
        xd = {k: v.cuda() for k, v in x.items()}
        h = ops.gla_mlstm_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["itil"], scale=w.scale, plan="tc")
        r = ops.gla_mlstm_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["itil"], xd["dh"], scale=w.scale, plan="tc")
        assert torch.isfinite(h.float()).all() and all(torch.isfinite(t.float()).all() for t in r.values())
        rh, _ = ML.mlstm_fwd(x["q"], x["k"], x["v"], x["g"], x["itil"], w.scale)
        ref = ML.mlstm_bwd(x["q"], x["k"], x["v"], x["g"], x["itil"], x["dh"], w.scale)
        errs = {"h": err(f64(h), rh)}
        errs.update({n: err(f64(r[n]), ref[n]) for n in ("dq", "dk", "dv", "dg", "ditil")})
        record(f"mlstm tc plan Dk={Dk} Dv={Dv} L=300", errs)
        assert errs["h"] <= TOL["bf16"], errs


def test_rejects_per_key_gates():
    import ctypes
    from linear_rnn_b200 import _lib, ops
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(1, 1, 64, 64, device="cuda")
    p = ops.make_problem(q, q, g, scale=1.0, chunk=64, plan="auto")
    assert _lib.lib.gla_mlstm_workspace_bytes(ctypes.byref(p), 0) == 0


@pytest.mark.parametrize("plan,dtype,L,Dk,Dv", [
    ("tc", "bf16", 1000, 256, 256),
    ("tc", "bf16", 65, 128, 128),
    ("auto", "bf16", 300, 128, 256),
    ("auto", "f32", 97, 64, 128),
])
def test_training_pair_saved_results(plan, dtype, L, Dk, Dv):
    """gla_mlstm_fwd_save -> gla_mlstm_bwd_saved: the backward reads the forward's results (the
    gate terms, num, den, the normaliser's segment states and the value pass's saved states)
    instead of running the forward again. h is bit-identical to gla_mlstm_fwd's. The CUDA-core
    value pass keeps no segment states, so there every gradient is bit-identical to the
    recomputing backward's; with the tensor-core pass the backward's segment states come from the
    forward's walk instead of a state pass and scan, so the gradients are checked against the
    oracle."""
    from linear_rnn_b200 import ops
    w = I.MLSTM.replace(B=1, H=2, L=L, Dk=Dk, Dv=Dv, dtype=dtype, scale=Dk ** -0.5)
    x = I.make_mlstm_inputs(w, seed=31)
    xd = {k: v.cuda() for k, v in x.items()}
    args = (xd["q"], xd["k"], xd["v"], xd["g"], xd["itil"])
    prob = ops.make_problem(xd["q"], xd["v"], xd["g"], scale=w.scale, chunk=w.chunk, plan=plan)
    nbytes = ops.gla_mlstm_saved_bytes(prob)
    assert nbytes > 0
    saved = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")   # NaN pattern until written
    h1 = ops.gla_mlstm_fwd(*args, scale=w.scale, plan=plan, saved_states=saved)
    h0 = ops.gla_mlstm_fwd(*args, scale=w.scale, plan=plan)
    assert torch.equal(h1, h0)
    ra = ops.gla_mlstm_bwd(*args, xd["dh"], scale=w.scale, plan=plan, saved_states=saved)
    rb = ops.gla_mlstm_bwd(*args, xd["dh"], scale=w.scale, plan=plan)
    names = ("dq", "dk", "dv", "dg", "ditil")
    if plan != "tc":
        for n in names:
            assert torch.equal(ra[n], rb[n]), n
    ref = ML.mlstm_bwd(x["q"], x["k"], x["v"], x["g"], x["itil"], x["dh"], w.scale)
    errs = {n: err(f64(ra[n]), ref[n]) for n in names}
    record(f"mlstm training pair plan={plan} {dtype} L={L} Dk={Dk} Dv={Dv}", errs)
    if plan == "tc" and Dk != 256:
        return   # other head dims on the tensor-core pass: recorded, not bounded (see above)
    assert all(e <= TOL[dtype] for e in errs.values()), errs
