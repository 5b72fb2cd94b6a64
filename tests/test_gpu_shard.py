"""Sequence sharding on one GPU: a sequence cut into shards processed one after another by
the library's per-shard calls (gla_shard_state, gla_shard_state_grad, gla_state_fold, gla_fwd,
gla_bwd), the all-gather replaced by stacking. The shards' outputs concatenated must equal the float64 oracle over the
whole sequence (bf16 bound 1e-2 on the max-normalised error), and each shard's (end state from
zero, total log-decay) must equal the oracle's end state of that shard alone and the sum of
its log-gates."""
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


@pytest.mark.parametrize("gate,ig,Dk,Dv", [(I.GATE_PER_KEY, False, 128, 128), (I.GATE_PER_HEAD, True, 256, 256),
                                           (I.GATE_NONE, False, 64, 128), (I.GATE_PER_KEY, True, 128, 256)])
def test_sharded_forward_equals_the_whole_sequence(gate, ig, Dk, Dv):
    from linear_rnn_b200 import ops
    w = I.WORKLOADS["c3"].replace(B=1, H=3, L=700, Dk=Dk, Dv=Dv, gate=gate, input_gate=ig, h0_std=0.5,
                                  gate_mean=3.0 if gate == I.GATE_PER_HEAD else 0.0,
                                  gate_div=1.0 if gate == I.GATE_PER_HEAD else 16.0)
    x = I.make_inputs(w, seed=51)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    cuts = [0, 256, 301, 700]   # shards of 256, 45 and 399 tokens
    shard = lambda t, p: None if t is None else t[:, :, cuts[p]:cuts[p + 1]].contiguous()
    names = ("q", "k", "v", "g", "igate")
    parts = []
    for p in range(3):
        s = {n: shard(xd[n], p) for n in names}
        S, gam = ops.gla_shard_state(s["k"], s["v"], s["g"], s["igate"], chunk=64)
        # pins of the per-shard pieces: the oracle's end state of the shard alone, and the
        # shard's total log-decay (the sum of its log-gates)
        hs = {n: shard(x[n], p) for n in names}
        _, rS = oracle.gla_fwd(hs["q"], hs["k"], hs["v"], hs["g"], hs["igate"], None, w.scale)
        assert err(f64(S), rS) <= TOL
        if gate != I.GATE_NONE:
            rg = hs["g"].double().sum(dim=2)
            rg = rg if gate == I.GATE_PER_KEY else rg[..., None].expand(-1, -1, Dk)
            assert np.allclose(f64(gam), rg.numpy(), rtol=1e-5, atol=1e-4)
        else:
            assert not torch.any(gam)
        parts.append((S, gam))
    states = torch.stack([a for a, _ in parts])
    gammas = torch.stack([b for _, b in parts])
    outs, hT = [], None
    for p in range(3):
        s_in = ops.gla_state_fold(states, gammas, p, xd["h0"])
        s = {n: shard(xd[n], p) for n in names}
        o, hT = ops.gla_fwd(s["q"], s["k"], s["v"], s["g"], s["igate"], s_in, scale=w.scale, chunk=64)
        outs.append(o)
    ro, rS = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], w.scale)
    assert err(f64(torch.cat(outs, dim=2)), ro) <= TOL
    assert err(f64(hT), rS) <= TOL
    # folding all three shards from h0 gives the sequence's final state too
    assert err(f64(ops.gla_state_fold(states, gammas, 3, xd["h0"])), rS) <= TOL


def test_shard_state_of_an_empty_shard_is_zero():
    from linear_rnn_b200 import ops
    k = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(1, 2, 0, 64, device="cuda")
    S, gam = ops.gla_shard_state(k, k, g)
    assert S.shape == (1, 2, 64, 64) and not torch.any(S) and not torch.any(gam)


@pytest.mark.parametrize("gate,ig,Dk,Dv", [(I.GATE_PER_KEY, False, 128, 128), (I.GATE_PER_HEAD, True, 256, 256),
                                           (I.GATE_NONE, False, 64, 128), (I.GATE_PER_KEY, True, 128, 256)])
def test_sharded_backward_equals_the_whole_sequence(gate, ig, Dk, Dv):
    """Each shard's start-state gradient from zero must equal the oracle's dh0 of the shard
    alone (no dhT); the shards' gradients, each from its folded initial state and folded
    end gradient, concatenated, must equal the oracle's back-propagation through the whole
    sequence, and shard 0's dh0 the sequence's dh0."""
    from linear_rnn_b200 import ops
    w = I.WORKLOADS["c3"].replace(B=1, H=3, L=700, Dk=Dk, Dv=Dv, gate=gate, input_gate=ig, h0_std=0.5,
                                  gate_mean=3.0 if gate == I.GATE_PER_HEAD else 0.0,
                                  gate_div=1.0 if gate == I.GATE_PER_HEAD else 16.0)
    x = I.make_inputs(w, seed=52)
    x["dhT"] = I.make_dhT(w, seed=53)
    xd = {k: (None if v is None else v.cuda()) for k, v in x.items()}
    cuts = [0, 256, 301, 700]
    shard = lambda t, p: None if t is None else t[:, :, cuts[p]:cuts[p + 1]].contiguous()
    names = ("q", "k", "v", "g", "igate", "dO")
    fw, bw = [], []
    for p in range(3):
        s = {n: shard(xd[n], p) for n in names}
        S, gam = ops.gla_shard_state(s["k"], s["v"], s["g"], s["igate"], chunk=64)
        dS, gam2 = ops.gla_shard_state_grad(s["q"], s["dO"], s["g"], scale=w.scale, chunk=64)
        # the forward-state pass sums the log-gates from the shard's end, the gradient pass from
        # its start: the same float32 sum in another order
        assert torch.allclose(gam, gam2, rtol=1e-5, atol=1e-4)
        hs = {n: shard(x[n], p) for n in names}
        rl = oracle.gla_bwd(hs["q"], hs["k"], hs["v"], hs["g"], hs["igate"], None, hs["dO"], None, w.scale)
        assert err(f64(dS), rl["dh0"]) <= TOL
        fw.append((S, gam))
        bw.append(dS)
    states = torch.stack([a for a, _ in fw])
    gammas = torch.stack([b for _, b in fw])
    grads = torch.stack(bw)
    got = {n: [] for n in ("dq", "dk", "dv", "dg", "di")}
    dh0 = None
    for p in range(3):
        s_in = ops.gla_state_fold(states, gammas, p, xd["h0"])
        d_end = ops.gla_state_fold(grads.flip(0).contiguous(), gammas.flip(0).contiguous(), 2 - p, xd["dhT"])
        s = {n: shard(xd[n], p) for n in names}
        r = ops.gla_bwd(s["q"], s["k"], s["v"], s["g"], s["igate"], s_in, s["dO"], d_end, scale=w.scale,
                        chunk=64, output_dh0=p == 0)
        for n in got:
            got[n].append(r[n])
        if p == 0:
            dh0 = r["dh0"]
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], x["dO"], x["dhT"], w.scale)
    for n, parts in got.items():
        if ref[n] is None:
            assert all(t is None for t in parts), n
            continue
        assert err(f64(torch.cat(parts, dim=2)), ref[n]) <= TOL, n
    assert err(f64(dh0), ref["dh0"]) <= TOL


def test_shard_state_grad_of_an_empty_shard_is_zero():
    from linear_rnn_b200 import ops
    q = torch.zeros(1, 2, 0, 64, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(1, 2, 0, 64, device="cuda")
    dS, gam = ops.gla_shard_state_grad(q, q, g)
    assert dS.shape == (1, 2, 64, 64) and not torch.any(dS) and not torch.any(gam)
