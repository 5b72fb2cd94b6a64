"""Pins for the float64 oracle: each test ties it to something other than itself.

* closed forms of the ungated case (causal masked matmul; the state is K^T V) -- the
  "parallel form" of linear attention (talk summary "Hardware-Efficient Training of
  Linear Attention Models", section 7:36) written as plain matrix products;
* the brute-force quadratic form with explicit products of decays for gated inputs;
* special cases that reduce to textbook results (alpha = 0, scalar gates, L = 1);
* invariants: state hand-off, linearity, chunk-size invariance of the chunkwise
  restatement (section 11:58: recurrent inter-chunk plus parallel intra-chunk parts);
* central finite differences of the forward for every input of the backward;
* the chunkwise closed form of dg and its shift-invariance property.
"""
import numpy as np
import pytest

import oracle
from chunk_algebra import chunk_bwd, chunk_fwd

RNG = np.random.default_rng(1234)


def rnd(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def gates(*shape):
    # log-decays in (-inf, 0): logsigmoid of a normal, as in the workloads
    return -np.log1p(np.exp(-rnd(*shape))) / 4.0


def rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ---------------------------------------------------------------- forward, closed forms

@pytest.mark.parametrize("with_h0", [False, True])
def test_ungated_is_causal_masked_matmul(with_h0):
    B, H, L, Dk, Dv = 2, 3, 37, 5, 4
    q, k, v = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv)
    h0 = rnd(B, H, Dk, Dv) if with_h0 else None
    scale = 0.7
    o, hT = oracle.gla_fwd(q, k, v, None, None, h0, scale)
    mask = np.tril(np.ones((L, L)))
    o_ref = scale * (np.einsum("bhtd,bhsd->bhts", q, k) * mask) @ v
    hT_ref = np.einsum("bhsd,bhse->bhde", k, v)
    if with_h0:
        o_ref = o_ref + scale * q @ h0
        hT_ref = hT_ref + h0
    assert rel(o, o_ref) < 1e-12
    assert rel(hT, hT_ref) < 1e-12


def quadratic_form(q, k, v, g, ig, h0, scale):
    """o_t = scale [ sum_{s<=t} sum_d q_td k_sd prod_{s<tau<=t} alpha_tau,d  v_s
                     + sum_d q_td prod_{tau<=t} alpha_tau,d h0_d ]  (explicit products)."""
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    if g.ndim == 3:
        g = np.repeat(g[..., None], Dk, axis=-1)
    if ig is not None:
        k = k * ig[..., None]
    alpha = np.exp(g)
    o = np.zeros((B, H, L, Dv))
    hT = np.zeros((B, H, Dk, Dv))
    for b in range(B):
        for h in range(H):
            for t in range(L):
                for s in range(t + 1):
                    dec = np.prod(alpha[b, h, s + 1:t + 1], axis=0)   # [Dk]
                    o[b, h, t] += np.sum(q[b, h, t] * k[b, h, s] * dec) * v[b, h, s]
                if h0 is not None:
                    dec0 = np.prod(alpha[b, h, :t + 1], axis=0)
                    o[b, h, t] += (q[b, h, t] * dec0) @ h0[b, h]
                o[b, h, t] *= scale
            for s in range(L):
                dec = np.prod(alpha[b, h, s + 1:], axis=0)
                hT[b, h] += np.outer(k[b, h, s] * dec, v[b, h, s])
            if h0 is not None:
                hT[b, h] += np.prod(alpha[b, h], axis=0)[:, None] * h0[b, h]
    return o, hT


@pytest.mark.parametrize("mode", ["key", "head"])
@pytest.mark.parametrize("with_h0,with_ig", [(False, False), (True, False), (True, True)])
def test_gated_matches_quadratic_form(mode, with_h0, with_ig):
    B, H, L, Dk, Dv = 1, 2, 23, 4, 3
    q, k, v = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv)
    g = gates(B, H, L, Dk) if mode == "key" else gates(B, H, L)
    h0 = rnd(B, H, Dk, Dv) if with_h0 else None
    ig = 1.0 / (1.0 + np.exp(-rnd(B, H, L))) if with_ig else None
    o, hT = oracle.gla_fwd(q, k, v, g, ig, h0, 0.5)
    o_ref, hT_ref = quadratic_form(q, k, v, g, ig, h0, 0.5)
    assert rel(o, o_ref) < 1e-12
    assert rel(hT, hT_ref) < 1e-12


def test_zero_gate_equals_ungated():
    B, H, L, Dk, Dv = 1, 2, 30, 6, 5
    q, k, v, h0 = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    a = oracle.gla_fwd(q, k, v, np.zeros((B, H, L, Dk)), None, h0, 0.3)
    b = oracle.gla_fwd(q, k, v, None, None, h0, 0.3)
    assert rel(a[0], b[0]) < 1e-14 and rel(a[1], b[1]) < 1e-14


def test_alpha_zero_keeps_only_current_token():
    """alpha = 0 (g = -inf) forgets everything: o_t = scale (q_t . k_t) v_t and
    hT = k_{L-1}^T v_{L-1}."""
    B, H, L, Dk, Dv = 1, 1, 12, 4, 3
    q, k, v, h0 = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    g = np.full((B, H, L, Dk), -np.inf)
    o, hT = oracle.gla_fwd(q, k, v, g, None, h0, 2.0)
    o_ref = 2.0 * np.sum(q * k, axis=-1, keepdims=True) * v
    assert rel(o, o_ref) < 1e-14
    assert rel(hT[0, 0], np.outer(k[0, 0, -1], v[0, 0, -1])) < 1e-14


def test_per_key_with_equal_dims_equals_per_head():
    B, H, L, Dk, Dv = 2, 1, 19, 5, 3
    q, k, v = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv)
    f = gates(B, H, L)
    a = oracle.gla_fwd(q, k, v, np.repeat(f[..., None], Dk, axis=-1), None, None, 1.0)
    b = oracle.gla_fwd(q, k, v, f, None, None, 1.0)
    assert rel(a[0], b[0]) < 1e-14 and rel(a[1], b[1]) < 1e-14


def test_single_token():
    B, H, Dk, Dv = 1, 2, 3, 4
    q, k, v = rnd(B, H, 1, Dk), rnd(B, H, 1, Dk), rnd(B, H, 1, Dv)
    g, h0 = gates(B, H, 1, Dk), rnd(B, H, Dk, Dv)
    o, hT = oracle.gla_fwd(q, k, v, g, None, h0, 1.5)
    hT_ref = np.exp(g[:, :, 0])[..., None] * h0 + np.einsum("bhd,bhe->bhde", k[:, :, 0], v[:, :, 0])
    assert rel(hT, hT_ref) < 1e-14
    assert rel(o[:, :, 0], 1.5 * np.einsum("bhd,bhde->bhe", q[:, :, 0], hT_ref)) < 1e-14


def test_empty_sequence_returns_h0():
    B, H, Dk, Dv = 1, 1, 3, 2
    h0 = rnd(B, H, Dk, Dv)
    o, hT = oracle.gla_fwd(np.zeros((B, H, 0, Dk)), np.zeros((B, H, 0, Dk)),
                           np.zeros((B, H, 0, Dv)), np.zeros((B, H, 0, Dk)), None, h0, 1.0)
    assert o.shape == (B, H, 0, Dv)
    assert np.array_equal(hT, h0)


def test_linearity_in_v_and_h0():
    B, H, L, Dk, Dv = 1, 2, 17, 4, 3
    q, k, g = rnd(B, H, L, Dk), rnd(B, H, L, Dk), gates(B, H, L, Dk)
    v1, v2, h1, h2 = rnd(B, H, L, Dv), rnd(B, H, L, Dv), rnd(B, H, Dk, Dv), rnd(B, H, Dk, Dv)
    a1 = oracle.gla_fwd(q, k, v1, g, None, h1, 1.0)
    a2 = oracle.gla_fwd(q, k, v2, g, None, h2, 1.0)
    a = oracle.gla_fwd(q, k, 2 * v1 - 3 * v2, g, None, 2 * h1 - 3 * h2, 1.0)
    assert rel(a[0], 2 * a1[0] - 3 * a2[0]) < 1e-12
    assert rel(a[1], 2 * a1[1] - 3 * a2[1]) < 1e-12


def test_state_hand_off():
    """fwd(L) == fwd(L1) then fwd(L2, h0 = hT of the first part)."""
    B, H, L, Dk, Dv, L1 = 1, 2, 41, 5, 4, 18
    q, k, v, g, h0 = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), gates(B, H, L, Dk), rnd(B, H, Dk, Dv)
    o, hT = oracle.gla_fwd(q, k, v, g, None, h0, 0.9)
    oa, ha = oracle.gla_fwd(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], g[:, :, :L1], None, h0, 0.9)
    ob, hb = oracle.gla_fwd(q[:, :, L1:], k[:, :, L1:], v[:, :, L1:], g[:, :, L1:], None, ha, 0.9)
    assert rel(np.concatenate([oa, ob], axis=2), o) < 1e-13
    assert rel(hb, hT) < 1e-13


def test_multithreaded_equals_single_threaded():
    B, H, L, Dk, Dv = 2, 3, 50, 8, 40
    q, k, v, g = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), gates(B, H, L, Dk)
    a = oracle.gla_fwd(q, k, v, g, None, None, 1.0, nthreads=1)
    b = oracle.gla_fwd(q, k, v, g, None, None, 1.0, nthreads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ------------------------------------------------------- chunkwise restatement invariance

@pytest.mark.parametrize("C", [1, 2, 3, 16, 64, 77])
@pytest.mark.parametrize("sub", [1, 4, 16])
def test_chunkwise_restatement_matches_recurrence(C, sub):
    B, H, L, Dk, Dv = 1, 2, 77, 6, 5
    q, k, v, g, h0 = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), gates(B, H, L, Dk), rnd(B, H, Dk, Dv)
    ig = 1.0 / (1.0 + np.exp(-rnd(B, H, L)))
    o, hT = oracle.gla_fwd(q, k, v, g, ig, h0, 0.4)
    oc, hc = chunk_fwd(q, k, v, g, ig, h0, 0.4, C=C, sub=sub)
    assert rel(oc, o) < 1e-10
    assert rel(hc, hT) < 1e-10


# ------------------------------------------------------------------------ gradients

def _loss(args, dO, dhT, scale):
    o, hT = oracle.gla_fwd(*args, scale)
    return float(np.sum(o * dO) + np.sum(hT * dhT))


@pytest.mark.parametrize("mode", ["key", "head", "none"])
def test_backward_matches_finite_differences(mode):
    B, H, L, Dk, Dv = 1, 2, 9, 3, 2
    q, k, v = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv)
    g = {"key": gates(B, H, L, Dk), "head": gates(B, H, L), "none": None}[mode]
    ig = 1.0 / (1.0 + np.exp(-rnd(B, H, L)))
    h0, dO, dhT = rnd(B, H, Dk, Dv), rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    scale = 0.8
    grads = oracle.gla_bwd(q, k, v, g, ig, h0, dO, dhT, scale)
    args = [q, k, v, g, ig, h0]
    names = {0: "dq", 1: "dk", 2: "dv", 3: "dg", 4: "di", 5: "dh0"}
    eps = 1e-6
    for idx, name in names.items():
        x = args[idx]
        if x is None:
            assert grads[name] is None
            continue
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            mi = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[mi] += eps
            xm[mi] -= eps
            ap, am = list(args), list(args)
            ap[idx], am[idx] = xp, xm
            num[mi] = (_loss(ap, dO, dhT, scale) - _loss(am, dO, dhT, scale)) / (2 * eps)
        assert rel(grads[name], num) < 1e-7, name


def test_ungated_gradient_closed_forms():
    """alpha = 1: o = scale tril(Q K^T) V + scale Q h0, hT = K^T V + h0. Then
    dq = scale tril(dO V^T) K + scale dO h0^T, dv = scale tril(Q K^T)^T dO + K dhT,
    dk = scale tril(dO V^T)^T Q + V dhT^T, dh0 = scale Q^T dO + dhT."""
    B, H, L, Dk, Dv = 1, 2, 29, 5, 4
    q, k, v, h0 = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    dO, dhT = rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    s = 0.6
    r = oracle.gla_bwd(q, k, v, None, None, h0, dO, dhT, s)
    M = np.tril(np.ones((L, L)))
    tT = lambda x: np.swapaxes(x, -1, -2)
    A = (q @ tT(k)) * M
    dA = (dO @ tT(v)) * M
    assert rel(r["dq"], s * dA @ k + s * dO @ tT(h0)) < 1e-12
    assert rel(r["dv"], s * tT(A) @ dO + k @ dhT) < 1e-12
    assert rel(r["dk"], s * tT(dA) @ q + v @ tT(dhT)) < 1e-12
    assert rel(r["dh0"], s * tT(q) @ dO + dhT) < 1e-12


@pytest.mark.parametrize("mode", ["key", "head"])
@pytest.mark.parametrize("C", [1, 16, 64, 50])
def test_chunkwise_backward_closed_form_matches_bptt(mode, C):
    """The chunkwise gradients (state-gradient reverse pass, per-chunk dq/dk/dv and dg
    as a reverse cumulative sum) equal back-propagation through time."""
    B, H, L, Dk, Dv = 1, 2, 70, 5, 4
    q, k, v = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv)
    g = gates(B, H, L, Dk) if mode == "key" else gates(B, H, L)
    ig = 1.0 / (1.0 + np.exp(-rnd(B, H, L)))
    h0, dO, dhT = rnd(B, H, Dk, Dv), rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    ref = oracle.gla_bwd(q, k, v, g, ig, h0, dO, dhT, 0.7)
    got = chunk_bwd(q, k, v, g, ig, h0, dO, dhT, 0.7, C=C, sub=16)
    for name in ("dq", "dk", "dv", "dg", "di", "dh0"):
        assert rel(got[name], ref[name]) < 1e-10, name


def test_dg_first_token_vanishes_without_h0_and_dhT():
    """Adding a constant to g_0 shifts every cumulative log-decay equally, so without
    an initial state and without a final-state gradient nothing depends on it."""
    B, H, L, Dk, Dv = 2, 2, 40, 4, 3
    q, k, v, g, dO = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), gates(B, H, L, Dk), rnd(B, H, L, Dv)
    r = oracle.gla_bwd(q, k, v, g, None, None, dO, None, 1.0)
    assert np.abs(r["dg"][:, :, 0]).max() < 1e-12 * np.abs(r["dg"]).max()
    dB = q * r["dq"] - k * r["dk"]
    assert np.abs(dB.sum(axis=2)).max() < 1e-11 * np.abs(dB).max()


def test_backward_linear_in_dO():
    B, H, L, Dk, Dv = 1, 1, 21, 4, 3
    q, k, v, g = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), gates(B, H, L, Dk)
    d1, d2 = rnd(B, H, L, Dv), rnd(B, H, L, Dv)
    a = oracle.gla_bwd(q, k, v, g, None, None, d1, None, 1.0)
    b = oracle.gla_bwd(q, k, v, g, None, None, d2, None, 1.0)
    c = oracle.gla_bwd(q, k, v, g, None, None, d1 + 2 * d2, None, 1.0)
    for name in ("dq", "dk", "dv", "dg"):
        assert rel(c[name], a[name] + 2 * b[name]) < 1e-12
