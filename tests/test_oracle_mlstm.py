"""Pins of the mLSTM oracle (oracle/mlstm.py) to facts other than itself, on the CPU.

Each pin takes the oracle module, so that the planted-mistake test at the end can run every pin
against a copy of the module with one textual mistake in it.
"""
import types

import numpy as np
import pytest

import oracle
from oracle import mlstm as ML


def _inputs(seed, B=1, H=2, L=9, Dk=4, Dv=3, ishift=0.0, gscale=1.0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, H, L, Dk))
    k = r.standard_normal((B, H, L, Dk))
    v = r.standard_normal((B, H, L, Dv))
    g = -np.log1p(np.exp(-(r.standard_normal((B, H, L)) + 1.0))) * gscale   # log sigmoid(N(1,1))
    itil = r.standard_normal((B, H, L)) + ishift
    return q, k, v, g, itil


def _unstabilised(q, k, v, g, itil, scale):
    """The same cell without the stabiliser: plain states, bound 1 (a different recurrence)."""
    B, H, L, Dk = k.shape
    Dv = v.shape[-1]
    h = np.zeros((B, H, L, Dv))
    for b in range(B):
        for hh in range(H):
            C = np.zeros((Dk, Dv))
            n = np.zeros(Dk)
            for t in range(L):
                a, i = np.exp(g[b, hh, t]), np.exp(itil[b, hh, t])
                C = a * C + i * np.outer(k[b, hh, t], v[b, hh, t])
                n = a * n + i * k[b, hh, t]
                qs = scale * q[b, hh, t]
                h[b, hh, t] = (qs @ C) / max(abs(qs @ n), 1.0)
    return h


def pin_matches_the_unstabilised_recurrence(M):
    for seed, ish in ((0, 0.0), (1, 2.0), (2, -3.0)):
        x = _inputs(seed, ishift=ish)
        h, _ = M.mlstm_fwd(*x, scale=0.7)
        ref = _unstabilised(*x, 0.7)
        assert np.allclose(h, ref, rtol=1e-12, atol=1e-12), (seed, np.abs(h - ref).max())


def pin_input_gates_beyond_exp_range_give_the_ratio(M):
    """i~ shifted by 800 (e^800 overflows float64): the stabilised cell stays finite and equals
    num / |den| of the unshifted gates (|den| is then far above the bound)."""
    q, k, v, g, itil = _inputs(3)
    h, st = M.mlstm_fwd(q, k, v, g, itil + 800.0, scale=1.0)
    assert np.isfinite(h).all() and np.isfinite(st["C"]).all()
    num = np.zeros_like(v)
    B, H, L, Dk = k.shape
    for b in range(B):
        for hh in range(H):
            C = np.zeros((Dk, v.shape[-1]))
            n = np.zeros(Dk)
            for t in range(L):
                a, i = np.exp(g[b, hh, t]), np.exp(itil[b, hh, t])
                C = a * C + i * np.outer(k[b, hh, t], v[b, hh, t])
                n = a * n + i * k[b, hh, t]
                num[b, hh, t] = (q[b, hh, t] @ C) / abs(q[b, hh, t] @ n)
    assert np.allclose(h, num, rtol=1e-9, atol=1e-12), np.abs(h - num).max()


def pin_equals_gated_attention_ratio(M):
    """num and den are the pinned gated oracle's outputs for values v and ones, with the
    per-head log-decay g and the input gate e^{i~}."""
    q, k, v, g, itil = _inputs(4, B=2, H=1, L=13)
    ig = np.exp(itil)
    num, _ = oracle.gla_fwd(q, k, v, g, ig, None, 0.9)
    den, _ = oracle.gla_fwd(q, k, np.ones(v.shape[:-1] + (1,)), g, ig, None, 0.9)
    ref = num / np.maximum(np.abs(den), 1.0)
    h, _ = M.mlstm_fwd(q, k, v, g, itil, scale=0.9)
    assert np.allclose(h, ref, rtol=1e-11, atol=1e-12), np.abs(h - ref).max()


def pin_quadratic_form_with_explicit_products(M):
    q, k, v, g, itil = _inputs(5, B=1, H=1, L=7, Dk=3, Dv=2)
    L = k.shape[2]
    ref = np.zeros_like(v)
    for t in range(L):
        num = np.zeros(v.shape[-1])
        den = 0.0
        for s in range(t + 1):
            w = np.exp(itil[0, 0, s])
            for tau in range(s + 1, t + 1):
                w *= np.exp(g[0, 0, tau])
            a = 0.5 * q[0, 0, t] @ k[0, 0, s]
            num += w * a * v[0, 0, s]
            den += w * a
        ref[0, 0, t] = num / max(abs(den), 1.0)
    h, _ = M.mlstm_fwd(q, k, v, g, itil, scale=0.5)
    assert np.allclose(h, ref, rtol=1e-12, atol=1e-13), np.abs(h - ref).max()


def pin_single_token_closed_form_both_sides_of_the_bound(M):
    r = np.random.default_rng(6)
    q = r.standard_normal((1, 1, 1, 4))
    k = q.copy()                        # q . k = |q|^2 > 0
    v = r.standard_normal((1, 1, 1, 3))
    g = np.array([[[-0.3]]])
    for itil, scale in ((np.array([[[3.0]]]), 1.0), (np.array([[[-6.0]]]), 0.01)):
        den = scale * float(q[0, 0, 0] @ k[0, 0, 0]) * np.exp(itil[0, 0, 0])
        ref = den * v[0, 0, 0] / max(abs(den), 1.0)
        h, st = M.mlstm_fwd(q, k, v, g, itil, scale=scale)
        assert np.allclose(h[0, 0, 0], ref, rtol=1e-13), (itil, h, ref)
        assert np.isclose(st["m"][0, 0], max(g[0, 0, 0], itil[0, 0, 0]))
    # the two cases sit on opposite sides of the bound
    assert abs(1.0 * float(q[0, 0, 0] @ k[0, 0, 0]) * np.exp(3.0)) > 1.0
    assert abs(0.01 * float(q[0, 0, 0] @ k[0, 0, 0]) * np.exp(-6.0)) < 1.0


def pin_shift_of_input_gate_where_normaliser_dominates(M):
    """Where every |den| > 1 before and after, h does not change when i~ shifts by a constant;
    where every |den| < 1, h scales by e^shift."""
    q, k, v, g, itil = _inputs(7, L=6)
    h0, _ = M.mlstm_fwd(q, k, v, g, itil + 20.0, scale=1.0)
    h1, _ = M.mlstm_fwd(q, k, v, g, itil + 22.5, scale=1.0)
    assert np.allclose(h0, h1, rtol=1e-10, atol=1e-13)
    l0, _ = M.mlstm_fwd(q, k, v, g, itil - 30.0, scale=1.0)
    l1, _ = M.mlstm_fwd(q, k, v, g, itil - 28.0, scale=1.0)
    assert np.allclose(l1, l0 * np.exp(2.0), rtol=1e-10, atol=1e-30)


def pin_backward_matches_finite_differences(M):
    q, k, v, g, itil = _inputs(8, B=1, H=2, L=6, Dk=3, Dv=2)
    dh = np.random.default_rng(9).standard_normal(v.shape)
    sc = 0.8
    grads = M.mlstm_bwd(q, k, v, g, itil, dh, scale=sc)
    # no token sits near the kink |den| = 1 of the bound
    den, _ = oracle.gla_fwd(q, k, np.ones(v.shape[:-1] + (1,)), g, np.exp(itil), None, sc)
    assert np.all(np.abs(np.abs(den) - 1.0) > 1e-3)
    names = ("q", "k", "v", "g", "itil")
    args = [q, k, v, g, itil]
    eps = 1e-6
    for ai, name in enumerate(names):
        x = args[ai]
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = [a.copy() for a in args]
            xm = [a.copy() for a in args]
            xp[ai][idx] += eps
            xm[ai][idx] -= eps
            fp = np.sum(dh * M.mlstm_fwd(*xp, scale=sc)[0])
            fm = np.sum(dh * M.mlstm_fwd(*xm, scale=sc)[0])
            num[idx] = (fp - fm) / (2 * eps)
        key = "d" + name
        assert np.allclose(grads[key], num, rtol=1e-6, atol=1e-7), (key, np.abs(grads[key] - num).max())


def pin_state_is_the_stabilised_plain_state(M):
    """The final (C, n) times e^m equal the plain states sum_s e^{F_T - F_s + i~_s} k_s^T v_s."""
    q, k, v, g, itil = _inputs(10, L=8)
    _, st = M.mlstm_fwd(q, k, v, g, itil, scale=1.0)
    B, H, L, Dk = k.shape
    for b in range(B):
        for hh in range(H):
            C = np.zeros((Dk, v.shape[-1]))
            n = np.zeros(Dk)
            for s in range(L):
                w = np.exp(itil[b, hh, s] + g[b, hh, s + 1:].sum())
                C += w * np.outer(k[b, hh, s], v[b, hh, s])
                n += w * k[b, hh, s]
            e = np.exp(st["m"][b, hh])
            assert np.allclose(st["C"][b, hh] * e, C, rtol=1e-12)
            assert np.allclose(st["n"][b, hh] * e, n, rtol=1e-12)


PINS = [pin_matches_the_unstabilised_recurrence, pin_input_gates_beyond_exp_range_give_the_ratio,
        pin_equals_gated_attention_ratio, pin_quadratic_form_with_explicit_products,
        pin_single_token_closed_form_both_sides_of_the_bound, pin_shift_of_input_gate_where_normaliser_dominates,
        pin_backward_matches_finite_differences, pin_state_is_the_stabilised_plain_state]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__[4:])
def test_pin(pin):
    pin(ML)


def test_empty_sequence():
    q = np.zeros((1, 2, 0, 4))
    v = np.zeros((1, 2, 0, 3))
    g = np.zeros((1, 2, 0))
    h, st = ML.mlstm_fwd(q, q, v, g, g, scale=1.0)
    assert h.shape == (1, 2, 0, 3) and np.all(st["C"] == 0)
    r = ML.mlstm_bwd(q, q, v, g, g, v, scale=1.0)
    assert r["dq"].shape == (1, 2, 0, 4) and r["ditil"].shape == (1, 2, 0)


# ------------------------------------------------------------- planted mistakes
# (text in oracle/mlstm.py, its replacement): the absolute value dropped from the bound, the
# bound 1 instead of exp(-m), the forget factor without m_{t-1}, the input gate without the
# stabiliser, a normaliser without the input gate, the readout from the old state, the wrong
# sign of dden, dden kept where the bound is active, d i~ without the gate factor, the second
# term of dk dropped.
MUTANTS = [
    ("np.maximum(np.abs(den), np.exp(-m))", "np.maximum(den, np.exp(-m))"),
    ("np.maximum(np.abs(den), np.exp(-m))", "np.maximum(np.abs(den), 1.0)"),
    ("fp = np.exp(gt + m_prev - m)", "fp = np.exp(gt - m)"),
    ("ip = np.exp(it - m)", "ip = np.exp(it)"),
    ("n = fp[..., None] * n + ip[..., None] * kt", "n = fp[..., None] * n + kt"),
    ('        C = fp[..., None, None] * C + ip[..., None, None] * np.einsum("bhi,bhj->bhij", kt, v[:, :, t])\n',
     '        Cold = C\n'
     '        C = fp[..., None, None] * C + ip[..., None, None] * np.einsum("bhi,bhj->bhij", kt, v[:, :, t])\n'),
    ("dden = np.where(active, -np.einsum", "dden = np.where(active, np.einsum"),
    ("dden = np.where(active, -np.einsum", "dden = np.where(True, -np.einsum"),
    ('"ditil": (r1["di"] + r2["di"]) * ig', '"ditil": (r1["di"] + r2["di"])'),
    ('"dk": r1["dk"] + r2["dk"]', '"dk": r1["dk"]'),
]
# the readout-from-the-old-state mistake needs the readout to use Cold as well
MUTANTS[5] = (MUTANTS[5][0] + '        n = fp[..., None] * n + ip[..., None] * kt\n'
              '        qs = scale * q[:, :, t]\n'
              '        num = np.einsum("bhi,bhij->bhj", qs, C)',
              MUTANTS[5][1] + '        n = fp[..., None] * n + ip[..., None] * kt\n'
              '        qs = scale * q[:, :, t]\n'
              '        num = np.einsum("bhi,bhij->bhj", qs, Cold)')


def _mutant_module(i):
    path = ML.__file__
    src = open(path).read()
    old, new = MUTANTS[i]
    assert src.count(old) == 1, old
    mod = types.ModuleType(f"mlstm_mutant_{i}")
    exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("i", range(len(MUTANTS)))
def test_planted_mistake_is_caught(i):
    mod = _mutant_module(i)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except (AssertionError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"mutant {i} passed every pin"
