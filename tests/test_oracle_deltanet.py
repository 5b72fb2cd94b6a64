"""Pins for the float64 delta-rule oracle (oracle/deltanet.py). Each ties it to something
other than itself: the talk summary "Hardware-Efficient Training of Linear Attention Models"
(DeltaNet sections 22:36 and 31:16) describes a memory that a writing strength beta_t
updates, by one gradient step on the key-to-value regression loss, through an
identity-plus-rank-one transition.

* beta = 0 writes nothing: the state stays h0;
* a unit key with beta = 1 fits its value exactly in one step (k_t S_t = v_t);
* an orthonormal key set recalls every stored value exactly, and rewriting a key replaces
  its value in the proportion beta (retain the old value or integrate the new one);
* the step equals S - beta * (central-difference gradient of 1/2 ||k S - v||^2);
* mutually orthogonal keys from a zero state give linear attention with input gate beta,
  which is the gated oracle (pinned on its own in test_oracle_pins.py);
* the state and outputs equal explicit products of the Dk x Dk transition matrices;
* the state hands off between two halves of a sequence;
* the backward equals central finite differences of the forward;
* the WY chunk form equals the recurrence for every chunk size, the ragged tail included.

Every planted mistake in test_planted_mistake_is_caught must fail at least one pin.
"""
import types

import numpy as np
import pytest

import oracle
from oracle import deltanet as DN

RNG = np.random.default_rng(4321)


def rnd(*shape):
    return RNG.standard_normal(shape)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def betas(*shape):
    return 1.0 / (1.0 + np.exp(-rnd(*shape)))


def rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ------------------------------------------------------------------------------- pins
def pin_beta_zero_freezes_the_state(D):
    B, H, L, Dk, Dv = 1, 2, 9, 4, 3
    q, k, v, h0 = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    o, hT = D.deltanet_fwd(q, k, v, np.zeros((B, H, L)), h0, 0.5)
    assert rel(hT, h0) < 1e-14
    assert rel(o, 0.5 * q @ h0) < 1e-14


def pin_unit_key_full_step_fits_the_value(D):
    B, H, Dk, Dv = 2, 1, 6, 5
    k = unit_rows(rnd(B, H, 1, Dk))
    v, h0 = rnd(B, H, 1, Dv), rnd(B, H, Dk, Dv)
    _, S = D.deltanet_fwd(rnd(B, H, 1, Dk), k, v, np.ones((B, H, 1)), h0)
    assert rel(np.einsum("bhi,bhij->bhj", k[:, :, 0], S), v[:, :, 0]) < 1e-13
    # directions orthogonal to k keep their old answers
    x = rnd(B, H, Dk)
    x = x - np.einsum("bhi,bhi->bh", x, k[:, :, 0])[..., None] * k[:, :, 0]
    assert rel(np.einsum("bhi,bhij->bhj", x, S), np.einsum("bhi,bhij->bhj", x, h0)) < 1e-12


def pin_orthonormal_keys_recall_and_overwrite(D):
    Dk, Dv, n = 8, 3, 6
    basis = np.linalg.qr(rnd(Dk, Dk))[0].T           # rows: an orthonormal basis
    keys = basis[:n]
    vals = rnd(n, Dv)
    b1 = betas(n)
    # write each key once (strength b1), then rewrite key 0 and key 3 with new values
    new = rnd(2, Dv)
    b2 = betas(2)
    k = np.concatenate([keys, keys[[0, 3]]])[None, None]
    v = np.concatenate([vals, new])[None, None]
    beta = np.concatenate([b1, b2])[None, None]
    _, S = D.deltanet_fwd(rnd(1, 1, n + 2, Dk), k, v, beta)
    got = keys @ S[0, 0]
    want = b1[:, None] * vals
    # rewriting moves the stored answer toward the new value by beta: (1 - b) old + b new
    want[0] = (1 - b2[0]) * want[0] + b2[0] * new[0]
    want[3] = (1 - b2[1]) * want[3] + b2[1] * new[1]
    assert rel(got, want) < 1e-12
    # with full strength every stored value comes back exactly
    _, S1 = D.deltanet_fwd(rnd(1, 1, n, Dk), keys[None, None], vals[None, None], np.ones((1, 1, n)))
    assert rel(keys @ S1[0, 0], vals) < 1e-12


def pin_step_is_a_gradient_step_by_finite_differences(D):
    Dk, Dv = 3, 2
    k, v, S0 = rnd(1, 1, 1, Dk), rnd(1, 1, 1, Dv), rnd(1, 1, Dk, Dv)
    b = 0.37

    def loss(S):
        r = k[0, 0, 0] @ S - v[0, 0, 0]
        return 0.5 * float(r @ r)

    grad = np.zeros((Dk, Dv))
    eps = 1e-6
    for i in range(Dk):
        for j in range(Dv):
            E = np.zeros((Dk, Dv))
            E[i, j] = eps
            grad[i, j] = (loss(S0[0, 0] + E) - loss(S0[0, 0] - E)) / (2 * eps)
    _, S1 = D.deltanet_fwd(rnd(1, 1, 1, Dk), k, v, np.full((1, 1, 1), b), S0)
    assert rel(S1[0, 0], S0[0, 0] - b * grad) < 1e-9


def pin_orthogonal_keys_reduce_to_linear_attention(D):
    B, H, L, Dk, Dv = 2, 2, 7, 12, 5
    k = np.stack([np.stack([np.linalg.qr(rnd(Dk, Dk))[0].T[:L] * RNG.uniform(0.5, 2.0, (L, 1))
                            for _ in range(H)]) for _ in range(B)])
    q, v, beta = rnd(B, H, L, Dk), rnd(B, H, L, Dv), betas(B, H, L)
    o, S = D.deltanet_fwd(q, k, v, beta, None, 0.3)
    # each key is orthogonal to every earlier one, so k_t S_{t-1} = 0 and the step only adds
    # beta_t k_t^T v_t, whatever the key's norm
    ro, rS = oracle.gla_fwd(q, k, v, None, beta, None, 0.3)
    assert rel(o, ro) < 1e-12
    assert rel(S, rS) < 1e-12


def pin_explicit_transition_products(D):
    B, H, L, Dk, Dv = 1, 2, 6, 4, 3
    q, k, v, beta, h0 = rnd(B, H, L, Dk), rnd(B, H, L, Dk), rnd(B, H, L, Dv), betas(B, H, L), rnd(B, H, Dk, Dv)
    o, S = D.deltanet_fwd(q, k, v, beta, h0, 0.8)
    for b in range(B):
        for h in range(H):
            M = [np.eye(Dk) - beta[b, h, t] * np.outer(k[b, h, t], k[b, h, t]) for t in range(L)]
            for t in range(L):
                # S_t = M_t ... M_1 h0 + sum_{s<=t} M_t ... M_{s+1} beta_s k_s^T v_s
                P = np.eye(Dk)
                for s in range(t + 1):
                    P = M[s] @ P
                St = P @ h0[b, h]
                for s in range(t + 1):
                    R = np.eye(Dk)
                    for u in range(s + 1, t + 1):
                        R = M[u] @ R
                    St = St + beta[b, h, s] * R @ np.outer(k[b, h, s], v[b, h, s])
                assert rel(o[b, h, t], 0.8 * q[b, h, t] @ St) < 1e-12
            assert rel(S[b, h], St) < 1e-12


def pin_state_hand_off(D):
    B, H, L, Dk, Dv = 1, 3, 20, 5, 4
    q, k, v, beta, h0 = rnd(B, H, L, Dk), unit_rows(rnd(B, H, L, Dk)), rnd(B, H, L, Dv), betas(B, H, L), \
        rnd(B, H, Dk, Dv)
    o, S = D.deltanet_fwd(q, k, v, beta, h0)
    o1, S1 = D.deltanet_fwd(q[:, :, :8], k[:, :, :8], v[:, :, :8], beta[:, :, :8], h0)
    o2, S2 = D.deltanet_fwd(q[:, :, 8:], k[:, :, 8:], v[:, :, 8:], beta[:, :, 8:], S1)
    assert rel(np.concatenate([o1, o2], axis=2), o) < 1e-13
    assert rel(S2, S) < 1e-13


def pin_backward_matches_finite_differences(D):
    B, H, L, Dk, Dv = 1, 2, 5, 3, 2
    x = {"q": rnd(B, H, L, Dk), "k": rnd(B, H, L, Dk) * 0.7, "v": rnd(B, H, L, Dv), "beta": betas(B, H, L),
         "h0": rnd(B, H, Dk, Dv)}
    dO, dhT = rnd(B, H, L, Dv), rnd(B, H, Dk, Dv)
    scale = 0.9

    def loss(xx):
        o, S = D.deltanet_fwd(xx["q"], xx["k"], xx["v"], xx["beta"], xx["h0"], scale)
        return float((o * dO).sum() + (S * dhT).sum())

    g = D.deltanet_bwd(x["q"], x["k"], x["v"], x["beta"], x["h0"], dO, dhT, scale)
    eps = 1e-6
    for name, gname in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("h0", "dh0")):
        num = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            xp = {n: a.copy() for n, a in x.items()}
            xm = {n: a.copy() for n, a in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            num[idx] = (loss(xp) - loss(xm)) / (2 * eps)
        assert rel(g[gname], num) < 1e-7, gname


def pin_chunk_form_equals_the_recurrence(D):
    B, H, L, Dk, Dv = 2, 2, 37, 6, 5
    q, k, v, beta, h0 = rnd(B, H, L, Dk), unit_rows(rnd(B, H, L, Dk)), rnd(B, H, L, Dv), betas(B, H, L), \
        rnd(B, H, Dk, Dv)
    o, S = D.deltanet_fwd(q, k, v, beta, h0, 0.6)
    for chunk in (1, 3, 4, 16, 37, 64):
        oc, Sc = D.deltanet_fwd_chunkwise(q, k, v, beta, h0, 0.6, chunk)
        assert rel(oc, o) < 1e-11, chunk
        assert rel(Sc, S) < 1e-11, chunk


PINS = [pin_beta_zero_freezes_the_state, pin_unit_key_full_step_fits_the_value,
        pin_orthonormal_keys_recall_and_overwrite, pin_step_is_a_gradient_step_by_finite_differences,
        pin_orthogonal_keys_reduce_to_linear_attention, pin_explicit_transition_products, pin_state_hand_off,
        pin_backward_matches_finite_differences, pin_chunk_form_equals_the_recurrence]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__[4:])
def test_pin(pin):
    pin(DN)


# ------------------------------------------------------------- planted mistakes
# (text in oracle/deltanet.py, its replacement): a residual of the wrong sign, a dropped
# writing strength, the delta correction dropped (plain linear attention), the output read
# from the old state, a wrong sign in dbeta, the second dk term dropped, the state gradient
# not carried through the transition, dv without beta, the diagonal dropped from the chunk
# form's causal mask, and the wrong sign in its triangular system.
MUTANTS = [
    ('resid = np.einsum("bhi,bhij->bhj", kt, S) - vt', 'resid = np.einsum("bhi,bhij->bhj", kt, S) + vt'),
    ('S = S - bt[..., None, None] * np.einsum("bhi,bhj->bhij", kt, resid)',
     'S = S - np.einsum("bhi,bhj->bhij", kt, resid)'),
    ('resid = np.einsum("bhi,bhij->bhj", kt, S) - vt', 'resid = -vt'),
    ('        S = S - bt[..., None, None] * np.einsum("bhi,bhj->bhij", kt, resid)\n'
     '        o[:, :, t] = scale * np.einsum("bhi,bhij->bhj", q[:, :, t], S)',
     '        o[:, :, t] = scale * np.einsum("bhi,bhij->bhj", q[:, :, t], S)\n'
     '        S = S - bt[..., None, None] * np.einsum("bhi,bhj->bhij", kt, resid)'),
    ('dbeta[:, :, t] = np.einsum(', 'dbeta[:, :, t] = -np.einsum('),
    ('np.einsum("bhj,bhij->bhi", kG, Sp))', '0.0 * np.einsum("bhj,bhij->bhi", kG, Sp))'),
    ('G = G - bt[..., None, None] * np.einsum("bhi,bhj->bhij", kt, kG)', 'G = G'),
    ('dv[:, :, t] = bt[..., None] * kG', 'dv[:, :, t] = kG'),
    ('QK = np.tril(np.einsum("bhti,bhsi->bhts", Q, K))', 'QK = np.tril(np.einsum("bhti,bhsi->bhts", Q, K), -1)'),
    ('A = np.eye(n) + np.tril(', 'A = np.eye(n) - np.tril('),
]


def _mutant_module(i):
    path = DN.__file__
    src = open(path).read()
    old, new = MUTANTS[i]
    assert src.count(old) == 1, old
    mod = types.ModuleType(f"deltanet_mutant_{i}")
    exec(compile(src.replace(old, new), path, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("i", range(len(MUTANTS)))
def test_planted_mistake_is_caught(i):
    mod = _mutant_module(i)
    caught = []
    for pin in PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {i} passed every pin"


def test_input_recipe():
    """The generator's keys have unit norm up to bf16 rounding and beta lies in (0, 1)."""
    import torch
    from linear_rnn_b200 import inputs as I
    x = I.make_deltanet_inputs(2, 3, 100, 64, 128, "bf16", seed=1, h0_std=0.5)
    n = x["k"].float().norm(dim=-1)
    assert torch.all((n - 1).abs() < 1e-2)
    assert torch.all(x["beta"] > 0) and torch.all(x["beta"] < 1)
    assert x["q"].dtype == torch.bfloat16 and x["beta"].dtype == torch.float32
    assert x["h0"].shape == (2, 3, 64, 128)
