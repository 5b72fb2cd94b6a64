"""Float64 CPU oracle for the delta rule (DeltaNet) -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this module.
The CUDA library and its Python binding never import it.

Source: the talk summary "Hardware-Efficient Training of Linear Attention Models", its
DeltaNet sections (22:36 and 31:16). There the state is an associative memory that a
per-token writing strength beta_t updates. The update is one stochastic-gradient step, with
step size beta_t, on the linear-regression loss between key and value. Its transition
matrix is the identity plus a rank-one term, and the chunkwise form goes through the WY
representation.

Conventions (the same row form as the gated linear attention oracle): the state S is
[Dk, Dv], and a key or query is a row vector, so the memory's answer to a key k is k S.
The loss of token t is l_t(S) = 1/2 ||k_t S - v_t||^2, with gradient k_t^T (k_t S - v_t). One
step of size beta_t from S_{t-1} gives

    S_t = S_{t-1} - beta_t k_t^T (k_t S_{t-1} - v_t) = (I - beta_t k_t^T k_t) S_{t-1} + beta_t k_t^T v_t,

and the output reads the updated state, o_t = scale * q_t S_t, as in the gated form. The
pages do not say whether keys are normalised. This oracle takes k as given; the input recipe
passes unit-norm keys, which keep the transition's spectrum in [1 - beta, 1].

Functions:
- deltanet_fwd: the token recurrence above. This is the definition.
- deltanet_bwd: back-propagation through time of that recurrence.
- deltanet_fwd_chunkwise: the chunk form through the WY representation, which a chunkwise
  kernel follows. It is pinned to deltanet_fwd, not used as a reference on its own.

Parity pins (tests/test_oracle_deltanet.py): beta = 0 freezes the state; unit keys with
beta = 1 make k_t S_t = v_t exactly; an orthonormal key set recalls and overwrites each value
exactly; the step equals a finite-difference gradient step of l_t; orthogonal keys from a
zero state reduce to linear attention with input gate beta (the gated oracle); the state is
the explicit product of the Dk x Dk transition matrices; the backward matches central finite
differences; and the chunk form equals the recurrence for every chunk size.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import numpy as np


def _f64(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    if hasattr(x, "detach"):   # torch tensor
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def deltanet_fwd(q, k, v, beta, h0=None, scale: float = 1.0) -> Tuple[np.ndarray, np.ndarray]:
    """o [B,H,L,Dv] and the final state [B,H,Dk,Dv], float64, by the token recurrence.
    q, k [B,H,L,Dk]; v [B,H,L,Dv]; beta [B,H,L]; h0 [B,H,Dk,Dv] or None (zero)."""
    q, k, v, beta, h0 = map(_f64, (q, k, v, beta, h0))
    B, H, L, Dk = k.shape
    Dv = v.shape[-1]
    S = np.zeros((B, H, Dk, Dv)) if h0 is None else h0.copy()
    o = np.zeros((B, H, L, Dv))
    for t in range(L):
        kt, vt, bt = k[:, :, t], v[:, :, t], beta[:, :, t]
        # residual of the memory's answer to k_t: k_t S - v_t
        resid = np.einsum("bhi,bhij->bhj", kt, S) - vt
        # S <- S - beta_t k_t^T (k_t S - v_t)
        S = S - bt[..., None, None] * np.einsum("bhi,bhj->bhij", kt, resid)
        o[:, :, t] = scale * np.einsum("bhi,bhij->bhj", q[:, :, t], S)
    return o, S


def deltanet_bwd(q, k, v, beta, h0=None, dO=None, dhT=None, scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Gradients of sum(dO * o) + sum(dhT * S_L) by back-propagation through time, float64:
    dict dq, dk, dv, dbeta, dh0.

    Per token, with r_t = v_t - k_t S_{t-1} and S_t = S_{t-1} + beta_t k_t^T r_t, and with G the
    gradient reaching S_t (from later tokens, plus scale q_t^T dO_t from o_t):
      dq_t = scale dO_t S_t^T
      dbeta_t = k_t G r_t^T
      dv_t = beta_t k_t G                      (r_t enters S_t through beta_t k_t^T r_t)
      dk_t = beta_t r_t G^T - beta_t (k_t G) S_{t-1}^T
      G <- G - beta_t k_t^T (k_t G)            (the transition I - beta_t k_t^T k_t is symmetric)
    """
    q, k, v, beta, h0, dO, dhT = map(_f64, (q, k, v, beta, h0, dO, dhT))
    B, H, L, Dk = k.shape
    Dv = v.shape[-1]
    S0 = np.zeros((B, H, Dk, Dv)) if h0 is None else h0
    dO = np.zeros((B, H, L, Dv)) if dO is None else dO
    # the states S_0 .. S_L of the forward, kept for the reverse walk
    states = np.zeros((L + 1, B, H, Dk, Dv))
    states[0] = S0
    for t in range(L):
        kt = k[:, :, t]
        resid = v[:, :, t] - np.einsum("bhi,bhij->bhj", kt, states[t])
        states[t + 1] = states[t] + beta[:, :, t][..., None, None] * np.einsum("bhi,bhj->bhij", kt, resid)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dbeta = np.zeros_like(beta)
    G = np.zeros((B, H, Dk, Dv)) if dhT is None else dhT.copy()
    for t in range(L - 1, -1, -1):
        qt, kt, bt = q[:, :, t], k[:, :, t], beta[:, :, t]
        St, Sp = states[t + 1], states[t]
        dq[:, :, t] = scale * np.einsum("bhj,bhij->bhi", dO[:, :, t], St)
        G = G + scale * np.einsum("bhi,bhj->bhij", qt, dO[:, :, t])
        resid = v[:, :, t] - np.einsum("bhi,bhij->bhj", kt, Sp)
        kG = np.einsum("bhi,bhij->bhj", kt, G)                       # k_t G  [B,H,Dv]
        dbeta[:, :, t] = np.einsum("bhj,bhj->bh", kG, resid)
        dv[:, :, t] = bt[..., None] * kG
        dk[:, :, t] = bt[..., None] * (np.einsum("bhij,bhj->bhi", G, resid) -
                                       np.einsum("bhj,bhij->bhi", kG, Sp))
        G = G - bt[..., None, None] * np.einsum("bhi,bhj->bhij", kt, kG)
    return {"dq": dq, "dk": dk, "dv": dv, "dbeta": dbeta, "dh0": G}


def deltanet_fwd_chunkwise(q, k, v, beta, h0=None, scale: float = 1.0,
                           chunk: int = 64) -> Tuple[np.ndarray, np.ndarray]:
    """The same o and final state by chunks of `chunk` tokens (the last one ragged) through
    the WY representation.

    Within a chunk that starts from state S, the product of the transitions up to token t is
    I - sum_{i<=t} k_i^T w_i, and the state the chunk's own writes add is sum_{i<=t} k_i^T u_i,
    where
        w_t = beta_t (k_t - sum_{i<t} (k_t . k_i) w_i),   u_t = beta_t (v_t - sum_{i<t} (k_t . k_i) u_i).
    Stacked as rows, W = T K and U = T V with T = (I + strict_lower(diag(beta) K K^T))^{-1} diag(beta),
    one unit-lower-triangular solve per chunk. Then
        O = scale (Q S + lower(Q K^T) (U - W S))    (lower includes the diagonal)
        S <- S + K^T (U - W S).
    """
    q, k, v, beta, h0 = map(_f64, (q, k, v, beta, h0))
    B, H, L, Dk = k.shape
    Dv = v.shape[-1]
    S = np.zeros((B, H, Dk, Dv)) if h0 is None else h0.copy()
    o = np.zeros((B, H, L, Dv))
    for c0 in range(0, L, chunk):
        c1 = min(L, c0 + chunk)
        n = c1 - c0
        Q, K, V, bet = q[:, :, c0:c1], k[:, :, c0:c1], v[:, :, c0:c1], beta[:, :, c0:c1]
        KK = np.einsum("bhti,bhsi->bhts", K, K)
        A = np.eye(n) + np.tril(bet[..., None] * KK, -1)
        W = np.linalg.solve(A, bet[..., None] * K)
        U = np.linalg.solve(A, bet[..., None] * V)
        X = U - np.einsum("bhti,bhij->bhtj", W, S)                  # U - W S  [B,H,n,Dv]
        QK = np.tril(np.einsum("bhti,bhsi->bhts", Q, K))
        o[:, :, c0:c1] = scale * (np.einsum("bhti,bhij->bhtj", Q, S) + np.einsum("bhts,bhsj->bhtj", QK, X))
        S = S + np.einsum("bhti,bhtj->bhij", K, X)
    return o, S
