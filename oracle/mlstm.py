"""Float64 CPU oracle for the mLSTM cell (matrix memory with an exponential input gate, a
normaliser state and a max-stabiliser) -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import this module.
The CUDA library and its Python binding never import it.

Source: "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
(abstract) names mLSTM, the matrix-memory cell of the xLSTM family, as the model its kernels
speed up; the pages print no formula for it. The reading taken here is the published mLSTM
cell, in the row form the gated linear attention oracle uses (state C is [Dk, Dv], keys and
queries are row vectors), per (batch, head):

    g_t   = log of the forget gate (<= 0),  i~_t = log of the exponential input gate (any real)
    m_t   = max(g_t + m_{t-1}, i~_t),            m_{-1} = 0         (the max-stabiliser)
    i'_t  = exp(i~_t - m_t),  f'_t = exp(g_t + m_{t-1} - m_t)
    C_t   = f'_t C_{t-1} + i'_t k_t^T v_t,       n_t = f'_t n_{t-1} + i'_t k_t,   C_{-1}, n_{-1} = 0
    h_t   = (scale q_t) C_t / max(|(scale q_t) . n_t|, exp(-m_t))

The readout uses the updated state, as in the gated form. The stabilised states are the plain
ones times exp(-m_t) (C_t = exp(m_t) C~_t by induction), so h_t equals the unstabilised
    h_t = (scale q_t) C_t / max(|(scale q_t) . n_t|, 1),  C_t = e^{g_t} C_{t-1} + e^{i~_t} k_t^T v_t
exactly: the stabiliser only keeps exp(i~) inside the floating-point range. `scale` on the
query is the xLSTM key scaling moved to the other side of the bilinear products.

Functions:
- mlstm_fwd: the stabilised token recurrence above. This is the definition.
- mlstm_bwd: its gradients. h = num / N with num_t = (scale q_t) C_t and den_t = (scale q_t)
  . n_t both gated linear attention outputs (value v, resp. a value of ones) with the per-head
  log-decay g and the input gate e^{i~}, and N_t = max(|den_t|, 1). So dnum = dh / N,
  dden = -(dh . h) / N * sign(den) where |den| > 1 (0 where the bound 1 is active), and the
  gated oracle's back-propagation through time (oracle.gla_bwd) carries dnum and dden back to
  q, k, v, g and the input gate; d i~ = d(input gate) * e^{i~}. Every exponential is taken
  relative to the head's largest i~ (a constant shift that cancels in h, like m_t).

Pins (tests/test_oracle_mlstm.py): the unstabilised recurrence, the ratio limit for input gates
far beyond exp's range, the gated oracle with values v and ones, a brute-force quadratic form
with explicit products of decays, the single-token closed form on both sides of the bound,
invariance of h to a shift of i~ where |den| > 1, central finite differences on every input,
and planted mistakes.
"""
from __future__ import annotations

from typing import Dict, Tuple

import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):   # torch tensor
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def mlstm_fwd(q, k, v, g, itil, scale: float = 1.0) -> Tuple[np.ndarray, Dict[str, np.ndarray]]:
    """h [B,H,L,Dv] by the stabilised token recurrence, float64, and the final stabilised
    state {"C": [B,H,Dk,Dv], "n": [B,H,Dk], "m": [B,H]}.
    q, k [B,H,L,Dk]; v [B,H,L,Dv]; g (log forget gate), itil (log input gate) [B,H,L]."""
    q, k, v, g, itil = map(_f64, (q, k, v, g, itil))
    B, H, L, Dk = k.shape
    Dv = v.shape[-1]
    C = np.zeros((B, H, Dk, Dv))
    n = np.zeros((B, H, Dk))
    m_prev = np.zeros((B, H))
    h = np.zeros((B, H, L, Dv))
    for t in range(L):
        gt, it = g[:, :, t], itil[:, :, t]
        m = np.maximum(gt + m_prev, it)
        ip = np.exp(it - m)
        fp = np.exp(gt + m_prev - m)
        kt = k[:, :, t]
        C = fp[..., None, None] * C + ip[..., None, None] * np.einsum("bhi,bhj->bhij", kt, v[:, :, t])
        n = fp[..., None] * n + ip[..., None] * kt
        qs = scale * q[:, :, t]
        num = np.einsum("bhi,bhij->bhj", qs, C)
        den = np.einsum("bhi,bhi->bh", qs, n)
        h[:, :, t] = num / np.maximum(np.abs(den), np.exp(-m))[..., None]
        m_prev = m
    return h, {"C": C, "n": n, "m": m_prev}


def mlstm_bwd(q, k, v, g, itil, dh, scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Gradients of sum(dh * h) w.r.t. q, k, v, g and itil, float64 (dict dq, dk, dv, dg, ditil)."""
    import oracle
    q, k, v, g, itil, dh = map(_f64, (q, k, v, g, itil, dh))
    B, H, L, Dk = k.shape
    # a per-head constant shift of the exponent (it cancels in h): every e^{i~ - c} <= 1
    c = itil.max(axis=2, keepdims=True) if L > 0 else np.zeros((B, H, 1))
    ig = np.exp(itil - c)
    ones = np.ones((B, H, L, 1))
    num, _ = oracle.gla_fwd(q, k, v, g, ig, None, scale)        # e^{-c} (scale q_t) C_t
    den, _ = oracle.gla_fwd(q, k, ones, g, ig, None, scale)     # e^{-c} (scale q_t) . n_t
    den = den[..., 0]
    bound = np.exp(-c)                                          # e^{-c} times the bound 1
    N = np.maximum(np.abs(den), bound)
    h = num / N[..., None]
    dnum = dh / N[..., None]
    active = np.abs(den) > bound
    dden = np.where(active, -np.einsum("bhtj,bhtj->bht", dh, h) / N * np.sign(den), 0.0)
    r1 = oracle.gla_bwd(q, k, v, g, ig, None, dnum, None, scale)
    r2 = oracle.gla_bwd(q, k, ones, g, ig, None, dden[..., None], None, scale)
    return {"dq": r1["dq"] + r2["dq"], "dk": r1["dk"] + r2["dk"], "dv": r1["dv"],
            "dg": r1["dg"] + r2["dg"], "ditil": (r1["di"] + r2["di"]) * ig}
