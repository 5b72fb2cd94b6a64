"""Float64 numpy restatement of the chunkwise equations, used only by the tests.

It restates, step by step, the algebra the CUDA kernels implement, so that the tests
can check that algebra against the token-recurrence oracle in exact-ish arithmetic:

* in-chunk log-cumsum of the gate, b_t = sum of g over the chunk up to t, and the
  chunk total Gamma (the chunk ("trunk") decomposition of the talk summary "Hardware-
  Efficient Training of Linear Attention Models", section 11:58);
* the inter-chunk state pass S_c = diag(e^Gamma) S_{c-1} + (k * e^(Gamma-b))^T V, a
  matrix product over the chunk (same section: states only at chunk boundaries,
  K_block^T V_block as a matmul);
* the output o = scale [ (q * e^b) S_{c-1} + masked intra-chunk product ], where the
  intra-chunk part is tiled into sub-tiles and each tile pair uses a reference point in
  log space so that no exponential exceeds the tile's span (off-diagonal pair: the last
  row of the key tile; diagonal pair: the first row of the tile);
* the backward: reverse state-gradient pass G_{c-1} = diag(e^Gamma) G_c +
  scale (q * e^b)^T dO, per-chunk dq/dk/dv, and dg as the reverse cumulative sum over
  the whole sequence of q*dq - k*dk plus the final-state term rowsum(dhT * hT).

This module shares nothing with the oracle (oracle/) or with the CUDA code.
"""
from __future__ import annotations

import numpy as np


def _prep(q, k, v, g, ig, h0):
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    if ig is not None:
        k = k * np.asarray(ig, np.float64)[..., None]
    if g is None:
        G = np.zeros((B, H, L, Dk))
    else:
        g = np.asarray(g, np.float64)
        G = g if g.ndim == 4 else np.broadcast_to(g[..., None], (B, H, L, Dk)).copy()
    S0 = np.zeros((B, H, Dk, Dv)) if h0 is None else np.asarray(h0, np.float64).copy()
    return q, k, v, G, S0


def _intra(qc, kc, b, sub):
    """Masked intra-chunk matrix A[t,s] = sum_d q_td k_sd e^(b_td - b_sd), s <= t,
    by sub-tiles with log-space reference points. qc,kc,b: [n, Dk] for one head."""
    n = qc.shape[0]
    A = np.zeros((n, n))
    for i0 in range(0, n, sub):
        i1 = min(i0 + sub, n)
        for j0 in range(0, i1, sub):
            j1 = min(j0 + sub, n)
            if j1 <= i0:   # key tile strictly before the query tile
                r = b[j1 - 1]
                A[i0:i1, j0:j1] = (qc[i0:i1] * np.exp(b[i0:i1] - r)) @ (kc[j0:j1] * np.exp(r - b[j0:j1])).T
            else:          # diagonal tile
                r = b[i0]
                blk = (qc[i0:i1] * np.exp(b[i0:i1] - r)) @ (kc[j0:j1] * np.exp(r - b[j0:j1])).T
                A[i0:i1, j0:j1] = np.tril(blk)
    return A


def chunk_fwd(q, k, v, g=None, ig=None, h0=None, scale=1.0, C=64, sub=16):
    q, k, v, G, S0 = _prep(q, k, v, g, ig, h0)
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    o = np.zeros((B, H, L, Dv))
    hT = np.zeros((B, H, Dk, Dv))
    for bb in range(B):
        for hh in range(H):
            S = S0[bb, hh].copy()
            for c0 in range(0, L, C):
                c1 = min(c0 + C, L)
                b = np.cumsum(G[bb, hh, c0:c1], axis=0)
                gam = b[-1]
                qc, kc, vc = q[bb, hh, c0:c1], k[bb, hh, c0:c1], v[bb, hh, c0:c1]
                A = _intra(qc, kc, b, sub)
                o[bb, hh, c0:c1] = scale * ((qc * np.exp(b)) @ S + A @ vc)
                S = np.exp(gam)[:, None] * S + (kc * np.exp(gam - b)).T @ vc
            hT[bb, hh] = S
    return o, hT


def chunk_bwd(q, k, v, g=None, ig=None, h0=None, dO=None, dhT=None, scale=1.0, C=64, sub=16):
    """Returns dq, dk, dv, dg (same shape as g, or None), di (or None), dh0."""
    ig_arr = None if ig is None else np.asarray(ig, np.float64)
    k_raw = np.asarray(k, np.float64)
    q, k, v, G, S0 = _prep(q, k, v, g, ig, h0)
    dO = np.asarray(dO, np.float64)
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    dq = np.zeros_like(q)
    dkp = np.zeros_like(k)
    dv = np.zeros_like(v)
    dh0 = np.zeros((B, H, Dk, Dv))
    dB = np.zeros_like(q)
    for bb in range(B):
        for hh in range(H):
            # forward: states before each chunk
            S = S0[bb, hh].copy()
            starts = list(range(0, L, C))
            Sprev = []
            for c0 in starts:
                c1 = min(c0 + C, L)
                b = np.cumsum(G[bb, hh, c0:c1], axis=0)
                gam = b[-1]
                Sprev.append(S.copy())
                S = np.exp(gam)[:, None] * S + (k[bb, hh, c0:c1] * np.exp(gam - b)).T @ v[bb, hh, c0:c1]
            hT = S
            Gs = np.zeros((Dk, Dv)) if dhT is None else np.asarray(dhT, np.float64)[bb, hh].copy()
            for ci in reversed(range(len(starts))):
                c0 = starts[ci]
                c1 = min(c0 + C, L)
                b = np.cumsum(G[bb, hh, c0:c1], axis=0)
                gam = b[-1]
                qc, kc, vc, dOc = q[bb, hh, c0:c1], k[bb, hh, c0:c1], v[bb, hh, c0:c1], dO[bb, hh, c0:c1]
                A = scale * _intra(qc, kc, b, sub)                   # A[t,s]
                dA = scale * np.tril(dOc @ vc.T)                      # dA[t,s], s <= t
                # sum_s dA_ts k_s e^(b_t - b_s) and sum_t dA_ts q_t e^(b_t - b_s), tiled
                n = c1 - c0
                dq_intra = np.zeros((n, Dk))
                dk_intra = np.zeros((n, Dk))
                for i0 in range(0, n, sub):
                    i1 = min(i0 + sub, n)
                    for j0 in range(0, i1, sub):
                        j1 = min(j0 + sub, n)
                        r = b[j1 - 1] if j1 <= i0 else b[i0]
                        qh = qc[i0:i1] * np.exp(b[i0:i1] - r)
                        kh = kc[j0:j1] * np.exp(r - b[j0:j1])
                        dAt = dA[i0:i1, j0:j1]
                        dq_intra[i0:i1] += np.exp(b[i0:i1] - r) * (dAt @ (kc[j0:j1] * np.exp(r - b[j0:j1])))
                        dk_intra[j0:j1] += np.exp(r - b[j0:j1]) * (dAt.T @ qh)
                        del kh
                dq[bb, hh, c0:c1] = np.exp(b) * (scale * dOc @ Sprev[ci].T) + dq_intra
                khat = kc * np.exp(gam - b)
                dkp[bb, hh, c0:c1] = np.exp(gam - b) * (vc @ Gs.T) + dk_intra
                dv[bb, hh, c0:c1] = khat @ Gs + A.T @ dOc
                Gs = np.exp(gam)[:, None] * Gs + scale * (qc * np.exp(b)).T @ dOc
            dh0[bb, hh] = Gs
            dB[bb, hh] = q[bb, hh] * dq[bb, hh] - k[bb, hh] * dkp[bb, hh]
            if dhT is not None and L > 0:
                dB[bb, hh, L - 1] += (np.asarray(dhT, np.float64)[bb, hh] * hT).sum(axis=1)
    dgk = np.flip(np.cumsum(np.flip(dB, axis=2), axis=2), axis=2)
    dg = None
    if g is not None:
        dg = dgk if np.asarray(g).ndim == 4 else dgk.sum(axis=-1)
    di = None
    dk_out = dkp
    if ig_arr is not None:
        di = (k_raw * dkp).sum(axis=-1)
        dk_out = dkp * ig_arr[..., None]
    return {"dq": dq, "dk": dk_out, "dv": dv, "dg": dg, "di": di, "dh0": dh0}
