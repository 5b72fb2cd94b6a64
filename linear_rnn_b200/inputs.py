"""Seeded synthetic inputs for the chunkwise gated-linear-attention workloads.

This module is shared by the CUDA path's tests/bench and by the oracle's tests. It
holds no arithmetic of the method itself: it only draws random tensors with the
shapes and distributions of the five workloads and rounds them to the I/O dtype.

Workloads (sizes from the method's published configurations):
  c1  ungated causal linear attention, fp32, B=1 H=1 L=256 Dk=Dv=64, C=64
  c2  GLA forward, bf16, B=8 H=16 L=2048 Dk=Dv=64, k pre-scaled by Dk^-1/2, scale=1, C=64
  c3  GLA forward+backward, bf16, B=4 H=16 L=4096 Dk=128 Dv=256, C=64
  c4  long-context GLA forward, bf16, B=1 H=8 L=65536 Dk=Dv=128, h0 ~ 0.1 N(0,1), C=256
  c5  scalar-gate mLSTM-style, bf16, B=2 H=8 L=8192 Dk=Dv=256, f=logsigmoid(N(3,1)),
      input gate i=sigmoid(N(0,1)) on k, forward+backward, C=64

Draw order from one torch CPU generator seeded with `seed`: q, k, v, gate
pre-activation, [h0], [input-gate pre-activation], [dO]; every draw is a standard
normal in fp32, then rounded (round-to-nearest-even) to bf16 where the I/O dtype is
bf16. Gates and h0 stay fp32.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, Optional

import torch

GATE_NONE, GATE_PER_KEY, GATE_PER_HEAD = 0, 1, 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    Dk: int
    Dv: int
    chunk: int
    dtype: str            # "f32" or "bf16"
    gate: int             # GATE_NONE / GATE_PER_KEY / GATE_PER_HEAD
    backward: bool
    scale: float
    k_prescale: float = 1.0   # k drawn as N(0,1) * k_prescale
    h0_std: float = 0.0       # 0 -> no initial state
    input_gate: bool = False
    gate_mean: float = 0.0    # mean of the gate pre-activation normal
    gate_div: float = 1.0     # gate = logsigmoid(pre) / gate_div

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def tokens(self) -> int:
        return self.B * self.L


WORKLOADS: Dict[str, Workload] = {
    "c1": Workload("c1", 1, 1, 256, 64, 64, 64, "f32", GATE_NONE, False, 64 ** -0.5),
    "c2": Workload("c2", 8, 16, 2048, 64, 64, 64, "bf16", GATE_PER_KEY, False, 1.0,
                   k_prescale=64 ** -0.5, gate_div=16.0),
    "c3": Workload("c3", 4, 16, 4096, 128, 256, 64, "bf16", GATE_PER_KEY, True, 128 ** -0.5,
                   gate_div=16.0),
    "c4": Workload("c4", 1, 8, 65536, 128, 128, 256, "bf16", GATE_PER_KEY, False, 128 ** -0.5,
                   h0_std=0.1, gate_div=16.0),
    "c5": Workload("c5", 2, 8, 8192, 256, 256, 64, "bf16", GATE_PER_HEAD, True, 256 ** -0.5,
                   input_gate=True, gate_mean=3.0, gate_div=1.0),
}


def _round_io(x: torch.Tensor, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return x.to(torch.bfloat16)
    if dtype == "f32":
        return x.contiguous()
    raise ValueError(f"unknown io dtype {dtype!r}")


# Single-token decode step from a given state at a serving batch: 64 sequences x 16 heads,
# Dk=128 Dv=256, bf16 I/O, per-key log-gate logsigmoid(N(0,1))/16 (the forward workloads'
# gates), state ~ N(0, 1) fp32 (1024 states of 128 x 256 = 128 MiB, more than L2).
DECODE = Workload("decode", 64, 16, 1, 128, 256, 64, "bf16", GATE_PER_KEY, False, 128 ** -0.5,
                  h0_std=1.0, gate_div=16.0)


def make_inputs(w: Workload, seed: int = 0) -> Dict[str, Optional[torch.Tensor]]:
    """Draw the workload's inputs on the CPU. Returns a dict of contiguous tensors:
    q, k [B,H,L,Dk]; v [B,H,L,Dv] (io dtype); g ([B,H,L,Dk] or [B,H,L] fp32, or None);
    h0 [B,H,Dk,Dv] fp32 or None; igate [B,H,L] fp32 or None; dO [B,H,L,Dv] io dtype or None.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    B, H, L, Dk, Dv = w.B, w.H, w.L, w.Dk, w.Dv

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = _round_io(randn(B, H, L, Dk), w.dtype)
    k = _round_io(randn(B, H, L, Dk) * w.k_prescale, w.dtype)
    v = _round_io(randn(B, H, L, Dv), w.dtype)
    g = None
    if w.gate == GATE_PER_KEY:
        g = torch.nn.functional.logsigmoid(randn(B, H, L, Dk) + w.gate_mean) / w.gate_div
    elif w.gate == GATE_PER_HEAD:
        g = torch.nn.functional.logsigmoid(randn(B, H, L) + w.gate_mean) / w.gate_div
    h0 = randn(B, H, Dk, Dv) * w.h0_std if w.h0_std > 0 else None
    igate = torch.sigmoid(randn(B, H, L)) if w.input_gate else None
    dO = _round_io(randn(B, H, L, Dv), w.dtype) if w.backward else None
    return {"q": q, "k": k, "v": v, "g": g, "h0": h0, "igate": igate, "dO": dO}


def make_dhT(w: Workload, seed: int = 0) -> torch.Tensor:
    """An upstream gradient for the final state (not part of the published workloads,
    which have none); drawn from its own generator so it does not shift other draws."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(10_000 + seed)
    return torch.randn(w.B, w.H, w.Dk, w.Dv, generator=gen, dtype=torch.float32)


def input_digest(inputs: Dict[str, Optional[torch.Tensor]]) -> str:
    """SHA-256 over the raw bytes of the drawn tensors, in draw order."""
    h = hashlib.sha256()
    for name in ("q", "k", "v", "g", "h0", "igate", "dO"):
        t = inputs.get(name)
        if t is None:
            continue
        h.update(name.encode())
        h.update(t.contiguous().view(torch.uint8).numpy().tobytes())
    return h.hexdigest()


def small(w: Workload, B: int = 1, H: int = 2, L: Optional[int] = None) -> Workload:
    """A reduced-size copy of a workload (same dims, dtype, gates, chunk), for parity
    runs the oracle finishes in seconds."""
    return w.replace(name=w.name + "-small", B=B, H=H, L=L if L is not None else min(w.L, 4 * w.chunk + 37))


def default_scale(Dk: int) -> float:
    return 1.0 / math.sqrt(Dk)


def make_deltanet_inputs(B: int, H: int, L: int, Dk: int, Dv: int, dtype: str = "bf16", seed: int = 0,
                         h0_std: float = 0.0) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of the delta-rule (DeltaNet) forward, drawn on the CPU: q, v ~ N(0,1); k ~ N(0,1)
    with each row scaled to unit L2 norm before rounding to the io dtype; beta =
    sigmoid(N(0,1)) in (0, 1), fp32 [B,H,L]; h0 ~ N(0, h0_std^2) fp32 or None. The unit-norm
    keys and beta in (0, 1) keep every transition I - beta k^T k contractive."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(20_000 + seed)

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = _round_io(randn(B, H, L, Dk), dtype)
    k = randn(B, H, L, Dk)
    k = _round_io(k / k.norm(dim=-1, keepdim=True).clamp_min(1e-6), dtype)
    v = _round_io(randn(B, H, L, Dv), dtype)
    beta = torch.sigmoid(randn(B, H, L))
    h0 = randn(B, H, Dk, Dv) * h0_std if h0_std > 0 else None
    return {"q": q, "k": k, "v": v, "beta": beta, "h0": h0}


# DeltaNet forward+backward: the pages give the method but no benchmark shape, so this takes
# the gated workloads' batch and length with square heads (Dk = Dv = 128), bf16 I/O.
DELTANET = dict(B=4, H=16, L=4096, Dk=128, Dv=128, dtype="bf16")


# mLSTM cell with an exponential input gate, normaliser and stabiliser: the shapes of the
# scalar-gate workload c5 (B=2 H=8 L=8192 Dk=Dv=256, bf16, log forget gate logsigmoid(N(3,1))
# per head, scale Dk^-1/2), with the log input gate i~ ~ N(0, 1) (the gate is e^{i~}).
MLSTM = Workload("mlstm", 2, 8, 8192, 256, 256, 64, "bf16", GATE_PER_HEAD, True, 256 ** -0.5,
                 gate_mean=3.0, gate_div=1.0)


def make_mlstm_inputs(w: Workload, seed: int = 0, itil_shift: float = 0.0) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs of the mLSTM cell, drawn on the CPU from one generator in the order q, k, v,
    forget-gate pre-activation, log input gate, dh: q, k, v, dh ~ N(0,1) in the io dtype;
    g = logsigmoid(N(gate_mean, 1)) / gate_div fp32 [B,H,L] (log forget gate); itil ~ N(0,1) +
    itil_shift fp32 [B,H,L] (log of the exponential input gate)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(30_000 + seed)
    B, H, L, Dk, Dv = w.B, w.H, w.L, w.Dk, w.Dv

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    q = _round_io(randn(B, H, L, Dk), w.dtype)
    k = _round_io(randn(B, H, L, Dk), w.dtype)
    v = _round_io(randn(B, H, L, Dv), w.dtype)
    g = torch.nn.functional.logsigmoid(randn(B, H, L) + w.gate_mean) / w.gate_div
    itil = randn(B, H, L) + itil_shift
    dh = _round_io(randn(B, H, L, Dv), w.dtype) if w.backward else None
    return {"q": q, "k": k, "v": v, "g": g, "itil": itil, "dh": dh}
