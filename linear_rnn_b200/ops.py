"""Python entry points with the names of the C ABI (include/gla.h): gla_fwd, gla_bwd,
gla_workspace_bytes, gla_check_device_status.

They marshal torch tensors into the C calls: shape/dtype checks, the gate mode read
from g's rank, a workspace allocated with torch (the library itself allocates nothing),
and the current torch CUDA stream. Tensors on the host are copied to the current CUDA
device and results copied back (the end-to-end call of a host-side user); tensors
already on the device are used in place.
"""
from __future__ import annotations

import ctypes
import math
from typing import Dict, Optional, Tuple

import torch

from . import _lib
from ._lib import GlaError, GlaProblem

_PLANS = {"auto": _lib.GLA_PLAN_AUTO, "simt": _lib.GLA_PLAN_SIMT, "tc": _lib.GLA_PLAN_TC}


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _io_dtype(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return _lib.GLA_F32
    if dt == torch.bfloat16:
        return _lib.GLA_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {dt}")


def make_problem(q: torch.Tensor, v: torch.Tensor, g: Optional[torch.Tensor], *, scale: Optional[float],
                 chunk: int, plan: str) -> GlaProblem:
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, L, D]")
    B, H, L, Dk = q.shape
    Dv = v.shape[-1]
    if g is None:
        gate = _lib.GLA_GATE_NONE
    elif g.dim() == 4:
        gate = _lib.GLA_GATE_PER_KEY
    elif g.dim() == 3:
        gate = _lib.GLA_GATE_PER_HEAD
    else:
        raise ValueError("g must be [B,H,L,Dk] (per key dim) or [B,H,L] (per head)")
    if plan not in _PLANS:
        raise ValueError(f"plan must be one of {sorted(_PLANS)}")
    return GlaProblem(B, H, L, Dk, Dv, int(chunk), float(1.0 / math.sqrt(Dk) if scale is None else scale),
                      _io_dtype(q.dtype), gate, _PLANS[plan])


def gla_workspace_bytes(problem: GlaProblem, for_backward: bool) -> int:
    return int(_lib.lib.gla_workspace_bytes(ctypes.byref(problem), int(for_backward)))


def _stream_handle(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _to_dev(t: Optional[torch.Tensor], device: torch.device) -> Optional[torch.Tensor]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("inputs must be contiguous (BHLD)")
    if t.device.type == "cuda":
        return t
    return t.to(device, non_blocking=True)


def _to_host(tensors):
    """Copy device results into pinned host tensors (asynchronously on the current
    stream), then wait for the stream once."""
    out = []
    for t in tensors:
        if t is None:
            out.append(None)
            continue
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t, non_blocking=True)
        out.append(h)
    torch.cuda.current_stream().synchronize()
    return out


def _check(status: int, where: str):
    if status != _lib.GLA_OK:
        raise GlaError(status, where)


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor]) -> torch.Tensor:
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise GlaError(_lib.GLA_ERR_WORKSPACE, "workspace")
        return workspace
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def gla_saved_states_bytes(problem: GlaProblem) -> int:
    return int(_lib.lib.gla_saved_states_bytes(ctypes.byref(problem)))


def gla_fwd(q, k, v, g=None, igate=None, h0=None, *, scale: Optional[float] = None, chunk: int = 64,
            plan: str = "auto", output_final_state: bool = True,
            workspace: Optional[torch.Tensor] = None,
            saved_states: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Forward pass. Returns (o, hT); hT is None when output_final_state is False.
    saved_states: optional device buffer (at least gla_saved_states_bytes) that receives the
    states gla_bwd(..., saved_states=) then uses instead of recomputing them."""
    host = q.device.type != "cuda"
    device = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    q, k, v, g, igate, h0 = (_to_dev(t, device) for t in (q, k, v, g, igate, h0))
    prob = make_problem(q, v, g, scale=scale, chunk=chunk, plan=plan)
    o = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=device)
    hT = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                     device=device) if output_final_state else None
    nbytes = gla_workspace_bytes(prob, False)
    if nbytes == 0:
        raise GlaError(_lib.GLA_ERR_UNSUPPORTED, "gla_workspace_bytes")
    ws = _workspace(nbytes, device, workspace)
    _check_saved(saved_states, prob)
    st = _lib.lib.gla_fwd_save(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(igate), _ptr(h0),
                               _ptr(o), _ptr(hT), _ptr(saved_states), _ptr(ws), ws.numel() * ws.element_size(),
                               _stream_handle(device))
    _check(st, "gla_fwd")
    if host:
        o, hT = _to_host([o, hT])
    return o, hT


def _mlstm_problem(q, v, g, itil, scale, chunk, plan):
    if g is None or g.dim() != 3 or g.dtype != torch.float32:
        raise ValueError("g (log forget gate) must be float32 [B, H, L]")
    if itil is None or itil.dtype != torch.float32 or tuple(itil.shape) != tuple(g.shape):
        raise ValueError("itil (log input gate) must be float32 [B, H, L] like g")
    return make_problem(q, v, g, scale=scale, chunk=chunk, plan=plan)


def gla_mlstm_saved_bytes(problem: GlaProblem) -> int:
    return int(_lib.lib.gla_mlstm_saved_bytes(ctypes.byref(problem)))


def _check_ml_saved(saved, prob):
    if saved is None:
        return
    if saved.device.type != "cuda" or not saved.is_contiguous():
        raise ValueError("saved_states must be a contiguous CUDA tensor")
    if saved.numel() * saved.element_size() < gla_mlstm_saved_bytes(prob):
        raise GlaError(_lib.GLA_ERR_WORKSPACE, "saved_states")


def gla_mlstm_fwd(q, k, v, g, itil, *, scale: Optional[float] = None, chunk: int = 64, plan: str = "auto",
                  workspace: Optional[torch.Tensor] = None,
                  saved_states: Optional[torch.Tensor] = None) -> torch.Tensor:
    """mLSTM cell (exponential input gate, normaliser, stabiliser): q, k [B,H,L,Dk], v [B,H,L,Dv],
    g = log forget gate and itil = log input gate, both fp32 [B,H,L]. Returns h [B,H,L,Dv].
    saved_states: optional device buffer (at least gla_mlstm_saved_bytes) that keeps the forward's
    results for gla_mlstm_bwd(..., saved_states=), which then does not run the forward again."""
    host = q.device.type != "cuda"
    device = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    q, k, v, g, itil = (_to_dev(t, device) for t in (q, k, v, g, itil))
    prob = _mlstm_problem(q, v, g, itil, scale, chunk, plan)
    nbytes = int(_lib.lib.gla_mlstm_workspace_bytes(ctypes.byref(prob), 0))
    if nbytes == 0:
        raise GlaError(_lib.GLA_ERR_UNSUPPORTED, "gla_mlstm_workspace_bytes")
    ws = _workspace(nbytes, device, workspace)
    _check_ml_saved(saved_states, prob)
    h = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=device)
    st = _lib.lib.gla_mlstm_fwd_save(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(itil), _ptr(h),
                                     _ptr(saved_states), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream_handle(device))
    _check(st, "gla_mlstm_fwd")
    if host:
        (h,) = _to_host([h])
    return h


def gla_mlstm_bwd(q, k, v, g, itil, dh, *, scale: Optional[float] = None, chunk: int = 64, plan: str = "auto",
                  workspace: Optional[torch.Tensor] = None,
                  saved_states: Optional[torch.Tensor] = None) -> Dict[str, torch.Tensor]:
    """Gradients of sum(dh * h) of gla_mlstm_fwd: dict dq, dk, dv (io dtype), dg, ditil (fp32).
    saved_states: the buffer a gla_mlstm_fwd with the same inputs and plan filled, or None to
    run the forward passes again."""
    host = q.device.type != "cuda"
    device = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    q, k, v, g, itil, dh = (_to_dev(t, device) for t in (q, k, v, g, itil, dh))
    prob = _mlstm_problem(q, v, g, itil, scale, chunk, plan)
    nbytes = int(_lib.lib.gla_mlstm_workspace_bytes(ctypes.byref(prob), 1))
    if nbytes == 0:
        raise GlaError(_lib.GLA_ERR_UNSUPPORTED, "gla_mlstm_workspace_bytes")
    ws = _workspace(nbytes, device, workspace)
    _check_ml_saved(saved_states, prob)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg, ditil = torch.empty_like(g), torch.empty_like(itil)
    st = _lib.lib.gla_mlstm_bwd_saved(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(itil), _ptr(dh),
                                      _ptr(saved_states), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(ditil),
                                      _ptr(ws), ws.numel() * ws.element_size(), _stream_handle(device))
    _check(st, "gla_mlstm_bwd")
    out = {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "ditil": ditil}
    if host:
        out = dict(zip(out, _to_host(list(out.values()))))
    return out


def gla_decode(q, k, v, g, igate, state, *, scale: Optional[float] = None) -> torch.Tensor:
    """One recurrent step per (b, h) from `state` (fp32 [B,H,Dk,Dv] on the GPU, updated in
    place): q, k [B,H,1,Dk], v [B,H,1,Dv], g [B,H,1,Dk] / [B,H,1] / None, igate [B,H,1] / None.
    Returns o [B,H,1,Dv]."""
    if state.device.type != "cuda" or state.dtype != torch.float32 or not state.is_contiguous():
        raise ValueError("state must be a contiguous float32 CUDA tensor (it is updated in place)")
    device = state.device
    q, k, v, g, igate = (_to_dev(t, device) for t in (q, k, v, g, igate))
    if q.shape[2] != 1:
        raise ValueError("gla_decode takes one token per (b, h): q must be [B, H, 1, Dk]")
    prob = make_problem(q, v, g, scale=scale, chunk=64, plan="auto")
    o = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=device)
    st = _lib.lib.gla_decode(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(igate), _ptr(state),
                             _ptr(o), _stream_handle(device))
    _check(st, "gla_decode")
    return o


def gla_deltanet_saved_bytes(problem: GlaProblem) -> int:
    return int(_lib.lib.gla_deltanet_saved_bytes(ctypes.byref(problem)))


def _check_dn_saved(saved, prob):
    if saved is None:
        return
    if saved.device.type != "cuda" or not saved.is_contiguous():
        raise ValueError("saved_states must be a contiguous CUDA tensor")
    if saved.numel() * saved.element_size() < gla_deltanet_saved_bytes(prob):
        raise GlaError(_lib.GLA_ERR_WORKSPACE, "saved_states")


def gla_deltanet_fwd(q, k, v, beta, h0=None, *, scale: Optional[float] = None,
                     output_final_state: bool = True,
                     saved_states: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunkwise DeltaNet forward: q, k [B,H,L,Dk], v [B,H,L,Dv] (bf16 or fp32), beta [B,H,L]
    fp32, h0 [B,H,Dk,Dv] fp32 or None. Returns o [B,H,L,Dv] and the final state (fp32, or None
    when output_final_state is False). saved_states: optional device buffer (at least
    gla_deltanet_saved_bytes) that receives the chunk start states, which
    gla_deltanet_bwd(..., saved_states=) then reads instead of walking the recurrence again.
    Host tensors are copied to the current device and the results back."""
    host = q.device.type != "cuda"
    device = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    q, k, v, beta, h0 = (_to_dev(t, device) for t in (q, k, v, beta, h0))
    if beta is None or beta.dtype != torch.float32 or tuple(beta.shape) != tuple(q.shape[:3]):
        raise ValueError("beta must be float32 [B, H, L]")
    prob = make_problem(q, v, None, scale=scale, chunk=64, plan="auto")
    _check_dn_saved(saved_states, prob)
    o = torch.empty(q.shape[:-1] + (v.shape[-1],), dtype=q.dtype, device=device)
    hT = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                     device=device) if output_final_state else None
    st = _lib.lib.gla_deltanet_fwd_save(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(h0),
                                        _ptr(o), _ptr(hT), _ptr(saved_states), _stream_handle(device))
    _check(st, "gla_deltanet_fwd")
    if host:
        o, hT = _to_host([o, hT])
    return o, hT


def gla_deltanet_bwd(q, k, v, beta, h0, dO, dhT=None, *, scale: Optional[float] = None,
                     output_dh0: bool = True, workspace: Optional[torch.Tensor] = None,
                     saved_states: Optional[torch.Tensor] = None) -> Dict[str, Optional[torch.Tensor]]:
    """DeltaNet backward: dict dq, dk, dv (io dtype), dbeta (fp32 [B,H,L]) and dh0 (fp32, or
    None when output_dh0 is False). saved_states: the buffer a gla_deltanet_fwd on the same
    inputs filled, or None to recompute the chunk start states. Host tensors are copied to the
    current device and the results back."""
    host = q.device.type != "cuda"
    device = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    q, k, v, beta, h0, dO, dhT = (_to_dev(t, device) for t in (q, k, v, beta, h0, dO, dhT))
    if beta is None or beta.dtype != torch.float32 or tuple(beta.shape) != tuple(q.shape[:3]):
        raise ValueError("beta must be float32 [B, H, L]")
    prob = make_problem(q, v, None, scale=scale, chunk=64, plan="auto")
    nbytes = _lib.lib.gla_deltanet_bwd_workspace_bytes(ctypes.byref(prob))
    if nbytes == 0:
        raise GlaError(_lib.GLA_ERR_UNSUPPORTED, "gla_deltanet_bwd_workspace_bytes")
    ws = _workspace(nbytes, device, workspace)
    _check_dn_saved(saved_states, prob)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dbeta = torch.empty_like(beta)
    dh0 = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                      device=device) if output_dh0 else None
    st = _lib.lib.gla_deltanet_bwd_saved(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(h0),
                                         _ptr(dO), _ptr(dhT), _ptr(saved_states), _ptr(dq), _ptr(dk), _ptr(dv),
                                         _ptr(dbeta), _ptr(dh0), _ptr(ws), ws.numel() * ws.element_size(),
                                         _stream_handle(device))
    _check(st, "gla_deltanet_bwd")
    out = {"dq": dq, "dk": dk, "dv": dv, "dbeta": dbeta, "dh0": dh0}
    if host:
        names = list(out)
        out = dict(zip(names, _to_host([out[n] for n in names])))
    return out


def gla_shard_state(k, v, g=None, igate=None, *, chunk: int = 64) -> Tuple[torch.Tensor, torch.Tensor]:
    """(state, gamma) of one sequence shard: its end state from a zero initial state
    [B,H,Dk,Dv] and its total log-decay per key dim [B,H,Dk], both fp32 on the GPU."""
    device = k.device
    prob = make_problem(k, v, g, scale=1.0, chunk=chunk, plan="tc")
    B, H, _, Dk = k.shape
    state = torch.empty(B, H, Dk, v.shape[-1], dtype=torch.float32, device=device)
    gamma = torch.empty(B, H, Dk, dtype=torch.float32, device=device)
    nb = max(int(_lib.lib.gla_shard_workspace_bytes(ctypes.byref(prob))), 256)
    ws = torch.empty(nb, dtype=torch.uint8, device=device)
    st = _lib.lib.gla_shard_state(ctypes.byref(prob), _ptr(k), _ptr(v), _ptr(g), _ptr(igate), _ptr(state),
                                  _ptr(gamma), _ptr(ws), nb, _stream_handle(device))
    _check(st, "gla_shard_state")
    return state, gamma


def gla_shard_state_grad(q, dO, g=None, *, scale: Optional[float] = None,
                         chunk: int = 64) -> Tuple[torch.Tensor, torch.Tensor]:
    """(state_grad, gamma) of one sequence shard: the gradient w.r.t. the state before its
    first token from its own outputs alone [B,H,Dk,Dv], and its total log-decay per key dim
    [B,H,Dk], both fp32 on the GPU."""
    device = q.device
    prob = make_problem(q, dO, g, scale=scale, chunk=chunk, plan="tc")
    B, H, _, Dk = q.shape
    dS = torch.empty(B, H, Dk, dO.shape[-1], dtype=torch.float32, device=device)
    gamma = torch.empty(B, H, Dk, dtype=torch.float32, device=device)
    nb = max(int(_lib.lib.gla_shard_workspace_bytes(ctypes.byref(prob))), 256)
    ws = torch.empty(nb, dtype=torch.uint8, device=device)
    st = _lib.lib.gla_shard_state_grad(ctypes.byref(prob), _ptr(q), _ptr(dO), _ptr(g), _ptr(dS), _ptr(gamma),
                                       _ptr(ws), nb, _stream_handle(device))
    _check(st, "gla_shard_state_grad")
    return dS, gamma


def gla_state_fold(states: torch.Tensor, gammas: torch.Tensor, count: int,
                   h0: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The state after the first `count` shards, given all shards' (state, gamma) stacked along
    a leading shard axis ([n,B,H,Dk,Dv], [n,B,H,Dk]), starting from h0 (or 0)."""
    if states.dim() != 5 or gammas.dim() != 4 or not (0 <= count <= states.shape[0]):
        raise ValueError("states [n,B,H,Dk,Dv], gammas [n,B,H,Dk], 0 <= count <= n")
    _, B, H, Dk, Dv = states.shape
    prob = GlaProblem(B, H, 1, Dk, Dv, 64, 1.0, _lib.GLA_F32, _lib.GLA_GATE_PER_KEY, _PLANS["auto"])
    out = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=states.device)
    st = _lib.lib.gla_state_fold(ctypes.byref(prob), int(count), _ptr(states.contiguous()), _ptr(gammas.contiguous()),
                                 _ptr(h0), _ptr(out), _stream_handle(states.device))
    _check(st, "gla_state_fold")
    return out


def gla_fwd_sequence_sharded(q, k, v, g=None, igate=None, h0=None, *, scale: Optional[float] = None,
                             chunk: int = 64, group=None, _shard_ops=None):
    """Forward over a sequence cut into contiguous shards, one per rank of `group` (rank order =
    sequence order): each rank passes its own shard of q, k, v, g, igate (and every rank the
    same h0), and gets its shard's o and end state (the last rank's is the sequence's hT).
    One all-gather of the shards' (end state from zero, total log-decay) is the only exchange.
    _shard_ops replaces the three per-rank steps (shard_state, fold, forward) for tests of the
    exchange on CPU ranks."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    shard_state, fold, fwd = _shard_ops or (
        lambda: gla_shard_state(k, v, g, igate, chunk=chunk),
        lambda states, gammas: gla_state_fold(states, gammas, rank, h0),
        lambda s_in: gla_fwd(q, k, v, g, igate, s_in, scale=scale, chunk=chunk))
    state, gamma = shard_state()
    parts_s = [torch.empty_like(state) for _ in range(world)]
    parts_g = [torch.empty_like(gamma) for _ in range(world)]
    dist.all_gather(parts_s, state.contiguous(), group=group)
    dist.all_gather(parts_g, gamma.contiguous(), group=group)
    return fwd(fold(torch.stack(parts_s), torch.stack(parts_g)))


def gla_bwd_sequence_sharded(q, k, v, g, igate, h0, dO, dhT=None, *, scale: Optional[float] = None,
                             chunk: int = 64, group=None, _shard_ops=None) -> Dict[str, Optional[torch.Tensor]]:
    """Backward over a sequence cut into contiguous shards, one per rank of `group` (rank order =
    sequence order): each rank passes its own shard of q, k, v, g, igate, dO, and every rank the
    same h0 and dhT (the gradient at the sequence's end). Returns gla_bwd's dict for the rank's
    shard; rank 0's dh0 is the sequence's, the other ranks' dh0 is None. One all-gather of the
    shards' (end state from zero, start-state gradient from zero, total log-decay) is the only
    exchange: rank r's initial state folds shards 0..r-1 from h0, the gradient at its end folds
    shards P-1..r+1 in reverse order from dhT. _shard_ops replaces the per-rank steps
    (shard_state, shard_state_grad, fold, backward) for tests of the exchange on CPU ranks."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    shard_state, shard_grad, fold, bwd = _shard_ops or (
        lambda: gla_shard_state(k, v, g, igate, chunk=chunk),
        lambda: gla_shard_state_grad(q, dO, g, scale=scale, chunk=chunk),
        gla_state_fold,
        lambda s_in, d_end: gla_bwd(q, k, v, g, igate, s_in, dO, d_end, scale=scale, chunk=chunk,
                                    output_dh0=rank == 0))
    S, gamma = shard_state()
    dS, _ = shard_grad()
    n_s, n_g = S.numel(), gamma.numel()
    pack = torch.cat([S.reshape(-1), dS.reshape(-1), gamma.reshape(-1)])
    parts = [torch.empty_like(pack) for _ in range(world)]
    dist.all_gather(parts, pack, group=group)
    allp = torch.stack(parts)
    states = allp[:, :n_s].reshape(world, *S.shape)
    grads = allp[:, n_s:2 * n_s].reshape(world, *S.shape)
    gammas = allp[:, 2 * n_s:2 * n_s + n_g].reshape(world, *gamma.shape)
    s_in = fold(states, gammas, rank, h0)
    d_end = fold(grads.flip(0).contiguous(), gammas.flip(0).contiguous(), world - 1 - rank, dhT)
    return bwd(s_in, d_end)


def _check_saved(saved, prob):
    if saved is None:
        return
    if saved.device.type != "cuda" or saved.dtype != torch.float32 or not saved.is_contiguous():
        raise ValueError("saved_states must be a contiguous float32 CUDA tensor")
    if saved.numel() * 4 < gla_saved_states_bytes(prob):
        raise GlaError(_lib.GLA_ERR_WORKSPACE, "saved_states")


def gla_bwd(q, k, v, g, igate, h0, dO, dhT=None, *, scale: Optional[float] = None, chunk: int = 64,
            plan: str = "auto", output_dh0: bool = True,
            workspace: Optional[torch.Tensor] = None,
            saved_states: Optional[torch.Tensor] = None) -> Dict[str, Optional[torch.Tensor]]:
    """Backward pass. Returns dict dq, dk, dv, dg (None if ungated), di (None without an
    input gate), dh0 (None when output_dh0 is False). saved_states: the buffer a gla_fwd on
    the same inputs filled, or None to recompute."""
    host = q.device.type != "cuda"
    device = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    q, k, v, g, igate, h0, dO, dhT = (_to_dev(t, device) for t in (q, k, v, g, igate, h0, dO, dhT))
    prob = make_problem(q, v, g, scale=scale, chunk=chunk, plan=plan)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dg = torch.empty_like(g) if g is not None else None
    di = torch.empty_like(igate) if igate is not None else None
    dh0 = torch.empty(q.shape[0], q.shape[1], q.shape[-1], v.shape[-1], dtype=torch.float32,
                      device=device) if output_dh0 else None
    nbytes = gla_workspace_bytes(prob, True)
    if nbytes == 0:
        raise GlaError(_lib.GLA_ERR_UNSUPPORTED, "gla_workspace_bytes")
    ws = _workspace(nbytes, device, workspace)
    _check_saved(saved_states, prob)
    st = _lib.lib.gla_bwd_saved(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(igate), _ptr(h0),
                                _ptr(dO), _ptr(dhT), _ptr(saved_states), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                                _ptr(di), _ptr(dh0), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream_handle(device))
    _check(st, "gla_bwd")
    out = {"dq": dq, "dk": dk, "dv": dv, "dg": dg, "di": di, "dh0": dh0}
    if host:
        names = list(out)
        out = dict(zip(names, _to_host([out[n] for n in names])))
    return out


def gla_check_device_status(workspace: torch.Tensor) -> int:
    device = workspace.device
    return int(_lib.lib.gla_check_device_status(_ptr(workspace), _stream_handle(device)))
