#!/usr/bin/env python
"""Benchmark of the chunkwise gated-linear-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3] [--impl ours|reference]

One step = one pass of the whole path over one batch of synthetic input: gla_fwd then
gla_bwd (workloads with a backward) through the library's C ABI. Default workload c3:
GLA forward+backward, B=4 H=16 L=4096 Dk=128 Dv=256, bf16 I/O, per-key log-gate
logsigmoid(N(0,1))/16, dO ~ N(0,1), chunk 64.

Prints one JSON line on rank 0. `value` is whole-job tokens/s with inputs resident in
HBM (CUDA events per step on the launching stream; the 256 MiB L2 flush between steps is
outside the events); `e2e` is the same metric through the public Python API with host
(pinned) tensors, host<->device copies inside the timed region. Under torchrun each rank
runs its own batch (weak scaling, no data-path collective); the step time is the max over
ranks. `--impl reference` times the float64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from linear_rnn_b200 import inputs as I  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ accounting
def io_bytes(w):
    return 2 if w.dtype == "bf16" else 4


def gate_elems(w):
    return {I.GATE_NONE: 0, I.GATE_PER_KEY: w.Dk, I.GATE_PER_HEAD: 1}[w.gate]


def flops(w, backward):
    """Algorithmic FLOPs: per token-head C*Dk + C*Dv + 4*Dk*Dv forward (causal-half intra
    products, inter q~S, state K^T V) and C*(3Dk+2Dv) + 8*Dk*Dv backward."""
    th = w.B * w.H * w.L
    if w.name == "decode":   # one token from a given state: the state update and q S
        return float(th * 4 * w.Dk * w.Dv)
    f = th * (w.chunk * w.Dk + w.chunk * w.Dv + 4 * w.Dk * w.Dv)
    if backward:
        f += th * (w.chunk * (3 * w.Dk + 2 * w.Dv) + 8 * w.Dk * w.Dv)
    return float(f)


def compulsory_bytes(w, backward):
    """Read every input once and write every output once (chunk states are not compulsory)."""
    th = w.B * w.H * w.L
    e = io_bytes(w)
    st = 4 * w.B * w.H * w.Dk * w.Dv
    ig = 4 * th if w.input_gate else 0
    fwd = th * (2 * w.Dk + w.Dv) * e + 4 * th * gate_elems(w) + ig + th * w.Dv * e + st
    fwd += st if w.h0_std > 0 else 0
    if not backward:
        return float(fwd)
    bwd = th * (2 * w.Dk + 2 * w.Dv) * e + 4 * th * gate_elems(w) + ig          # q k v dO g (i)
    bwd += th * (2 * w.Dk + w.Dv) * e + 4 * th * gate_elems(w) + ig              # dq dk dv dg (di)
    bwd += 2 * st if w.h0_std > 0 else 0                                         # h0, dh0
    return float(fwd + bwd)


def _mean(xs):
    return sum(xs) / len(xs) if xs else 0.0


def kernel_bytes(name, w, fseg=1, bseg=1, bwd_state=False):
    """Bytes of one launch of each kernel, split in two:
    method: the path's own inputs the kernel reads and outputs it writes, each once (q, k, v,
            dO, g, i, h0, dhT in; o, hT, dq, dk, dv, dg, di, dh0 out);
    plan:   the plan's intermediates it reads or writes in the workspace (segment states and
            log-decay totals, the dq kernel's in-segment prefixes of q*dq, saved states).
    fseg / bseg: sequence segments of the forward / backward plan (gla_plan_info). bwd_state:
    the backward runs its own state pass and scan (gla_bwd without saved states); the training
    pair's backward starts from the states its forward saved. Returns (method, plan)."""
    th = w.B * w.H * w.L
    BH = w.B * w.H
    e = io_bytes(w)
    ge = 4 * th * gate_elems(w)
    ig = 4 * th if w.input_gate else 0
    N = math.ceil(w.L / w.chunk)
    s1 = 4.0 * BH * w.Dk * w.Dv                  # one fp32 state per head
    h0 = s1 if w.h0_std > 0 else 0
    states = s1 * N
    q = k = th * w.Dk * e
    v = o = th * w.Dv * e
    dgb = 4 * th * gate_elems(w)                 # fp32 dg (or its in-segment prefix)
    gam = 4.0 * BH * w.Dk                        # one segment's log-decay totals
    frac_f = (fseg - 1) / fseg                   # share of the sequence the state passes cover
    frac_b = (bseg - 1) / bseg
    bs = bseg > 1 and bwd_state                  # a backward state pass and scan are launched
    di = ig
    table = {
        "simt_cumsum": (ge, ge),
        "simt_state": (k + v + ge + h0, states),
        "simt_out": (q + k + v + ge + o, states),
        "simt_dstate": (q + o + ge, states),
        "simt_dq": (q + k + v + o + ge + q, states + 4 * th * w.Dk),
        "simt_dk": (q + k + v + o + ge + k, states + 2 * 4 * th * w.Dk),
        "simt_dv": (q + k + o + ge + v, states),
        "simt_dg_key": (dgb, 4 * th * w.Dk),
        # forward output pass: reads the segment initial states; the training pair also writes
        # the states the backward's segments start from
        "tc_fwd": (q + k + v + ge + ig + o + s1 + h0, s1 * (fseg - 1) + s1 * (bseg - 1)),
        "tc_seg_scan": (_mean([h0] * (fseg > 1) + [h0] * bs),
                        _mean([2 * s1 * (fseg - 1) + 2 * gam * (fseg - 1)] * (fseg > 1) +
                              [2 * s1 * (bseg - 1) + 2 * gam * (bseg - 1)] * bs)),
        # the forward's (or the backward's own) state pass over segments 0..nseg-2; per launch
        # averaged when both plans launch one
        "tc_state": (_mean([frac_f * (k + v + ge + ig)] * (fseg > 1) + [frac_b * (k + v + ge + ig)] * bs),
                     _mean([(s1 + gam) * (fseg - 1)] * (fseg > 1) + [(s1 + gam) * (bseg - 1)] * bs)),
        "tc_gstate": (frac_b * (q + o + ge), (s1 + gam) * (bseg - 1)),
        "tc_seg_rscan": (0.0, 2 * (s1 + gam) * (bseg - 1)),
        "tc_bwd_dq": (q + k + v + o + ge + ig + h0 + q,
                      s1 * (bseg - 1) + dgb + 4 * BH * bseg * w.Dk),
        "tc_bwd_dkdv": (q + k + v + o + ge + ig + k + v + dgb + di + h0,
                        2 * s1 * bseg + dgb + 4 * BH * bseg * w.Dk),
        # decode step: q, k, v, g, i read, o written, the state read and written once
        "decode": (compulsory_bytes(w, False), 0.0),
    }
    m, pl = table.get(name, (0.0, 0.0))
    return float(m), float(pl)


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch from one ncu capture,
# with the SHA-256 prefix of the kernel's source file the counters apply to: the file at capture
# time, or after a later change to host code only (launch set-up outside the kernels; the commit
# that re-confirmed the prefix says so). A kernel whose source has changed otherwise reports
# traffic null. `scale`: the capture ran a smaller case of the same workload (`case`); traffic
# grows with the heads processed.
MEASURED_TRAFFIC = {
    ("tc_fwd", "c2"): {"bytes": 187.0e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_fwd.cu",
                       "sha": "66a83723972df331", "case": "c2"},
    ("tc_fwd", "c4"): {"bytes": 805.2e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_fwd.cu",
                       "sha": "66a83723972df331", "case": "c4"},
    ("tc_fwd", "c3"): {"bytes": 566.8e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_fwd.cu",
                       "sha": "66a83723972df331", "case": "c3 training pair"},
    ("tc_fwd", "c5"): {"bytes": 295.9e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_fwd.cu",
                       "sha": "66a83723972df331", "case": "c5 training pair"},
    ("tc_bwd_dkdv", "c3"): {"bytes": 1086.7e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_bwd.cu",
                            "sha": "4657481726eb25d5", "case": "c3"},
    ("tc_bwd_dkdv", "c5"): {"bytes": 484.1e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_bwd.cu",
                            "sha": "4657481726eb25d5", "case": "c5"},
    ("tc_bwd_dq", "c3"): {"bytes": 782.2e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_bwd.cu",
                          "sha": "4657481726eb25d5", "case": "c3"},
    ("tc_bwd_dq", "c5"): {"bytes": 392.6e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_tc_bwd.cu",
                          "sha": "4657481726eb25d5", "case": "c5"},
    ("deltanet_bwd_walk", "deltanet"): {"bytes": 490.5e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_deltanet_tc.cu",
                                         "sha": "b19710d35dc88dde", "case": "deltanet"},
    ("deltanet_bwd_grads", "deltanet"): {"bytes": 793.1e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_deltanet_tc.cu",
                                          "sha": "b19710d35dc88dde", "case": "deltanet"},
    ("decode", "decode"): {"bytes": 214.9e6, "scale": 1, "src": "linear_rnn_b200/csrc/gla_decode.cu",
                           "sha": "45347f72608393eb", "case": "decode, 1024 heads"},
}


def measured_traffic(kernel, workload):
    m = MEASURED_TRAFFIC.get((kernel, workload))
    if not m:
        return None
    try:
        with open(os.path.join(ROOT, m["src"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != m["sha"]:
                return None
    except OSError:
        return None
    return m["bytes"] * m["scale"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi every 200 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.error = None

    def start(self):
        try:
            uuid = None
            try:
                uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
                uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            except Exception:
                pass
            sel = ["--id=" + uuid] if uuid else ["-i", str(self.dev)]
            self.proc = subprocess.Popen(["nvidia-smi", *sel, "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception as ex:  # nvidia-smi missing
            self.error = str(ex)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.error or "no sampler"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle baseline
def oracle_sample(w, seed, heads):
    """Times the float64 oracle on `heads` whole heads (full L) of the workload.
    Returns (tokens_equivalent, seconds, threads)."""
    import oracle
    sub = w.replace(B=1, H=heads)
    x = I.make_inputs(sub, seed=seed)
    t0 = time.perf_counter()
    oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], w.scale)
    if w.backward:
        oracle.gla_bwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], x["dO"], None, w.scale)
    dt = time.perf_counter() - t0
    return w.L * heads / w.H, dt, oracle.num_threads()


def oracle_heads(w):
    # about 10-30 s of host work on a multi-core box; heads are the unit of parallelism
    return max(1, min(w.B * w.H, 4 * (os.cpu_count() or 8)))


# ------------------------------------------------------------------ main
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group(
            "nccl" if torch.cuda.is_available() else "gloo", timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def base_line(w, args, world):
    return {"metric": "GLA chunkwise fwd/bwd tokens/s", "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded; linear_rnn_b200/inputs.py)",
            "config": {"workload": f"{w.name}: {'GLA decode step' if w.name == 'decode' else 'GLA forward+backward' if w.backward else 'GLA forward'}, "
                                   f"B={w.B} H={w.H} L={w.L} Dk={w.Dk} Dv={w.Dv} chunk={w.chunk} {w.dtype}",
                       "global_batch": w.B * world, "seq_len": w.L, "parallelism": f"replicas x{world}",
                       "l2": "256 MiB L2 flush between steps, outside the per-step events; inputs > L2"}}


def run_reference(args, w, world, rank):
    """The float64 oracle on the host cores, each step a bounded sample of whole heads of the
    workload (full L); `value` = tokens per second of the sample, `ms_per_step` = the time
    the oracle would take for the workload's whole batch at that rate."""
    if rank != 0:
        return
    heads = max(1, oracle_heads(w) // 2)
    for _ in range(args.warmup):
        oracle_sample(w, 0, heads)
    tok = 0.0
    tot = 0.0
    thr = 1
    for i in range(args.steps):
        t, dt, thr = oracle_sample(w, i, heads)
        tok += t
        tot += dt
    val = tok / tot
    line = base_line(w, args, 1)
    line.update({"impl": "reference", "value": val, "ms_per_step": 1e3 * w.B * w.L / val, "dtype": "f64",
                 "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                                  "sample": f"{heads} of {w.B * w.H} heads, full L={w.L}, "
                                            f"{'fwd+bwd' if w.backward else 'fwd'} per step; ms_per_step is the "
                                            f"whole batch at the sample's rate ({1e3 * tot / args.steps:.0f} ms per "
                                            f"sample step)"},
                 "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                 "gpu_launches": 0})
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ DeltaNet workload
DN_C = 64


def deltanet_kernel_flops(name, B, H, L, Dk, Dv):
    """Algorithmic FLOPs of one launch (per token-head, multiplied by B*H*L): causal C x C
    products count their lower half, K K^T and Q K^T once per head (not per value slice), a
    chunk's triangular solve C per value column and token (C^2/3 per token for the inverse of the
    CUDA-core plan). The tensor-core backward splits its work differently from the CUDA-core one
    (the walk keeps only the dS chain, the gradient kernel forms X and U), so bf16 and fp32 I/O
    have their own rows."""
    C = DN_C
    tc = I.DELTANET["dtype"] == "bf16"
    per = {
        # K K^T, Q K^T; K S, Q S, K^T X; the solve for X, lower(Q K^T) X
        "deltanet_fwd": 2 * C * Dk + 6 * Dk * Dv + 2 * C * Dv + (0 if tc else C * C / 3),
        # the backward's state pass (no output): K K^T; K S, K^T X; the solve for X
        "deltanet_state": C * Dk + 4 * Dk * Dv + C * Dv + (0 if tc else C * C / 3),
    }
    if tc:
        # K K^T, Q K^T; K dS', Q^T dO, K^T diag(beta) dR; P^T dO; the transposed solve
        per["deltanet_bwd_walk"] = 2 * C * Dk + 6 * Dk * Dv + 2 * C * Dv
        # K K^T, K S, the solve for X; dO X^T, dR X^T; dO S^T, X dS'^T, dR S^T; dP K, dP^T Q, G K, G^T K
        per["deltanet_bwd_grads"] = 5 * C * Dk + 8 * Dk * Dv + 3 * C * Dv
    else:
        # K K^T, P; K S, K dS', the dS update (2 products); P^T dO, T R, T^T dX; the inverse
        per["deltanet_bwd_walk"] = 2 * C * Dk + 8 * Dk * Dv + 3 * C * Dv + C * C / 3
        # dO X^T, dR X^T; dO S^T, X dS'^T, dR S^T; dP K, dP^T Q, G K, G^T (beta K)
        per["deltanet_bwd_grads"] = 2 * C * Dv + 6 * Dk * Dv + 4 * C * Dk
    return float(per.get(name, 0.0)) * B * H * L


def deltanet_alu_peak_tflops(sm_mhz):
    """FP32 FMA peak from the unit counts: 148 SMs x 128 FP32 lanes x 2 FLOPs x the SM clock."""
    return 148 * 128 * 2 * (sm_mhz or 1965.0) * 1e6 / 1e12


def deltanet_line(args, world, tokens, ms, extra):
    cfg = I.DELTANET
    line = {"metric": "DeltaNet chunkwise fwd+bwd tokens/s", "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg["dtype"], "data": "synthetic (seeded; linear_rnn_b200/inputs.py)",
            "config": {"workload": "deltanet: DeltaNet forward+backward, B={B} H={H} L={L} Dk={Dk} Dv={Dv} "
                                   "chunk=64 {dtype} I/O".format(**cfg),
                       "global_batch": cfg["B"] * world, "seq_len": cfg["L"], "parallelism": f"replicas x{world}",
                       "l2": "256 MiB L2 flush between steps, outside the per-step events; inputs > L2"},
            "value": tokens / (ms / 1e3), "ms_per_step": ms / args.steps}
    line.update(extra)
    return line


def blas_threads():
    """Threads of the BLAS library numpy's matrix products (the DeltaNet oracle) run on."""
    try:
        import threadpoolctl
        n = [i.get("num_threads") for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return torch.get_num_threads()


def deltanet_oracle_sample(seed, heads):
    """Times the float64 delta-rule oracle (forward, then back-propagation through time) on
    `heads` whole heads. Returns (tokens_equivalent, seconds)."""
    from oracle import deltanet as DN
    cfg = I.DELTANET
    x = I.make_deltanet_inputs(1, heads, cfg["L"], cfg["Dk"], cfg["Dv"], cfg["dtype"], seed=seed, h0_std=0.5)
    dO = torch.randn(1, heads, cfg["L"], cfg["Dv"], generator=torch.Generator().manual_seed(seed))
    sc = cfg["Dk"] ** -0.5
    t0 = time.perf_counter()
    DN.deltanet_fwd(x["q"], x["k"], x["v"], x["beta"], x["h0"], sc)
    DN.deltanet_bwd(x["q"], x["k"], x["v"], x["beta"], x["h0"], dO, None, sc)
    return cfg["L"] * heads / cfg["H"], time.perf_counter() - t0


def run_deltanet(args, world, rank, local):
    cfg = I.DELTANET
    heads = 1   # the oracle keeps every state of a head (L x Dk x Dv float64): one head per sample
    if args.impl == "reference":
        if rank != 0:
            return
        for _ in range(args.warmup):
            deltanet_oracle_sample(0, heads)
        tok = tot = 0.0
        for i in range(args.steps):
            t, dt = deltanet_oracle_sample(i, heads)
            tok += t
            tot += dt
        val = tok / tot
        base = deltanet_line(args, 1, tok, 1e3 * tot, {})
        base.update({"impl": "reference", "value": val, "dtype": "f64", "gpu_launches": 0,
                     "ms_per_step": 1e3 * cfg["B"] * cfg["L"] / val,
                     "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": blas_threads(),
                                      "kind": "oracle", "sample": f"{heads} of {cfg['B'] * cfg['H']} heads, "
                                                                  f"full L={cfg['L']}, fwd+bwd per step"},
                     "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        print(json.dumps(base), flush=True)
        return

    from linear_rnn_b200 import _lib, ops
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, L, Dk, Dv = cfg["B"], cfg["H"], cfg["L"], cfg["Dk"], cfg["Dv"]
    x = I.make_deltanet_inputs(B, H, L, Dk, Dv, cfg["dtype"], seed=rank, h0_std=0.5)
    dO = torch.randn(B, H, L, Dv, generator=torch.Generator().manual_seed(1000 + rank)).to(x["q"].dtype)
    xd = {n: t.to(dev) for n, t in x.items()}
    dOd = dO.to(dev)
    sc = Dk ** -0.5
    # training pair: the forward leaves the chunk start states the backward reads
    prob = ops.make_problem(xd["q"], xd["v"], None, scale=sc, chunk=64, plan="auto")
    saved = torch.empty(max(ops.gla_deltanet_saved_bytes(prob), 16), dtype=torch.uint8, device=dev)
    ws = torch.empty(_lib.lib.gla_deltanet_bwd_workspace_bytes(ctypes.byref(prob)), dtype=torch.uint8, device=dev)

    def step():
        ops.gla_deltanet_fwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], scale=sc, saved_states=saved)
        ops.gla_deltanet_bwd(xd["q"], xd["k"], xd["v"], xd["beta"], xd["h0"], dOd, None, scale=sc, workspace=ws,
                             saved_states=saved)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()

    def timed(per_kernel):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        n0 = _lib.launch_count()
        _lib.profiler_enable(per_kernel)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        _lib.profiler_enable(False)
        return sum(a.elapsed_time(b) for a, b in ev), _lib.launch_count() - n0, (_lib.profiler_read() if per_kernel
                                                                                 else {})

    total_ms, launches, _ = timed(False)
    _, _, kprof = timed(True)
    clocks = sampler.stop()
    total_ms = max_over_ranks(total_ms, dev)
    tokens = B * L * args.steps * world

    e2e = None
    if not args.no_e2e:
        xh = {n: t.pin_memory() for n, t in x.items()}
        dOh = dO.pin_memory()
        h2d = 2 * sum(t.numel() * t.element_size() for t in xh.values()) + dOh.numel() * dOh.element_size()
        d2h = 0

        def e2e_step():
            nonlocal d2h
            o, hT = ops.gla_deltanet_fwd(xh["q"], xh["k"], xh["v"], xh["beta"], xh["h0"], scale=sc,
                                         saved_states=saved)
            r = ops.gla_deltanet_bwd(xh["q"], xh["k"], xh["v"], xh["beta"], xh["h0"], dOh, None, scale=sc,
                                     saved_states=saved)
            d2h = sum(t.numel() * t.element_size() for t in [o, hT, *r.values()] if t is not None)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(args.steps):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(s0.elapsed_time(s1), dev)
        e2e = {"value": tokens / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h)}

    if rank != 0:
        return
    # bf16 I/O runs the chunk products on the tensor cores (against the measured bf16 GEMM peak);
    # fp32 I/O on the CUDA cores (against the FP32 FMA peak derived from the unit counts)
    tensor = I.DELTANET["dtype"] == "bf16"
    peaks, peak_src = load_peaks()
    peak = peaks["bf16_tflops"] if tensor else deltanet_alu_peak_tflops(clocks.get("sm_max_mhz"))
    roofline = None
    if kprof:
        name, (cnt, ms) = max(kprof.items(), key=lambda kv: kv[1][1])
        avg_s = ms / cnt / 1e3
        fl = deltanet_kernel_flops(name, B, H, L, Dk, Dv)
        ach = fl / avg_s / 1e12
        roofline = {"bound": "tensor" if tensor else "alu", "kernel": name, "achieved": ach, "peak": peak,
                    "unit": "TFLOP/s", "frac": ach / peak,
                    "traffic": measured_traffic(name, "deltanet") if tensor else None,
                    "peak_source": peak_src if tensor else
                    "nominal, derived (not measured): 148 SMs x 128 FP32 lanes x 2 FLOPs x the sampled max SM clock",
                    "algorithmic_flops_per_launch": fl, "avg_launch_us": avg_s * 1e6,
                    "share_of_step": ms / sum(v[1] for v in kprof.values())}
    extra = {"e2e": e2e, "gpu_launches": int(launches), "roofline": roofline, "clocks": clocks,
             "kernels": {n: {"launches": c, "avg_us": 1e3 * m / c} for n, (c, m) in sorted(kprof.items())}}
    if world == 1 and not args.no_cpu_baseline:
        tk, dt = deltanet_oracle_sample(0, heads)
        extra["cpu_baseline"] = {"value": tk / dt, "unit": "tokens/s", "cores": blas_threads(),
                                 "kind": "oracle", "sample": f"{heads} of {B * H} heads, full L={L}, fwd+bwd, "
                                                             f"float64 numpy, {dt:.1f} s"}
    print(json.dumps(deltanet_line(args, world, tokens, total_ms, extra)), flush=True)


def run_shard(args, world, rank, local, nshards=8):
    """Sequence-sharded forward on one GPU: workload c4 (B=1 H=8 L=65536) cut into `nshards`
    contiguous shards that run one after another (virtual ranks, nothing waits across them).
    Per step: gla_shard_state on every shard, then per shard gla_state_fold (its initial state
    from the earlier shards' pairs) and gla_fwd from that state. Timed against one gla_fwd over
    the whole sequence, with the same method as the main line. The per-rank estimate on
    `nshards` GPUs is one shard's state pass + fold + forward (the all-gather, ~0.5 MB per rank,
    is not measured here: every call of this build has one GPU)."""
    from linear_rnn_b200 import _lib, ops
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = I.WORKLOADS["c4"]
    x = I.make_inputs(w, seed=rank)
    xd = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    Ls = w.L // nshards
    sh = [{n: (None if xd[n] is None else xd[n][:, :, r * Ls:(r + 1) * Ls].contiguous())
           for n in ("q", "k", "v", "g", "igate")} for r in range(nshards)]
    kw = dict(scale=w.scale, chunk=w.chunk)

    def whole():
        ops.gla_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], **kw)

    def sharded():
        pairs = [ops.gla_shard_state(t["k"], t["v"], t["g"], t["igate"], chunk=w.chunk) for t in sh]
        states = torch.stack([p[0] for p in pairs])
        gammas = torch.stack([p[1] for p in pairs])
        for r, t in enumerate(sh):
            s_in = ops.gla_state_fold(states, gammas, r, xd["h0"])
            ops.gla_fwd(t["q"], t["k"], t["v"], t["g"], t["igate"], s_in, **kw)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    res = {}
    for name, fn in (("whole", whole), ("sharded", sharded)):
        for i in range(args.warmup):
            flush.fill_(i & 0xFF)
            fn()
        torch.cuda.synchronize()
        tot, per, n, _ = time_steps(fn, flush, args.steps, world)
        _, _, _, kp = time_steps(fn, flush, args.steps, world, per_kernel=True)
        res[name] = {"us_per_step": 1e3 * max_over_ranks(tot, dev) / args.steps, "launches_per_step": n / args.steps,
                     "kernels_us_per_step": {k: 1e3 * m / args.steps for k, (c, m) in sorted(kp.items())}}
    clocks = sampler.stop()
    if rank != 0:
        return
    ks = res["sharded"]["kernels_us_per_step"]
    per_rank = sum(ks.values()) / nshards
    t_whole = res["whole"]["us_per_step"]
    line = {"metric": "sequence-sharded GLA forward, one GPU with virtual shards", "unit": "us",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "higher_is_better": False,
            "scaling": "strong", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded; linear_rnn_b200/inputs.py)",
            "config": {"workload": f"c4 forward, B={w.B} H={w.H} L={w.L} Dk={w.Dk} Dv={w.Dv} chunk={w.chunk} bf16, "
                                   f"cut into {nshards} shards of {Ls} tokens",
                       "l2": "256 MiB L2 flush between steps, outside the per-step events; inputs > L2"},
            "value": res["sharded"]["us_per_step"], "ms_per_step": res["sharded"]["us_per_step"] / 1e3,
            "whole_sequence_us": t_whole, "sharded": res["sharded"], "whole": res["whole"],
            "per_rank_estimate_us": per_rank,
            "per_rank_estimate_note": f"kernel time of one shard's state pass + fold + forward (sum over the "
                                      f"{nshards} shards / {nshards}); all-gather not included",
            "overhead_vs_ideal": per_rank / (t_whole / nshards), "clocks": clocks,
            "gpu_launches": int(res["sharded"]["launches_per_step"] * args.steps)}
    print(json.dumps(line), flush=True)


def mlstm_oracle_sample(seed, heads):
    """Times the float64 mLSTM oracle (stabilised recurrence, then its gradients) on `heads`
    whole heads of the mLSTM workload. Returns (tokens_equivalent, seconds)."""
    from oracle import mlstm as ML
    w = I.MLSTM.replace(B=1, H=heads)
    x = I.make_mlstm_inputs(w, seed=seed)
    t0 = time.perf_counter()
    ML.mlstm_fwd(x["q"], x["k"], x["v"], x["g"], x["itil"], w.scale)
    ML.mlstm_bwd(x["q"], x["k"], x["v"], x["g"], x["itil"], x["dh"], w.scale)
    return w.L * heads / I.MLSTM.H, time.perf_counter() - t0


def run_mlstm(args, world, rank, local):
    """mLSTM cell forward+backward on its workload (B=2 H=8 L=8192 Dk=Dv=256, bf16): one step is
    gla_mlstm_fwd then gla_mlstm_bwd through the C ABI on HBM-resident inputs. The plan is the
    tensor-core one (numerator on the tensor cores in bf16, normaliser recurrence in fp32) unless
    --plan names another."""
    w = I.MLSTM
    mplan = "tc" if args.plan == "auto" else args.plan
    th = w.B * w.H * w.L
    e = 2
    # compulsory bytes: q, k, v, g, i~ read and h written (forward); q, k, v, g, i~, dh read and
    # dq, dk, dv, dg, d i~ written (backward)
    fwd_b = th * ((2 * w.Dk + w.Dv) * e + 8 + w.Dv * e)
    bwd_b = th * ((2 * w.Dk + 2 * w.Dv) * e + 8 + (2 * w.Dk + w.Dv) * e + 8)
    base = {"metric": "mLSTM cell fwd+bwd tokens/s", "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded; linear_rnn_b200/inputs.py)",
            "config": {"workload": f"mlstm: exponential input gate, normaliser, stabiliser; B={w.B} H={w.H} L={w.L} "
                                   f"Dk={w.Dk} Dv={w.Dv} chunk={w.chunk} bf16",
                       "global_batch": w.B * world, "seq_len": w.L, "parallelism": f"replicas x{world}",
                       "plan": mplan,
                       "l2": "256 MiB L2 flush between steps, outside the per-step events; inputs > L2"}}
    if args.impl == "reference":
        if rank != 0:
            return
        for _ in range(args.warmup):
            mlstm_oracle_sample(0, 1)
        tok = tot = 0.0
        for i in range(args.steps):
            t, dt = mlstm_oracle_sample(i, 1)
            tok += t
            tot += dt
        val = tok / tot
        base.update({"impl": "reference", "value": val, "ms_per_step": 1e3 * w.B * w.L / val, "dtype": "f64",
                     "gpu_launches": 0,
                     "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                      "sample": f"1 of {w.B * w.H} heads, full L={w.L}, fwd+bwd per step"},
                     "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        print(json.dumps(base), flush=True)
        return
    from linear_rnn_b200 import ops
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    x = I.make_mlstm_inputs(w, seed=rank)
    xd = {k: v.to(dev) for k, v in x.items()}
    kw = dict(scale=w.scale, chunk=w.chunk, plan=mplan)
    prob = ops.make_problem(xd["q"], xd["v"], xd["g"], scale=w.scale, chunk=w.chunk, plan=mplan)
    from linear_rnn_b200 import _lib
    ws = torch.empty(max(_lib.lib.gla_mlstm_workspace_bytes(ctypes.byref(prob), 0),
                         _lib.lib.gla_mlstm_workspace_bytes(ctypes.byref(prob), 1)), dtype=torch.uint8, device=dev)
    # training pair: the forward keeps its results for the backward
    saved = torch.empty(max(ops.gla_mlstm_saved_bytes(prob), 16), dtype=torch.uint8, device=dev)

    def step():
        ops.gla_mlstm_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["itil"], workspace=ws, saved_states=saved, **kw)
        ops.gla_mlstm_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["itil"], xd["dh"], workspace=ws, saved_states=saved,
                          **kw)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()
    tot, per, launches, _ = time_steps(step, flush, args.steps, world)
    _, _, _, kp = time_steps(step, flush, args.steps, world, per_kernel=True)
    clocks = sampler.stop()
    tot = max_over_ranks(tot, dev)
    e2e = None
    if not args.no_e2e:
        xh = {k: v.pin_memory() for k, v in x.items()}
        h2d = 2 * sum(t.numel() * t.element_size() for n, t in xh.items() if n != "dh") + \
            xh["dh"].numel() * xh["dh"].element_size()
        d2h = 0

        def e2e_step():
            nonlocal d2h
            h = ops.gla_mlstm_fwd(xh["q"], xh["k"], xh["v"], xh["g"], xh["itil"], saved_states=saved, **kw)
            r = ops.gla_mlstm_bwd(xh["q"], xh["k"], xh["v"], xh["g"], xh["itil"], xh["dh"], saved_states=saved, **kw)
            d2h = sum(t.numel() * t.element_size() for t in [h, *r.values()])

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(args.steps):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(s0.elapsed_time(s1), dev)
        e2e = {"value": w.B * w.L * args.steps * world / (e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    t = tot / args.steps / 1e3
    by = fwd_b + bwd_b
    base.update({"value": w.B * w.L * world / t, "ms_per_step": tot / args.steps, "e2e": e2e,
                 "gpu_launches": int(launches), "clocks": clocks,
                 "step_roofline": {"gbs_compulsory": by / t / 1e9, "roofline_us": by / (peaks["hbm_gbs"] * 1e9) * 1e6,
                                   "frac": by / (peaks["hbm_gbs"] * 1e9) / t, "peak_source": peak_src,
                                   "bound": "hbm (compulsory bytes of the cell's inputs and outputs)"},
                 "kernels": {n: {"launches": c, "avg_us": 1e3 * m / c} for n, (c, m) in sorted(kp.items())}})
    if world == 1 and not args.no_cpu_baseline:
        tk, dt = mlstm_oracle_sample(0, 1)
        base["cpu_baseline"] = {"value": tk / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"1 of {w.B * w.H} heads, full L={w.L}, fwd+bwd, float64, {dt:.1f} s"}
    print(json.dumps(base), flush=True)


def time_steps(step, flush, steps, world, per_kernel=False, flush_l2=True):
    """K steps bracketed by barrier + synchronize; per-step CUDA events on the stream, with the
    256 MiB L2 flush before each step outside the events (flush_l2=False: warm L2). per_kernel:
    the library also brackets every launch with CUDA events (per-kernel durations), which costs
    a few microseconds per launch, so step times come from a pass without it.
    Returns (total_ms, per-step ms list, library launches, per-kernel profile)."""
    from linear_rnn_b200 import _lib
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    n0 = _lib.launch_count()
    _lib.profiler_enable(per_kernel)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    flush.fill_(0xA5)   # lead-in (outside the events): the host queues step 0 while this runs
    for i in range(steps):
        if flush_l2:
            flush.fill_(i & 0xFF)
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    _lib.profiler_enable(False)
    n = _lib.launch_count() - n0
    kp = _lib.profiler_read() if per_kernel else {}
    per = [a.elapsed_time(b) for a, b in ev]
    return sum(per), per, n, kp


def forward_targets(args, world, dev, flush):
    """The bf16 GLA forward at L >= 2048 on its own (workloads c2 and c4, forward only),
    timed like the main line: warm-up, then K steps with the L2 flush between them, CUDA
    events per step, max over ranks. Returns {workload: {...}} with each step's fraction of
    its roofline max(FLOPs / bf16 peak, compulsory bytes / HBM peak)."""
    from linear_rnn_b200 import ops
    peaks, peak_src = load_peaks()
    out = {}
    for name in ("c2", "c4"):
        w = I.WORKLOADS[name]
        x = I.make_inputs(w, seed=0)
        xd = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
        kw = dict(scale=w.scale, chunk=w.chunk, plan=args.plan)
        prob = ops.make_problem(xd["q"], xd["v"], xd["g"], **kw)
        ws = torch.empty(ops.gla_workspace_bytes(prob, False), dtype=torch.uint8, device=dev)

        def step():
            ops.gla_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], workspace=ws, **kw)

        for i in range(args.warmup):
            flush.fill_(i & 0xFF)
            step()
        torch.cuda.synchronize()
        tot, per, _, _ = time_steps(step, flush, args.steps, world)
        tot = max_over_ranks(tot, dev)
        t = tot / args.steps / 1e3
        fl, by = flops(w, False), compulsory_bytes(w, False)
        roof = max(fl / (peaks["bf16_tflops"] * 1e12), by / (peaks["hbm_gbs"] * 1e9))
        out[name] = {"workload": f"GLA forward, B={w.B} H={w.H} L={w.L} Dk={w.Dk} Dv={w.Dv} chunk={w.chunk} bf16",
                     "us_per_step": t * 1e6, "us_median": statistics.median(per) * 1e3,
                     "tokens_per_s": w.B * w.L * world / t, "tflops": fl / t / 1e12,
                     "gbs_compulsory": by / t / 1e9, "roofline_us": roof * 1e6, "frac": roof / t,
                     "peak_source": peak_src}
        del xd, ws
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="c3",
                    choices=sorted(I.WORKLOADS) + ["decode", "deltanet", "shard", "mlstm"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--plan", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fwd-target", action="store_true",
                    help="skip the forward-only c2 / c4 measurements added to the c3 line")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch B (smaller cases for profiling; not a bench line)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.workload in ("deltanet", "shard", "mlstm"):
        world, rank, local = dist_setup()
        if args.workload == "deltanet":
            run_deltanet(args, world, rank, local)
        elif args.workload == "mlstm":
            run_mlstm(args, world, rank, local)
        elif args.impl != "reference":
            run_shard(args, world, rank, local)
        elif rank == 0:
            print(json.dumps({"impl": "reference", "unavailable": "the sharded forward has no oracle arm of its own; "
                              "its parity is tested against the oracle over the whole sequence"}), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    w = I.DECODE if args.workload == "decode" else I.WORKLOADS[args.workload]
    decode = w.name == "decode"
    if args.batch is not None:
        w = w.replace(B=args.batch)
    world, rank, local = dist_setup()
    if args.impl == "reference":
        run_reference(args, w, world, rank)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    from linear_rnn_b200 import _lib, ops
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    x = I.make_inputs(w, seed=rank)
    xd = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    kw = dict(scale=w.scale, chunk=w.chunk, plan=args.plan)
    prob = ops.make_problem(xd["q"], xd["v"], xd["g"], **kw)
    _, fseg, _ = _lib.plan_info(prob, False)
    bplan, bseg, _ = _lib.plan_info(prob, True)
    bseg = bseg if (w.backward and bplan == _lib.GLA_PLAN_TC) else 1
    ws = torch.empty(max(ops.gla_workspace_bytes(prob, False), ops.gla_workspace_bytes(prob, True) if w.backward
                         else 0), dtype=torch.uint8, device=dev)

    # training pair: the forward leaves the states the backward's segments start from
    nsaved = ops.gla_saved_states_bytes(prob) if w.backward else 0
    saved = torch.empty(max(nsaved // 4, 1), dtype=torch.float32, device=dev) if nsaved else None

    def step():
        if decode:   # one token per (b, h) from the state, updated in place (xd["h0"])
            ops.gla_decode(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], scale=w.scale)
            return
        ops.gla_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], workspace=ws, saved_states=saved,
                    **kw)
        if w.backward:
            ops.gla_bwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["igate"], xd["h0"], xd["dO"], None, workspace=ws,
                        saved_states=saved, **kw)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    # warm-up right before the timed steps (same pattern, flush included), so that the timed
    # region starts with warm clocks and the host already ahead of the device
    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()

    total_ms, per_ms, launches, _ = time_steps(step, flush, args.steps, world)
    prof_ms, _, _, kprof = time_steps(step, flush, args.steps, world, per_kernel=True)
    warm_ms, warm_per, _, _ = time_steps(step, flush, args.steps, world, flush_l2=False)
    ftarget = None
    if w.name == "c3" and args.batch is None and not args.no_fwd_target and args.plan != "simt":
        ftarget = forward_targets(args, world, dev, flush)
    clocks = sampler.stop()
    total_ms = max_over_ranks(total_ms, dev)
    tokens = w.B * w.L * args.steps * world
    value = tokens / (total_ms / 1e3)

    # ------- end to end: host (pinned) tensors through the public API
    e2e = None
    if not args.no_e2e:
        xh = {k: (None if v is None else v.pin_memory()) for k, v in x.items()}
        h2d = sum(t.numel() * t.element_size() for n, t in xh.items()
                  if t is not None and n in ("q", "k", "v", "g", "igate", "h0"))
        d2h = 0

        def e2e_step():
            nonlocal d2h
            if decode:   # the state stays on the device; the token's inputs come from the host
                o = ops.gla_decode(*(None if xh[n] is None else xh[n].to(dev, non_blocking=True)
                                     for n in ("q", "k", "v", "g", "igate")), xd["h0"], scale=w.scale).cpu()
                d2h = o.numel() * o.element_size()
                return
            o, hT = ops.gla_fwd(xh["q"], xh["k"], xh["v"], xh["g"], xh["igate"], xh["h0"], saved_states=saved,
                                **kw)
            nb = o.numel() * o.element_size() + hT.numel() * hT.element_size()
            if w.backward:
                r = ops.gla_bwd(xh["q"], xh["k"], xh["v"], xh["g"], xh["igate"], xh["h0"], xh["dO"], None,
                                saved_states=saved, **kw)
                nb += sum(t.numel() * t.element_size() for t in r.values() if t is not None)
            d2h = nb

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(args.steps):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        e_ms = s0.elapsed_time(s1)
        e_ms = max_over_ranks(e_ms, dev)
        h2d_step = h2d * (2 if w.backward else 1) + (sum(xh[n].numel() * xh[n].element_size() for n in ("dO",))
                                                     if w.backward else 0)
        if decode:
            h2d_step = sum(xh[n].numel() * xh[n].element_size() for n in ("q", "k", "v", "g", "igate")
                           if xh[n] is not None)
        e2e = {"value": tokens / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d_step),
               "d2h_bytes_per_step": int(d2h)}

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    peaks, peak_src = load_peaks()
    fl = flops(w, w.backward)
    by = compulsory_bytes(w, w.backward)
    t_step = total_ms / args.steps / 1e3
    roof_t = max(fl / (peaks["bf16_tflops"] * 1e12), by / (peaks["hbm_gbs"] * 1e9))
    dom = max(kprof.items(), key=lambda kv: kv[1][1]) if kprof else None
    roofline = None
    if dom:
        name, (cnt, ms) = dom
        avg_s = ms / cnt / 1e3
        mb, pb = kernel_bytes(name, w, fseg, bseg)
        ach = mb / avg_s / 1e9
        share = ms / sum(v[1] for v in kprof.values())
        roofline = {"bound": "hbm", "kernel": name, "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"],
                    "traffic": measured_traffic(name, w.name if args.batch is None else None),
                    "peak_source": peak_src,
                    "algorithmic_bytes_per_launch": mb, "plan_bytes_per_launch": pb,
                    "frac_with_plan_bytes": (mb + pb) / avg_s / 1e9 / peaks["hbm_gbs"],
                    "bytes_note": "algorithmic = the path's inputs this kernel reads and outputs it writes, "
                                  "once each; plan = workspace intermediates (segment states, prefixes)",
                    "avg_launch_us": avg_s * 1e6, "share_of_step": share}
    line = base_line(w, args, world)
    line.update({"value": value, "ms_per_step": total_ms / args.steps, "e2e": e2e, "gpu_launches": int(launches),
                 "roofline": roofline, "clocks": clocks,
                 "step_roofline": {"tflops": fl / t_step / 1e12, "gbs_compulsory": by / t_step / 1e9,
                                   "roofline_us": roof_t * 1e6, "frac": roof_t / t_step, "peak_source": peak_src},
                 "step_ms": {"median": statistics.median(per_ms), "min": min(per_ms), "max": max(per_ms),
                             "warm_l2_median": statistics.median(warm_per),
                             "note": "rank 0's per-step CUDA-event times; warm_l2 = a third pass without the "
                                     "L2 flush"},
                 "kernels": {n: {"launches": c, "avg_us": 1e3 * m / c} for n, (c, m) in sorted(kprof.items())},
                 "kernel_timing": {"source": "a second pass of the same K steps with CUDA events around "
                                             "every library launch (kernels, roofline); value and "
                                             "ms_per_step come from the pass without them",
                                   "ms_per_step_instrumented": prof_ms / args.steps},
                 "plan": args.plan})
    if ftarget is not None:
        line["fwd_target"] = ftarget
    if world == 1 and not args.no_cpu_baseline:
        heads = oracle_heads(w)
        tk, dt, thr = oracle_sample(w, 0, heads)
        line["cpu_baseline"] = {"value": tk / dt, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                                "sample": f"{heads} of {w.B * w.H} heads, full L={w.L}, "
                                          f"{'fwd+bwd' if w.backward else 'fwd'}, float64, {dt:.1f} s"}
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
