"""Multi-process paths on the CPU (gloo, world_size 2): the benchmark's max-over-ranks
timing reduction, per-rank input seeding of the replicas, and the reference arm under
torchrun (rank 0 prints one JSON line, the other rank exits 0 without work)."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    from linear_rnn_b200 import inputs as I
    m = bench.max_over_ranks(10.0 + rank * 5.0, torch.device("cpu"))
    w = I.small(I.WORKLOADS["c2"], B=1, H=1, L=64)
    digest = I.input_digest(I.make_inputs(w, seed=rank))
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    out.put((rank, m, digest))


def test_max_over_ranks_and_replica_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert res[0][1] == res[1][1] == 15.0       # every rank sees the max
    assert res[0][2] != res[1][2]               # replicas draw different batches


def test_max_over_ranks_without_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5


def test_reference_arm_json_contract():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "c1",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["value"] > 0


def test_deltanet_reference_arm_and_flop_model():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "deltanet", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"].startswith("DeltaNet") and d["value"] > 0
    assert d["config"]["workload"].startswith("deltanet:") and d["e2e"]["d2h_bytes_per_step"] == 0
    sys.path.insert(0, ROOT)
    import bench
    # per token-head at C = 64, Dk = Dv = 128 on the tensor-core plan (the bf16 workload): the chunk
    # products and the substitution, no triangular inverse: 2*64*128 + 6*128^2 + 2*64*128
    per = 2 * 64 * 128 + 6 * 128 * 128 + 2 * 64 * 128
    assert bench.deltanet_kernel_flops("deltanet_fwd", 1, 2, 10, 128, 128) == per * 20
    # the gradient kernel: 5 C Dk + 8 Dk Dv + 3 C Dv
    assert bench.deltanet_kernel_flops("deltanet_bwd_grads", 1, 1, 1, 128, 128) == 5 * 64 * 128 + 8 * 128 * 128 + 3 * 64 * 128
    assert bench.deltanet_kernel_flops("other", 1, 1, 1, 64, 64) == 0.0
    assert abs(bench.deltanet_alu_peak_tflops(1965.0) - 74.45) < 0.01


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "c1", "--steps", "1", "--warmup", "3", "--gpus", "2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["impl"] == "reference"


# ----------------------------------------------- sequence-sharded forward, exchange on CPU ranks
def _shard_worker(rank, world, port, out):
    """Each rank holds one contiguous shard; the per-rank steps are the float64 oracle (this
    tests the exchange and the fold order, not the kernels)."""
    import datetime

    import numpy as np
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import oracle
    from linear_rnn_b200 import inputs as I
    from linear_rnn_b200 import ops
    w = I.WORKLOADS["c3"].replace(B=1, H=2, L=150, Dk=64, Dv=64, dtype="f32", input_gate=True, h0_std=0.5)
    x = I.make_inputs(w, seed=7)
    cuts = [0, 70, 150]
    sl = lambda t: None if t is None else t[:, :, cuts[rank]:cuts[rank + 1]].contiguous()
    xs = {n: sl(x[n]) for n in ("q", "k", "v", "g", "igate")}

    def shard_state():
        _, S = oracle.gla_fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["igate"], None, w.scale)
        gam = xs["g"].double().sum(dim=2)
        return torch.from_numpy(S), gam

    def fold(states, gammas):
        S = x["h0"].double().clone()
        for p in range(rank):
            S = torch.exp(gammas[p])[..., None] * S + states[p]
        return S

    def fwd(s_in):
        return oracle.gla_fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["igate"], s_in.numpy(), w.scale)

    o, hT = ops.gla_fwd_sequence_sharded(None, None, None, _shard_ops=(shard_state, fold, fwd))
    ro, rS = oracle.gla_fwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], w.scale)
    err_o = float(np.abs(o - ro[:, :, cuts[rank]:cuts[rank + 1]]).max() / np.abs(ro).max())
    err_h = float(np.abs(hT - rS).max() / np.abs(rS).max()) if rank == world - 1 else 0.0
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    out.put((rank, err_o, err_h))


def test_sequence_sharded_forward_exchange_on_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err_o, err_h in res:
        assert err_o < 1e-10 and err_h < 1e-10, (rank, err_o, err_h)


# ---------------------------------------------- sequence-sharded backward, exchange on CPU ranks
def _shard_bwd_worker(rank, world, port, out):
    """Three ranks, one contiguous shard each; the per-rank steps are the float64 oracle (the
    start-state gradient from zero of a shard is the oracle's dh0 of that shard alone), so
    this tests the single packed all-gather and both fold orders, not the kernels."""
    import datetime

    import numpy as np
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import oracle
    from linear_rnn_b200 import inputs as I
    from linear_rnn_b200 import ops
    w = I.WORKLOADS["c3"].replace(B=1, H=2, L=150, Dk=64, Dv=64, dtype="f32", input_gate=True, h0_std=0.5)
    x = I.make_inputs(w, seed=8)
    dhT = I.make_dhT(w, seed=9)
    cuts = [0, 40, 41, 150]
    sl = lambda t: None if t is None else t[:, :, cuts[rank]:cuts[rank + 1]].contiguous()
    xs = {n: sl(x[n]) for n in ("q", "k", "v", "g", "igate", "dO")}

    def shard_state():
        _, S = oracle.gla_fwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["igate"], None, w.scale)
        return torch.from_numpy(S), xs["g"].double().sum(dim=2)

    def shard_grad():
        r = oracle.gla_bwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["igate"], None, xs["dO"], None, w.scale)
        return torch.from_numpy(r["dh0"]), xs["g"].double().sum(dim=2)

    def fold(states, gammas, count, init):
        S = torch.zeros_like(states[0]) if init is None else init.double().clone()
        for p in range(count):
            S = torch.exp(gammas[p])[..., None] * S + states[p]
        return S

    def bwd(s_in, d_end):
        return oracle.gla_bwd(xs["q"], xs["k"], xs["v"], xs["g"], xs["igate"], s_in.numpy(), xs["dO"],
                              d_end.numpy(), w.scale)

    r = ops.gla_bwd_sequence_sharded(None, None, None, None, None, x["h0"], None, dhT,
                                     _shard_ops=(shard_state, shard_grad, fold, bwd))
    ref = oracle.gla_bwd(x["q"], x["k"], x["v"], x["g"], x["igate"], x["h0"], x["dO"], dhT, w.scale)
    errs = {}
    for n in ("dq", "dk", "dv", "dg", "di"):
        part = ref[n][:, :, cuts[rank]:cuts[rank + 1]]
        errs[n] = float(np.abs(r[n] - part).max() / np.abs(ref[n]).max())
    if rank == 0:
        errs["dh0"] = float(np.abs(r["dh0"] - ref["dh0"]).max() / np.abs(ref["dh0"]).max())
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    out.put((rank, errs))


def test_sequence_sharded_backward_exchange_on_three_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_bwd_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, errs in res:
        assert (rank != 0) or "dh0" in errs
        assert all(e < 1e-10 for e in errs.values()), (rank, errs)
