"""Host-only checks of the C ABI: the library loads, exports every symbol that
include/gla.h declares, and validates arguments on the host (no GPU needed: every call
here fails validation before any CUDA call)."""
import ctypes
import os
import re
import subprocess

import pytest

from linear_rnn_b200 import _lib, build
from linear_rnn_b200._lib import GlaProblem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    syms = set()
    for name in os.listdir(os.path.join(ROOT, "include")):
        if name.endswith(".h"):
            text = open(os.path.join(ROOT, "include", name)).read()
            syms |= set(re.findall(r"GLA_API\s+[\w\s\*]+?\b(gla_\w+)\s*\(", text))
    return syms


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert {"gla_fwd", "gla_bwd", "gla_workspace_bytes"} <= syms
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gla_\w+)", out))
    assert syms <= exported, syms - exported
    assert set(_lib.EXPORTED) == syms
    for s in syms:
        assert hasattr(_lib.lib, s)


def test_library_is_built_for_sm100a_only():
    out = subprocess.run(["cuobjdump", "--list-elf", build.LIB], capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    archs = set(re.findall(r"sm_\w+", out.stdout))
    assert archs == {"sm_100a"}, archs


def prob(**kw):
    base = dict(B=2, H=3, L=300, Dk=128, Dv=64, chunk=64, scale=0.1, io=_lib.GLA_BF16,
                gate=_lib.GLA_GATE_PER_KEY, plan=_lib.GLA_PLAN_SIMT)
    base.update(kw)
    return GlaProblem(*[base[f] for f, _ in GlaProblem._fields_])


def ws_bytes(**kw):
    p = prob(**kw)
    return _lib.lib.gla_workspace_bytes(ctypes.byref(p), 0), _lib.lib.gla_workspace_bytes(ctypes.byref(p), 1)


def test_workspace_sizes():
    f, b = ws_bytes()
    assert 0 < f < b
    # states at chunk boundaries only: ceil(300/64) = 5 states of 128x64 fp32 per head
    assert f >= 2 * 3 * 5 * 128 * 64 * 4
    assert ws_bytes(Dk=96) == (0, 0)
    assert ws_bytes(chunk=24) == (0, 0)
    assert ws_bytes(chunk=2048) == (0, 0)
    assert ws_bytes(L=-1) == (0, 0)
    assert ws_bytes(io=7) == (0, 0)
    assert ws_bytes(gate=9) == (0, 0)
    # larger chunks materialise fewer states
    assert ws_bytes(chunk=256)[0] < ws_bytes(chunk=64)[0]


def test_saved_state_sizes_follow_the_backward_plan():
    saved = lambda **kw: _lib.lib.gla_saved_states_bytes(ctypes.byref(prob(**kw)))
    # tensor-core backward in several segments: one f32 state per (head, segment)
    p = prob(B=4, H=16, L=4096, Dk=128, Dv=256, plan=_lib.GLA_PLAN_AUTO)
    _, nseg, _ = _lib.plan_info(p, True)
    assert nseg > 1
    assert saved(B=4, H=16, L=4096, Dk=128, Dv=256, plan=_lib.GLA_PLAN_AUTO) == 4 * 64 * nseg * 128 * 256
    assert saved(plan=_lib.GLA_PLAN_SIMT) == 0            # CUDA-core backward recomputes
    assert saved(io=_lib.GLA_F32, plan=_lib.GLA_PLAN_AUTO) == 0
    assert saved(Dk=96) == 0                                # invalid problem


def test_backward_segments_whole_chunks_and_bounded():
    """Backward segments are whole chunks of about ten tiles at most (dg's accuracy bound)
    unless one chunk is longer, and cover the sequence. Without a GPU the library assumes 148
    SMs."""
    auto = _lib.GLA_PLAN_AUTO
    for B, H, L, Dk, Dv, C in [(4, 16, 4096, 128, 256, 64), (2, 8, 8192, 256, 256, 64), (1, 2, 333, 256, 128, 64),
                               (1, 8, 65536, 128, 128, 256), (1, 1, 5000, 64, 64, 1024), (3, 5, 1, 64, 64, 64)]:
        plan, nseg, tps = _lib.plan_info(prob(B=B, H=H, L=L, Dk=Dk, Dv=Dv, chunk=C, plan=auto), True)
        ntiles = -(-L // 64)
        assert plan == _lib.GLA_PLAN_TC
        assert tps % (C // 64) == 0 and tps < 10 + C // 64   # ten tiles, rounded up to whole chunks
        assert nseg == -(-ntiles // tps)
    # c3: 7 segments of 10 tiles per head; c5: 13 of 10 per (head, key block)
    assert _lib.plan_info(prob(B=4, H=16, L=4096, Dk=128, Dv=256, plan=auto), True) == (_lib.GLA_PLAN_TC, 7, 10)
    assert _lib.plan_info(prob(B=2, H=8, L=8192, Dk=256, Dv=256, plan=auto), True) == (_lib.GLA_PLAN_TC, 13, 10)
    # Dk = 256 runs on tensor cores with Dv >= 128 (the key-split CTA pair), else on CUDA cores
    assert _lib.plan_info(prob(Dk=256, Dv=64, plan=auto), True)[0] == _lib.GLA_PLAN_SIMT


def test_status_strings():
    for s in range(7):
        assert len(_lib.status_string(s)) >= 2
    assert "range" in _lib.status_string(_lib.GLA_ERR_RANGE)
    assert "unknown" in _lib.status_string(99)


def _fwd(p, **ptrs):
    args = dict(q=16, k=16, v=16, g=16, ig=None, h0=None, o=16, hT=None, ws=16, nbytes=1 << 30)
    args.update(ptrs)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    return _lib.lib.gla_fwd(ctypes.byref(p), vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["g"]),
                            vp(args["ig"]), vp(args["h0"]), vp(args["o"]), vp(args["hT"]), vp(args["ws"]),
                            args["nbytes"], None)


def test_fwd_argument_validation_happens_before_launch():
    p = prob()
    assert _fwd(p, q=None) == _lib.GLA_ERR_INVALID_ARG
    assert _fwd(p, g=None) == _lib.GLA_ERR_INVALID_ARG           # gate mode says per-key
    assert _fwd(prob(gate=_lib.GLA_GATE_NONE)) == _lib.GLA_ERR_INVALID_ARG  # g given, no gate
    assert _fwd(p, k=24) == _lib.GLA_ERR_INVALID_ARG              # misaligned
    assert _fwd(p, ws=None) == _lib.GLA_ERR_INVALID_ARG
    assert _fwd(p, nbytes=100) == _lib.GLA_ERR_WORKSPACE
    assert _fwd(prob(Dv=32)) == _lib.GLA_ERR_UNSUPPORTED
    assert _fwd(prob(chunk=40)) == _lib.GLA_ERR_UNSUPPORTED
    assert _lib.lib.gla_fwd(None, None, None, None, None, None, None, None, None, None, 0, None) == \
        _lib.GLA_ERR_INVALID_ARG


def test_bwd_argument_validation_happens_before_launch():
    p = prob()
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(**kw):
        a = dict(q=16, k=16, v=16, g=16, ig=None, h0=None, dO=16, dhT=None, dq=16, dk=16, dv=16, dg=16,
                 di=None, dh0=None, ws=16, nbytes=1 << 30, p=p)
        a.update(kw)
        return _lib.lib.gla_bwd(ctypes.byref(a["p"]), *(vp(a[n]) for n in
                                ("q", "k", "v", "g", "ig", "h0", "dO", "dhT", "dq", "dk", "dv", "dg", "di", "dh0",
                                 "ws")), a["nbytes"], None)
    assert call(dO=None) == _lib.GLA_ERR_INVALID_ARG
    assert call(dg=None) == _lib.GLA_ERR_INVALID_ARG
    assert call(di=16) == _lib.GLA_ERR_INVALID_ARG       # di without an input gate
    assert call(dq=8) == _lib.GLA_ERR_INVALID_ARG
    assert call(nbytes=4096) == _lib.GLA_ERR_WORKSPACE


def test_decode_validates_before_launch():
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(p, **kw):
        a = dict(q=16, k=16, v=16, g=16, ig=None, state=16, o=16)
        a.update(kw)
        return _lib.lib.gla_decode(ctypes.byref(p), *(vp(a[n]) for n in ("q", "k", "v", "g", "ig", "state", "o")),
                                   None)
    one = prob(L=1)
    assert call(prob(L=2)) == _lib.GLA_ERR_INVALID_ARG              # one token per (b, h)
    assert call(one, state=None) == _lib.GLA_ERR_INVALID_ARG
    assert call(one, g=None) == _lib.GLA_ERR_INVALID_ARG            # gate mode says per-key
    assert call(prob(L=1, gate=_lib.GLA_GATE_NONE)) == _lib.GLA_ERR_INVALID_ARG   # g given, no gate
    assert call(one, v=24) == _lib.GLA_ERR_INVALID_ARG              # misaligned
    assert call(prob(L=1, Dk=96)) == _lib.GLA_ERR_UNSUPPORTED
    assert call(prob(L=1, io=7)) == _lib.GLA_ERR_INVALID_ARG
    assert _lib.lib.gla_decode(None, None, None, None, None, None, None, None, None) == _lib.GLA_ERR_INVALID_ARG


def test_shard_calls_validate_before_launch():
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def shard(p, **kw):
        a = dict(k=16, v=16, g=16, ig=None, state=16, gamma=16, ws=16, nbytes=256)
        a.update(kw)
        return _lib.lib.gla_shard_state(ctypes.byref(p), *(vp(a[n]) for n in ("k", "v", "g", "ig", "state", "gamma",
                                                                              "ws")), a["nbytes"], None)
    bf = prob(io=_lib.GLA_BF16)
    assert shard(prob(io=_lib.GLA_F32)) == _lib.GLA_ERR_UNSUPPORTED      # tensor-core state pass: bf16
    assert shard(prob(chunk=96)) == _lib.GLA_ERR_UNSUPPORTED             # whole 64-token tiles
    assert shard(bf, state=None) == _lib.GLA_ERR_INVALID_ARG
    assert shard(bf, g=None) == _lib.GLA_ERR_INVALID_ARG                 # gate mode says per-key
    assert shard(bf, k=24) == _lib.GLA_ERR_INVALID_ARG                   # misaligned
    assert shard(bf, nbytes=100) == _lib.GLA_ERR_WORKSPACE

    def grad(p, **kw):
        a = dict(q=16, dO=16, g=16, dS=16, gamma=16, ws=16, nbytes=256)
        a.update(kw)
        return _lib.lib.gla_shard_state_grad(ctypes.byref(p), *(vp(a[n]) for n in ("q", "dO", "g", "dS", "gamma",
                                                                                   "ws")), a["nbytes"], None)
    assert grad(prob(io=_lib.GLA_F32)) == _lib.GLA_ERR_UNSUPPORTED
    assert grad(prob(chunk=96)) == _lib.GLA_ERR_UNSUPPORTED
    assert grad(bf, dS=None) == _lib.GLA_ERR_INVALID_ARG
    assert grad(bf, dO=None) == _lib.GLA_ERR_INVALID_ARG
    assert grad(bf, g=None) == _lib.GLA_ERR_INVALID_ARG                  # gate mode says per-key
    assert grad(bf, q=24) == _lib.GLA_ERR_INVALID_ARG                    # misaligned
    assert grad(bf, nbytes=100) == _lib.GLA_ERR_WORKSPACE

    def fold(p, count, **kw):
        a = dict(states=16, gammas=16, h0=None, out=16)
        a.update(kw)
        return _lib.lib.gla_state_fold(ctypes.byref(p), count, *(vp(a[n]) for n in ("states", "gammas", "h0", "out")),
                                       None)
    assert fold(bf, -1) == _lib.GLA_ERR_INVALID_ARG
    assert fold(bf, 2, out=None) == _lib.GLA_ERR_INVALID_ARG
    assert fold(bf, 2, states=None) == _lib.GLA_ERR_INVALID_ARG
    assert fold(bf, 2, gammas=8) == _lib.GLA_ERR_INVALID_ARG             # misaligned
    assert fold(prob(Dv=96), 1) == _lib.GLA_ERR_UNSUPPORTED


def test_deltanet_validates_before_launch():
    vp = lambda x: None if x is None else ctypes.c_void_p(x)

    def call(p, **kw):
        a = dict(q=16, k=16, v=16, beta=16, h0=None, o=16, hT=None)
        a.update(kw)
        return _lib.lib.gla_deltanet_fwd(ctypes.byref(p), *(vp(a[n]) for n in ("q", "k", "v", "beta", "h0", "o",
                                                                              "hT")), None)
    dn = lambda **kw: prob(**dict(dict(gate=_lib.GLA_GATE_NONE, Dk=64, Dv=64), **kw))
    assert call(dn(gate=_lib.GLA_GATE_PER_KEY)) == _lib.GLA_ERR_INVALID_ARG   # no decay gates
    assert call(dn(io=7)) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(Dk=256)) == _lib.GLA_ERR_UNSUPPORTED
    assert call(dn(Dv=96)) == _lib.GLA_ERR_UNSUPPORTED                        # 64-column slices
    assert call(dn(chunk=128)) == _lib.GLA_ERR_UNSUPPORTED
    assert call(dn(), beta=None) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(), o=None) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(), k=24) == _lib.GLA_ERR_INVALID_ARG                       # misaligned
    assert call(dn(), hT=8) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(L=-1)) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(B=0)) == _lib.GLA_OK                                      # nothing to do, no launch
    assert _lib.lib.gla_deltanet_fwd(None, None, None, None, None, None, None, None, None) == \
        _lib.GLA_ERR_INVALID_ARG


def test_deltanet_backward_validates_before_launch():
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    names = ("q", "k", "v", "beta", "h0", "dO", "dhT", "dq", "dk", "dv", "dbeta", "dh0", "ws")

    def call(p, **kw):
        a = dict(q=16, k=16, v=16, beta=16, h0=None, dO=16, dhT=None, dq=16, dk=16, dv=16, dbeta=16, dh0=None,
                 ws=16, nbytes=1 << 40)
        a.update(kw)
        return _lib.lib.gla_deltanet_bwd(ctypes.byref(p), *(vp(a[n]) for n in names), a["nbytes"], None)
    dn = lambda **kw: prob(**dict(dict(gate=_lib.GLA_GATE_NONE, Dk=64, Dv=64), **kw))
    need = _lib.lib.gla_deltanet_bwd_workspace_bytes(ctypes.byref(dn()))
    # each region rounded up to 256 bytes. fp32 I/O (CUDA-core kernels): chunk start states and
    # end gradients (2 x B*H*5 chunks*Dk*Dv fp32), X and dR (2 x B*H*L*Dv fp32), per-slice sums
    # (B*H*L fp32). bf16 I/O (tensor-core kernels): the states and end gradients in bf16, dR fp32.
    BH, L = 6, 300
    rnd = lambda b: (b + 255) // 256 * 256
    st, tok = BH * 5 * 64 * 64, BH * L * 64
    assert _lib.lib.gla_deltanet_bwd_workspace_bytes(ctypes.byref(dn(io=_lib.GLA_F32))) == \
        sum(rnd(4 * n) for n in (st, tok, tok, st, BH * L))
    io = dn().io
    assert need == (rnd(2 * st) + rnd(4 * tok) + rnd(2 * st) if io == _lib.GLA_BF16 else
                    sum(rnd(4 * n) for n in (st, tok, tok, st, BH * L)))
    assert _lib.lib.gla_deltanet_bwd_workspace_bytes(ctypes.byref(dn(Dk=256))) == 0
    assert _lib.lib.gla_deltanet_bwd_workspace_bytes(ctypes.byref(dn(L=0))) == 256   # empty, still usable
    assert call(dn(), nbytes=need - 1) == _lib.GLA_ERR_WORKSPACE
    assert call(dn(), ws=None) == _lib.GLA_ERR_WORKSPACE
    assert call(dn(gate=_lib.GLA_GATE_PER_HEAD)) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(Dv=32)) == _lib.GLA_ERR_UNSUPPORTED
    assert call(dn(B=300, H=300)) == _lib.GLA_ERR_UNSUPPORTED             # B*H above 65535
    assert call(dn(), dO=None) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(), dbeta=None) == _lib.GLA_ERR_INVALID_ARG
    assert call(dn(), dq=8) == _lib.GLA_ERR_INVALID_ARG                   # misaligned
    assert call(dn(H=0)) == _lib.GLA_OK



def test_deltanet_training_pair_validates_before_launch():
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    dn = lambda **kw: prob(**dict(dict(gate=_lib.GLA_GATE_NONE, Dk=64, Dv=64), **kw))
    saved_bytes = lambda p: _lib.lib.gla_deltanet_saved_bytes(ctypes.byref(p))
    # the chunk start states: B*H x ceil(L/64) x Dk x Dv, bf16 for bf16 I/O and fp32 for fp32 I/O
    BH, nc = 6, 5
    assert saved_bytes(dn(io=_lib.GLA_BF16)) == BH * nc * 64 * 64 * 2
    assert saved_bytes(dn(io=_lib.GLA_F32, Dk=128, Dv=192)) == BH * nc * 128 * 192 * 4
    assert saved_bytes(dn(L=0)) == 0
    assert saved_bytes(dn(Dk=256)) == 0 and saved_bytes(dn(gate=_lib.GLA_GATE_PER_KEY)) == 0

    def fwd(p, **kw):
        a = dict(q=16, k=16, v=16, beta=16, h0=None, o=16, hT=None, saved=16)
        a.update(kw)
        return _lib.lib.gla_deltanet_fwd_save(ctypes.byref(p), *(vp(a[n]) for n in ("q", "k", "v", "beta", "h0", "o",
                                                                                   "hT", "saved")), None)
    assert fwd(dn(), saved=24) == _lib.GLA_ERR_INVALID_ARG                   # misaligned
    assert fwd(dn(Dv=96)) == _lib.GLA_ERR_UNSUPPORTED
    assert fwd(dn(), o=None) == _lib.GLA_ERR_INVALID_ARG
    assert fwd(dn(B=0)) == _lib.GLA_OK

    names = ("q", "k", "v", "beta", "h0", "dO", "dhT", "saved", "dq", "dk", "dv", "dbeta", "dh0", "ws")

    def bwd(p, **kw):
        a = dict(q=16, k=16, v=16, beta=16, h0=None, dO=16, dhT=None, saved=16, dq=16, dk=16, dv=16, dbeta=16,
                 dh0=None, ws=16, nbytes=1 << 40)
        a.update(kw)
        return _lib.lib.gla_deltanet_bwd_saved(ctypes.byref(p), *(vp(a[n]) for n in names), a["nbytes"], None)
    need = _lib.lib.gla_deltanet_bwd_workspace_bytes(ctypes.byref(dn()))
    assert bwd(dn(), saved=40) == _lib.GLA_ERR_INVALID_ARG                   # misaligned
    assert bwd(dn(), nbytes=need - 1) == _lib.GLA_ERR_WORKSPACE              # the same workspace as without
    assert bwd(dn(gate=_lib.GLA_GATE_PER_HEAD)) == _lib.GLA_ERR_INVALID_ARG
    assert bwd(dn(), dv=None) == _lib.GLA_ERR_INVALID_ARG
    assert bwd(dn(H=0)) == _lib.GLA_OK


def test_mlstm_validates_before_launch():
    vp = lambda x: None if x is None else ctypes.c_void_p(x)
    ml = lambda **kw: prob(**dict(dict(gate=_lib.GLA_GATE_PER_HEAD, Dk=128, Dv=128, plan=_lib.GLA_PLAN_TC), **kw))
    wsb = lambda p, bwd: _lib.lib.gla_mlstm_workspace_bytes(ctypes.byref(p), bwd)
    saved_bytes = lambda p: _lib.lib.gla_mlstm_saved_bytes(ctypes.byref(p))
    assert wsb(ml(gate=_lib.GLA_GATE_PER_KEY), 0) == 0                  # per-head forget gate only
    assert wsb(ml(io=9), 1) == 0
    assert wsb(ml(), 1) >= wsb(ml(), 0) > 0
    # the forward's results: gate terms, num, den and the normaliser's segment states, plus the
    # value pass's saved states (tensor-core plan)
    BH, L = 6, 300
    assert saved_bytes(ml()) >= BH * L * 128 * 2 + 2 * BH * L * 4
    assert saved_bytes(ml(plan=_lib.GLA_PLAN_SIMT)) >= BH * L * 128 * 4   # fp32 numerator
    assert saved_bytes(ml(L=0)) == 0 and saved_bytes(ml(gate=_lib.GLA_GATE_NONE)) == 0

    def fwd(p, **kw):
        a = dict(q=16, k=16, v=16, g=16, itil=16, h=16, saved=16, ws=16, nbytes=1 << 40)
        a.update(kw)
        return _lib.lib.gla_mlstm_fwd_save(ctypes.byref(p), *(vp(a[n]) for n in ("q", "k", "v", "g", "itil", "h",
                                                                                "saved", "ws")), a["nbytes"], None)
    assert fwd(ml(), saved=24) == _lib.GLA_ERR_INVALID_ARG                   # misaligned
    assert fwd(ml(), ws=None) == _lib.GLA_ERR_INVALID_ARG
    assert fwd(ml(), nbytes=wsb(ml(), 0) - 1) == _lib.GLA_ERR_WORKSPACE
    assert fwd(ml(), itil=None) == _lib.GLA_ERR_INVALID_ARG

    names = ("q", "k", "v", "g", "itil", "dh", "saved", "dq", "dk", "dv", "dg", "ditil", "ws")

    def bwd(p, **kw):
        a = dict(q=16, k=16, v=16, g=16, itil=16, dh=16, saved=16, dq=16, dk=16, dv=16, dg=16, ditil=16, ws=16,
                 nbytes=1 << 40)
        a.update(kw)
        return _lib.lib.gla_mlstm_bwd_saved(ctypes.byref(p), *(vp(a[n]) for n in names), a["nbytes"], None)
    assert bwd(ml(), saved=40) == _lib.GLA_ERR_INVALID_ARG                   # misaligned
    assert bwd(ml(), nbytes=wsb(ml(), 1) - 1) == _lib.GLA_ERR_WORKSPACE
    assert bwd(ml(), ditil=None) == _lib.GLA_ERR_INVALID_ARG
    assert bwd(ml(gate=_lib.GLA_GATE_NONE)) == _lib.GLA_ERR_INVALID_ARG

def test_debug_wait_timeout_validates_before_launch():
    assert _lib.lib.gla_debug_wait_timeout(None, 100, None) == _lib.GLA_ERR_INVALID_ARG
    assert _lib.lib.gla_debug_wait_timeout(ctypes.c_void_p(24), 100, None) == _lib.GLA_ERR_INVALID_ARG  # misaligned
    assert _lib.lib.gla_debug_wait_timeout(ctypes.c_void_p(16), 0, None) == _lib.GLA_ERR_INVALID_ARG
    assert _lib.lib.gla_debug_wait_timeout(ctypes.c_void_p(16), (1 << 20) + 1, None) == _lib.GLA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError, match="no CPU fallback"):
        _lib._load()
    importlib.reload(_lib)
