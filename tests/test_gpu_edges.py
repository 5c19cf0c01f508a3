"""Edge cases on the GPU against the fp64 oracle: degenerate windows (one
record, so every step flushes; five records), group sizes that are not a power
of two or exceed eight heads, fp32 Gated DeltaNet inputs and short GDN windows,
an empty batch, a forced flush and materialisation with a read copy, and
verify rounds with fewer drafts than the buffer's draft capacity."""
import numpy as np
import pytest
import torch

import oracle
from ssm_state_storage_b200 import replayssm as rs
from ssm_state_storage_b200 import workloads as wl
from tests import _gpu
from tests._util import per_step_rel_err, rel_err, worst_step_err

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _m2(T, **kw):
    w = wl.make("m2_serving", **kw)
    g = wl.Generator(w)
    A, D = g.params()
    return w, A, D, g.initial_state(), g.steps(T)


def _check_m2(w, A, D, S0, st, **fmt):
    got = _gpu.m2_replay_run(w, A, D, S0, st, layer=_gpu.layer_for(w, **fmt) if fmt else None)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, **fmt)
    y, lt, _ = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt)
    assert worst_step_err(got["y"], y) < TOL
    assert _gpu.m2_buffer_matches(got["state"], orc, w.H // w.G)
    assert rel_err(_gpu.f64(got["state"].h0), orc.h0) < TOL
    return got, orc


@pytest.mark.parametrize("L", [1, 5])
def test_m2_short_windows(L):
    """L = 1: every step appends its record and folds it at once."""
    _check_m2(*_m2(12, B=2, H=16, G=2, L=L))


@pytest.mark.parametrize("H,G", [(6, 2), (32, 2)])
def test_m2_group_sizes(H, G):
    """3 heads per group (one-head work items) and 16 (two chunks of 8)."""
    _check_m2(*_m2(20, B=2, H=H, G=G))


@pytest.mark.parametrize("L,dtype", [(1, torch.bfloat16), (5, torch.bfloat16), (16, torch.float32)])
def test_gdn_windows_and_fp32_inputs(L, dtype):
    w = wl.make("gdn_serving", B=2, H=4, L=L, in_dtype=dtype)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(20)
    got = _gpu.gdn_replay_run(w, S0, st)
    orc = oracle.GDNReplay(S0, L=L)
    o, lt, _ = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt)
    assert per_step_rel_err(got["y"], o) < TOL
    assert rel_err(_gpu.f64(got["state"].h0), orc.h0) < TOL


@pytest.mark.parametrize("L,dtype", [(1, torch.bfloat16), (2, torch.bfloat16), (16, torch.float32)])
def test_kda_windows_and_fp32_inputs(L, dtype):
    """Kimi Delta Attention with a one-record window (a fold every step), a
    two-record window, and fp32 inputs (two record buffers instead of four)."""
    w = wl.make("kda_serving", B=2, H=4, L=L, in_dtype=dtype)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(20)
    got = _gpu.gdn_replay_run(w, S0, st)
    orc = oracle.KDAReplay(S0, L=L)
    o, lt, _ = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt)
    assert per_step_rel_err(got["y"], o) < TOL
    assert rel_err(_gpu.f64(got["state"].h0), orc.h0) < TOL


def test_empty_batch_is_a_no_op():
    for kind in ("m2", "gdn"):
        w = wl.make("m2_serving" if kind == "m2" else "gdn_serving", B=0, H=16 if kind == "m2" else 4,
                    G=2 if kind == "m2" else 4)
        layer = _gpu.layer_for(w)
        state = rs.ReplayState(layer)
        rs.replayssm_init(layer, state, torch.empty(0, w.H, w.P, w.N, device="cuda"))
        y = torch.empty(0, w.H, w.P, device="cuda")
        if kind == "m2":
            e = lambda *s, dt=w.in_dtype: torch.empty(*s, dtype=dt, device="cuda")
            inp = dict(x=e(0, w.H, w.P), dt=e(0, w.H), Bm=e(0, w.G, w.N), Cm=e(0, w.G, w.N),
                       A=torch.zeros(w.H, device="cuda"), D=torch.zeros(w.H, device="cuda"))
        else:
            e = lambda *s, dt=w.in_dtype: torch.empty(*s, dtype=dt, device="cuda")
            inp = dict(q=e(0, w.H, w.N), k=e(0, w.H, w.N), v=e(0, w.H, w.P),
                       alpha=e(0, w.H, dt=torch.float32), beta=e(0, w.H, dt=torch.float32))
        rs.replayssm_decode_step(layer, state, inp, y)
        rs.replayssm_full_decode_step(layer, torch.empty(0, w.H, w.P, w.N, device="cuda"), inp, y)
        torch.cuda.synchronize()


def test_read_copy_forced_flush_and_materialize():
    """21 steps leave 5 records buffered; materialising reads the fp32
    checkpoint, a forced flush folds the records and re-encodes the copy."""
    w, A, D, S0, st = _m2(21, B=2, H=16, G=2)
    got, orc = _check_m2(w, A, D, S0, st, read_fmt="fp8")
    layer, state = got["layer"], got["state"]
    S_out = torch.empty_like(state.h0)
    rs.replayssm_materialize(layer, state, S_out, A.cuda())
    assert rel_err(_gpu.f64(S_out), orc.materialize(A)) < TOL
    rs.replayssm_flush(layer, state, A.cuda(), force=True)
    orc.flush(A, force=True)
    assert int(state.len.abs().sum()) == 0 and int(orc.len.sum()) == 0
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL
    c = torch.empty_like(state.rc)
    rs.replayssm_quantize("fp8", state.h0, c)
    assert torch.equal(c, state.rc)
    assert state.status() == 0


@pytest.mark.parametrize("dmax,nd", [(1, 1), (3, 2), (4, 3)])
def test_verify_fewer_drafts(dmax, nd):
    w = wl.make("m2_verify", B=3, H=16, G=2)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    rd = g.rounds(10)
    rd = {k: (v[:, :, :nd] if k != "acc" else v.clamp(max=nd)) for k, v in rd.items()}
    layer = _gpu.layer_for(w, draft_max=dmax)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    R = rd["x"].shape[0]
    y = torch.empty(R, w.B, nd, w.H, w.P, device="cuda")
    lens = []
    for r in range(R):
        drafts = dict(x=dev["x"][r], dt=dev["dt"][r], Bm=dev["Bm"][r], Cm=dev["Cm"][r],
                      A=A.cuda(), D=D.cuda())
        rs.replayssm_verify_commit(layer, state, dev["acc"][r - 1] if r else None, drafts, y[r])
        lens.append(state.len.clone())
    rs.replayssm_commit(layer, state, dev["acc"][R - 1].contiguous(), A.cuda())
    lens.append(state.len.clone())
    torch.cuda.synchronize()
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, cap=w.L + max(dmax - 1, 0))
    yo, lt = orc.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, rd["acc"])
    yg = y.cpu().numpy()
    assert state.status() == 0
    assert np.array_equal(torch.stack(lens).cpu().numpy()[1:], lt)
    assert per_step_rel_err(yg.reshape(-1, *yg.shape[3:]), yo.reshape(-1, *yo.shape[3:])) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL
