"""The failure path of the kernels' bounded waits, exercised without any GPU
fault: a test hook makes the record-staging warp skip one work item, so the
compute warps wait for records that never arrive.  With their wait limit set
to a fraction of a millisecond they give up, the kernel writes
RSSM_ERR_TIMEOUT (7) to the status word, stops and returns (its own bulk
copies land first).  The batch is one work item, so nothing of the state was
touched, and the next launch on the same state, with the hooks cleared, must
decode exactly like the oracle."""
import numpy as np
import pytest
import torch

import oracle
from ssm_state_storage_b200 import replayssm as rs
from ssm_state_storage_b200 import workloads as wl
from tests import _gpu
from tests._util import per_step_rel_err, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-4
WAIT_NS = 200_000  # 0.2 ms


def _withheld_launch(fn):
    rs.replayssm_set_test_hooks(WAIT_NS, 0)
    try:
        fn()
        torch.cuda.synchronize()  # the kernel returned
    finally:
        rs.replayssm_set_test_hooks()


def test_m2_decode_wait_runs_out_then_recovers():
    w = wl.make("m2_serving", B=1, H=8, G=1)  # one (sequence, group) work item
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(20)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(st)
    Ad, Dd = A.cuda(), D.cuda()
    y = torch.zeros(w.B, w.H, w.P, device="cuda")
    inp = lambda t: dict(x=dev["x"][t], dt=dev["dt"][t], Bm=dev["Bm"][t], Cm=dev["Cm"][t],
                         A=Ad, D=Dd)
    _withheld_launch(lambda: rs.replayssm_decode_step(layer, state, inp(0), y))
    assert state.status() == 7
    assert int(state.len.abs().sum()) == 0 and torch.equal(state.h0.cpu(), S0)
    state.clear_status()
    yg = torch.empty(20, w.B, w.H, w.P, device="cuda")
    for t in range(20):
        rs.replayssm_decode_step(layer, state, inp(t), yg[t])
    torch.cuda.synchronize()
    assert state.status() == 0
    orc = oracle.M2Replay(S0, G=w.G, L=w.L)
    yo, lt, _ = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert np.array_equal(state.len.cpu().numpy(), orc.len)
    assert per_step_rel_err(yg.cpu().numpy(), yo) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL


def test_gdn_decode_wait_runs_out_then_recovers():
    w = wl.make("gdn_serving", B=1, H=1)  # one (sequence, head) work item
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(20)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(st)
    o = torch.zeros(w.B, w.H, w.P, device="cuda")
    inp = lambda t: {k: dev[k][t] for k in ("q", "k", "v", "alpha", "beta")}
    _withheld_launch(lambda: rs.replayssm_decode_step(layer, state, inp(0), o))
    assert state.status() == 7
    assert int(state.len.abs().sum()) == 0 and torch.equal(state.h0.cpu(), S0)
    state.clear_status()
    og = torch.empty(20, w.B, w.H, w.P, device="cuda")
    for t in range(20):
        rs.replayssm_decode_step(layer, state, inp(t), og[t])
    torch.cuda.synchronize()
    assert state.status() == 0
    orc = oracle.GDNReplay(S0, L=w.L)
    oo, _, _ = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert np.array_equal(state.len.cpu().numpy(), orc.len)
    assert per_step_rel_err(og.cpu().numpy(), oo) < TOL


def test_kda_decode_wait_runs_out_then_recovers():
    w = wl.make("kda_serving", B=1, H=1)  # one (sequence, head) work item
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(20)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(st)
    o = torch.zeros(w.B, w.H, w.P, device="cuda")
    inp = lambda t: {k: dev[k][t] for k in ("q", "k", "v", "alpha", "beta")}
    _withheld_launch(lambda: rs.replayssm_decode_step(layer, state, inp(0), o))
    assert state.status() == 7
    assert int(state.len.abs().sum()) == 0 and torch.equal(state.h0.cpu(), S0)
    state.clear_status()
    og = torch.empty(20, w.B, w.H, w.P, device="cuda")
    for t in range(20):
        rs.replayssm_decode_step(layer, state, inp(t), og[t])
    torch.cuda.synchronize()
    assert state.status() == 0
    orc = oracle.KDAReplay(S0, L=w.L)
    oo, _, _ = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert np.array_equal(state.len.cpu().numpy(), orc.len)
    assert per_step_rel_err(og.cpu().numpy(), oo) < TOL


def test_m2_verify_wait_runs_out_then_recovers():
    w = wl.make("m2_verify", B=1, H=8, G=1)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    rd = g.rounds(3)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    Ad, Dd = A.cuda(), D.cuda()
    drafts = lambda r: dict(x=dev["x"][r], dt=dev["dt"][r], Bm=dev["Bm"][r], Cm=dev["Cm"][r],
                            A=Ad, D=Dd)
    y = torch.zeros(w.B, w.n_draft, w.H, w.P, device="cuda")
    _withheld_launch(lambda: rs.replayssm_verify_commit(layer, state, None, drafts(0), y))
    assert state.status() == 7
    assert int(state.len.abs().sum()) == 0 and torch.equal(state.h0.cpu(), S0)
    state.clear_status()
    yg = torch.empty(3, w.B, w.n_draft, w.H, w.P, device="cuda")
    for r in range(3):
        rs.replayssm_verify_commit(layer, state, dev["acc"][r - 1] if r else None, drafts(r), yg[r])
    rs.replayssm_commit(layer, state, dev["acc"][2].contiguous(), Ad)
    torch.cuda.synchronize()
    assert state.status() == 0
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, cap=w.L + w.n_draft - 1)
    yo, lt = orc.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, rd["acc"])
    assert np.array_equal(state.len.cpu().numpy(), orc.len)
    yg = yg.cpu().numpy()
    assert per_step_rel_err(yg.reshape(-1, *yg.shape[3:]), yo.reshape(-1, *yo.shape[3:])) < TOL


def test_gdn_verify_wait_runs_out_then_recovers():
    w = wl.make("gdn_verify", B=1, H=1)  # one (sequence, head) work item
    g = wl.Generator(w)
    S0 = g.initial_state()
    rd = g.rounds(3)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    drafts = lambda r: {k: dev[k][r] for k in ("q", "k", "v", "alpha", "beta")}
    y = torch.zeros(w.B, w.n_draft, w.H, w.P, device="cuda")
    _withheld_launch(lambda: rs.replayssm_verify_commit(layer, state, None, drafts(0), y))
    assert state.status() == 7
    assert int(state.len.abs().sum()) == 0 and torch.equal(state.h0.cpu(), S0)
    state.clear_status()
    yg = torch.empty(3, w.B, w.n_draft, w.H, w.P, device="cuda")
    for r in range(3):
        rs.replayssm_verify_commit(layer, state, dev["acc"][r - 1] if r else None, drafts(r), yg[r])
    rs.replayssm_commit(layer, state, dev["acc"][2].contiguous())
    torch.cuda.synchronize()
    assert state.status() == 0
    orc = oracle.GDNReplay(S0, L=w.L, cap=w.L + w.n_draft - 1)
    yo, lt = orc.verify(rd["q"], rd["k"], rd["v"], rd["alpha"], rd["beta"], rd["acc"])
    assert np.array_equal(state.len.cpu().numpy(), orc.len)
    yg = yg.cpu().numpy()
    assert per_step_rel_err(yg.reshape(-1, *yg.shape[3:]), yo.reshape(-1, *yo.shape[3:])) < TOL
