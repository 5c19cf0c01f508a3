"""Decode steps whose record the upstream producer writes straight into its
buffer slot (replayssm_decode_step_inplace): an emulated producer stores each
step's inputs at slot len[b][h], read from the device lengths; the step must
then give exactly what the ordinary step gives -- outputs, checkpoint,
lengths and buffers bit-identical -- and match the oracle.  Run from ragged
lengths (Mamba-2 after speculative rounds) so the producer's slots differ
between sequences."""
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


def _write_m2(state, x, dt, Bm, Cm, hpg):
    """The producer: record of step t into slot len[b][h] of every buffer."""
    B, H = state.len.shape
    ln = state.len.long()
    b = torch.arange(B, device="cuda")[:, None].expand(B, H)
    h = torch.arange(H, device="cuda")[None, :].expand(B, H)
    state.buf[0][b, h, ln] = x
    state.buf[1][b, h, ln] = dt.float()
    G = Bm.shape[1]
    gl = ln[:, ::hpg]  # a group's heads share the length
    bg = torch.arange(B, device="cuda")[:, None].expand(B, G)
    g = torch.arange(G, device="cuda")[None, :].expand(B, G)
    state.buf[2][bg, g, gl] = Bm
    state.buf[3][bg, g, gl] = Cm


def _write_gdn(state, q, k, v, alpha, beta):
    B, H = state.len.shape
    ln = state.len.long()
    b = torch.arange(B, device="cuda")[:, None].expand(B, H)
    h = torch.arange(H, device="cuda")[None, :].expand(B, H)
    for i, t in enumerate((q, k, v, alpha, beta)):
        state.buf[i][b, h, ln] = t


def _clone(state, layer):
    c = rs.ReplayState(layer)
    c.h0.copy_(state.h0)
    c.len.copy_(state.len)
    for a, b_ in zip(c.buf, state.buf):
        a.copy_(b_)
    return c


def test_m2_inplace_equals_ordinary_step_from_ragged_lengths():
    w = wl.make("m2_verify", B=8, H=16, G=2)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    rd = g.rounds(5)
    st = g.steps(30)
    layer = _gpu.layer_for(w)
    ref = rs.ReplayState(layer)
    rs.replayssm_init(layer, ref, S0.cuda())
    dev = _gpu.to_dev(rd)
    Ad, Dd = A.cuda(), D.cuda()
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device="cuda")
    for r in range(5):
        drafts = dict(x=dev["x"][r], dt=dev["dt"][r], Bm=dev["Bm"][r], Cm=dev["Cm"][r], A=Ad, D=Dd)
        rs.replayssm_verify_commit(layer, ref, dev["acc"][r - 1] if r else None, drafts, y)
    rs.replayssm_commit(layer, ref, dev["acc"][4].contiguous(), Ad)
    torch.cuda.synchronize()
    assert len(set(ref.len[:, 0].tolist())) >= 3  # ragged
    inp = _clone(ref, layer)
    sd = _gpu.to_dev(st)
    y1 = torch.empty(30, w.B, w.H, w.P, device="cuda")
    y2 = torch.empty_like(y1)
    for t in range(30):
        rs.replayssm_decode_step(layer, ref, dict(x=sd["x"][t], dt=sd["dt"][t], Bm=sd["Bm"][t],
                                                  Cm=sd["Cm"][t], A=Ad, D=Dd), y1[t])
        _write_m2(inp, sd["x"][t], sd["dt"][t], sd["Bm"][t], sd["Cm"][t], w.H // w.G)
        rs.replayssm_decode_step_inplace(layer, inp, y2[t], Ad, Dd)
    torch.cuda.synchronize()
    assert ref.status() == 0 and inp.status() == 0
    assert torch.equal(y1, y2)
    assert torch.equal(ref.h0, inp.h0) and torch.equal(ref.len, inp.len)
    n = ref.len.cpu().numpy()
    for i in range(4):
        a, b_ = _gpu.f64(ref.buf[i]), _gpu.f64(inp.buf[i])
        for bb in range(w.B):
            for hh in range(a.shape[1]):
                k = n[bb, hh * (w.H // w.G) if i >= 2 else hh]
                assert np.array_equal(a[bb, hh, :k], b_[bb, hh, :k]), (i, bb, hh)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, cap=w.L + w.n_draft - 1)
    orc.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, rd["acc"])
    yo, lt, _ = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert per_step_rel_err(y2.cpu().numpy(), yo) < TOL
    assert rel_err(_gpu.f64(inp.h0), orc.h0) < TOL


@pytest.mark.parametrize("kind", ["gdn", "kda"])
def test_delta_rule_inplace_equals_ordinary_step(kind):
    w = wl.make("gdn_serving" if kind == "gdn" else "kda_serving", B=3, H=4)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(36)
    layer = _gpu.layer_for(w)
    ref = rs.ReplayState(layer)
    rs.replayssm_init(layer, ref, S0.cuda())
    inp = rs.ReplayState(layer)
    rs.replayssm_init(layer, inp, S0.cuda())
    sd = _gpu.to_dev(st)
    names = ("q", "k", "v", "alpha", "beta")
    y1 = torch.empty(36, w.B, w.H, w.P, device="cuda")
    y2 = torch.empty_like(y1)
    for t in range(36):
        rs.replayssm_decode_step(layer, ref, {k: sd[k][t] for k in names}, y1[t])
        _write_gdn(inp, *(sd[k][t] for k in names))
        rs.replayssm_decode_step_inplace(layer, inp, y2[t])
    torch.cuda.synchronize()
    assert ref.status() == 0 and inp.status() == 0
    assert torch.equal(y1, y2)
    assert torch.equal(ref.h0, inp.h0) and torch.equal(ref.len, inp.len)
    if kind == "gdn":
        orc = oracle.GDNReplay(S0, L=w.L)
    else:
        orc = oracle.KDAReplay(S0, L=w.L)
    o, _, _ = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert per_step_rel_err(y2.cpu().numpy(), o) < TOL
