"""Gated DeltaNet speculative verify / commit on the GPU against the fp64
oracle: drafts appended and evaluated output-only from h0 and the buffer, the
accepted prefix committed (with a fold when the buffer reaches the window),
compared with the oracle's replay rounds and with snapshot-and-restore decoding
of the full state [sitech §Reducing state traffic and simplifying rollback],
[hamidun §Where the state problem appears]."""
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


def _draw(R, **kw):
    w = wl.make("gdn_verify", **kw)
    g = wl.Generator(w)
    S0 = g.initial_state()
    return w, S0, g.rounds(R)


def _gpu_rounds(w, S0, rd, acc=None, commit_last=True):
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    acc = dev["acc"] if acc is None else acc.cuda()
    R = rd["q"].shape[0]
    y = torch.empty(R, w.B, w.n_draft, w.H, w.P, device="cuda")
    lens = []
    for r in range(R):
        drafts = {k: dev[k][r] for k in ("q", "k", "v", "alpha", "beta")}
        rs.replayssm_verify_commit(layer, state, acc[r - 1] if r else None, drafts, y[r])
        lens.append(state.len.clone())
    if commit_last:
        rs.replayssm_commit(layer, state, acc[R - 1].contiguous())
        lens.append(state.len.clone())
    torch.cuda.synchronize()
    return layer, state, y.cpu().numpy(), torch.stack(lens).cpu().numpy()


def _oracle(w, S0, rd):
    orc = oracle.GDNReplay(S0, L=w.L, cap=w.L + w.n_draft - 1)
    yo, lt = orc.verify(rd["q"], rd["k"], rd["v"], rd["alpha"], rd["beta"], rd["acc"])
    return orc, yo, lt


def _flat(y):
    return y.reshape(-1, *y.shape[3:])


@pytest.mark.parametrize("kw", [{"B": 3, "H": 4}, {"B": 2, "H": 2, "in_dtype": torch.float32}])
def test_gdn_verify_rounds_match_oracle(kw):
    w, S0, rd = _draw(24, **kw)
    layer, state, y, lens = _gpu_rounds(w, S0, rd)
    orc, yo, lt = _oracle(w, S0, rd)
    assert state.status() == 0
    assert np.array_equal(lens[1:], lt)           # committed lengths, bit-exact
    assert per_step_rel_err(_flat(y), _flat(yo)) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL
    n = state.len.cpu().numpy()
    for i, rec in enumerate((orc.rec_q, orc.rec_k, orc.rec_v, orc.rec_alpha, orc.rec_beta)):
        got = _gpu.f64(state.buf[i])
        for b in range(w.B):
            for h in range(w.H):
                assert np.array_equal(got[b, h, :n[b, h]], rec[b, h, :n[b, h]]), (i, b, h)
    # against snapshot-and-restore decoding of the full state
    ys, Ss, _ = oracle.gdn_verify_snapshot(S0, rd["q"], rd["k"], rd["v"], rd["alpha"],
                                           rd["beta"], rd["acc"])
    assert per_step_rel_err(_flat(y), _flat(ys)) < TOL
    S_out = torch.empty_like(state.h0)
    rs.replayssm_materialize(layer, state, S_out)
    assert rel_err(_gpu.f64(S_out), Ss) < TOL


def test_gdn_verify_full_batch_sampled():
    """gdn_verify at its full batch of 256 (the benchmark's launch) over 10
    rounds; the oracle checks 3 sequences, all 32 heads."""
    w, S0, rd = _draw(10)
    layer, state, y, lens = _gpu_rounds(w, S0, rd)
    assert state.status() == 0
    seqs = [0, 131, 255]
    orc = oracle.GDNReplay(S0[seqs], L=w.L, cap=w.L + w.n_draft - 1)
    sub = {k: v[:, seqs] for k, v in rd.items()}
    yo, lt = orc.verify(sub["q"], sub["k"], sub["v"], sub["alpha"], sub["beta"], sub["acc"])
    assert np.array_equal(lens[1:][:, seqs], lt)
    ys = y[:, seqs]
    assert per_step_rel_err(_flat(ys), _flat(yo)) < TOL
    assert rel_err(_gpu.f64(state.h0[seqs]), orc.h0) < TOL


def test_gdn_verify_accept_none_keeps_checkpoint_bit_exact():
    w, S0, rd = _draw(6, B=2, H=4)
    _, state, _, lens = _gpu_rounds(w, S0, rd, acc=torch.zeros_like(rd["acc"]))
    assert torch.equal(state.h0.cpu(), S0)
    assert np.all(lens == 0)


def test_gdn_verify_accept_all_equals_decoding():
    """Accepting every draft is plain decoding of the drafts in order."""
    w, S0, rd = _draw(5, B=2, H=4)
    acc = torch.full_like(rd["acc"], w.n_draft)
    layer, state, y, lens = _gpu_rounds(w, S0, rd, acc=acc)
    steps = {k: rd[k].transpose(1, 2).reshape(-1, *rd[k].shape[1:2], *rd[k].shape[3:])
             for k in ("q", "k", "v", "alpha", "beta")}
    oc, Sc, _, _ = oracle.gdn_conventional(S0, steps["q"], steps["k"], steps["v"],
                                           steps["alpha"], steps["beta"])
    yd = y.transpose(0, 2, 1, 3, 4).reshape(-1, w.B, w.H, w.P)
    assert per_step_rel_err(yd, oc) < TOL
    S_out = torch.empty_like(state.h0)
    rs.replayssm_materialize(layer, state, S_out)
    assert rel_err(_gpu.f64(S_out), Sc) < TOL


def test_gdn_decode_after_verify_rounds():
    """Decode steps after speculative rounds read the corrections the verify
    kernel cached for the accepted drafts."""
    w, S0, rd = _draw(5, B=4, H=4)
    layer, state, y, lens = _gpu_rounds(w, S0, rd)
    g = wl.Generator(w)
    g.initial_state()
    g.rounds(5)
    st = g.steps(24)
    orc, _, _ = _oracle(w, S0, rd)
    o, lt, _ = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    dev = _gpu.to_dev(st)
    og = torch.empty(24, w.B, w.H, w.P, device="cuda")
    for t in range(24):
        rs.replayssm_decode_step(layer, state, {k: dev[k][t] for k in dev}, og[t])
    torch.cuda.synchronize()
    assert state.status() == 0
    assert np.array_equal(state.len.cpu().numpy(), orc.len)
    assert per_step_rel_err(og.cpu().numpy(), o) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL


def test_gdn_verify_bad_acceptance_sets_status():
    w, S0, rd = _draw(2, B=2, H=2)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device="cuda")
    drafts = {k: dev[k][0] for k in ("q", "k", "v", "alpha", "beta")}
    rs.replayssm_verify_commit(layer, state, None, drafts, y)
    bad = torch.tensor([5, 1], dtype=torch.int32, device="cuda")  # 5 > draft_max
    rs.replayssm_verify_commit(layer, state, bad, drafts, y)
    assert state.status() == 9
    assert int(state.len[0, 0]) == 0 and int(state.len[1, 0]) == 1


@pytest.mark.parametrize("dmax,nd", [(1, 1), (3, 2), (4, 3)])
def test_gdn_verify_fewer_drafts(dmax, nd):
    """Rounds of 1-3 drafts, with draft_max (and so the buffer capacity) both
    equal to and above the round's count."""
    w, S0, rd = _draw(12, B=3, H=4)
    rd = {k: (v[:, :, :nd].contiguous() if k != "acc" else v.clamp(max=nd)) for k, v in rd.items()}
    layer = _gpu.layer_for(w, draft_max=dmax)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    R = rd["q"].shape[0]
    y = torch.empty(R, w.B, nd, w.H, w.P, device="cuda")
    lens = []
    for r in range(R):
        drafts = {k: dev[k][r] for k in ("q", "k", "v", "alpha", "beta")}
        rs.replayssm_verify_commit(layer, state, dev["acc"][r - 1] if r else None, drafts, y[r])
        lens.append(state.len.clone())
    rs.replayssm_commit(layer, state, dev["acc"][R - 1].contiguous())
    lens.append(state.len.clone())
    torch.cuda.synchronize()
    orc = oracle.GDNReplay(S0, L=w.L, cap=w.L + max(dmax - 1, 0))
    yo, lt = orc.verify(rd["q"], rd["k"], rd["v"], rd["alpha"], rd["beta"], rd["acc"])
    yg = y.cpu().numpy()
    assert state.status() == 0
    assert np.array_equal(torch.stack(lens).cpu().numpy()[1:], lt)
    assert per_step_rel_err(_flat(yg), _flat(yo)) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL
