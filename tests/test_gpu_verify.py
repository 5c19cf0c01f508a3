"""Speculative verify / commit parity on the GPU against the CPU oracle."""
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
    w = wl.make("m2_verify", **kw)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    rd = g.rounds(R)
    return w, A, D, S0, rd


def _gpu_rounds(w, A, D, S0, rd, acc=None):
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    acc = dev["acc"] if acc is None else acc.cuda()
    R = rd["x"].shape[0]
    y = torch.empty(R, w.B, w.n_draft, w.H, w.P, device="cuda")
    lens = []
    Ad, Dd = A.cuda(), D.cuda()
    for r in range(R):
        drafts = dict(x=dev["x"][r], dt=dev["dt"][r], Bm=dev["Bm"][r], Cm=dev["Cm"][r], A=Ad, D=Dd)
        rs.replayssm_verify_commit(layer, state, acc[r - 1] if r else None, drafts, y[r])
        lens.append(state.len.clone())
    rs.replayssm_commit(layer, state, acc[R - 1].contiguous(), Ad)
    lens.append(state.len.clone())
    torch.cuda.synchronize()
    return layer, state, y.cpu().numpy(), torch.stack(lens).cpu().numpy()


def test_verify_rounds_match_oracle():
    w, A, D, S0, rd = _draw(24, B=3, H=32, G=4)
    layer, state, y, lens = _gpu_rounds(w, A, D, S0, rd)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, cap=w.L + w.n_draft - 1)
    yo, lt = orc.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, rd["acc"])
    assert state.status() == 0
    # committed lengths: GPU length after call r+1 == oracle length after round r
    assert np.array_equal(lens[1:], lt)
    assert per_step_rel_err(y.reshape(-1, *y.shape[3:]), yo.reshape(-1, *yo.shape[3:])) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL
    assert _gpu.m2_buffer_matches(state, orc, w.H // w.G)
    # against snapshot-and-restore decoding of the full state
    ys, Ss, _ = oracle.m2_verify_snapshot(S0, rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D,
                                          rd["acc"])
    S_out = torch.empty_like(state.h0)
    rs.replayssm_materialize(layer, state, S_out, A.cuda())
    assert rel_err(_gpu.f64(S_out), Ss) < TOL


@pytest.mark.parametrize("P,N,dtype,H,G", [
    (128, 128, torch.float32, 16, 2),   # 8 heads per group do not fit one CTA: head chunks
    (64, 64, torch.float32, 12, 2),     # 6 heads per group
    (128, 64, torch.bfloat16, 8, 8),    # one head per group
    (64, 128, torch.bfloat16, 6, 2),    # 3 heads per group
    (128, 128, torch.bfloat16, 8, 2),   # 128 x 128 tiles, tensor-core commit fold
])
def test_verify_shapes_match_oracle(P, N, dtype, H, G):
    w, A, D, S0, rd = _draw(20, B=3, H=H, G=G, P=P, N=N, in_dtype=dtype)
    layer, state, y, lens = _gpu_rounds(w, A, D, S0, rd)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, cap=w.L + w.n_draft - 1)
    yo, lt = orc.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, rd["acc"])
    assert state.status() == 0
    assert np.array_equal(lens[1:], lt)
    assert per_step_rel_err(y.reshape(-1, *y.shape[3:]), yo.reshape(-1, *yo.shape[3:])) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL
    assert _gpu.m2_buffer_matches(state, orc, w.H // w.G)


def test_verify_full_batch_sampled():
    """m2_verify at its full batch of 512 (the benchmark's launch shape: many
    items per CTA, both consumer groups busy) over 12 rounds; the oracle checks
    4 sequences, all 128 heads."""
    w, A, D, S0, rd = _draw(12)
    layer, state, y, lens = _gpu_rounds(w, A, D, S0, rd)
    assert state.status() == 0
    seqs = [0, 203, 257, 511]
    orc = oracle.M2Replay(S0[seqs], G=w.G, L=w.L, cap=w.L + w.n_draft - 1)
    sub = {k: v[:, seqs] for k, v in rd.items()}
    yo, lt = orc.verify(sub["x"], sub["dt"], sub["Bm"], sub["Cm"], A, D, sub["acc"])
    ys = y[:, seqs]
    assert np.array_equal(lens[1:][:, seqs], lt)
    assert per_step_rel_err(ys.reshape(-1, *ys.shape[3:]), yo.reshape(-1, *yo.shape[3:])) < TOL
    assert rel_err(_gpu.f64(state.h0[seqs]), orc.h0) < TOL


def test_verify_rejects_misaligned_draft_rows():
    w, A, D, S0, rd = _draw(1, B=2, H=16, G=2)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    x = dev["x"][0]
    raw = torch.empty(x.numel() + 1, dtype=x.dtype, device="cuda")
    xm = raw[1:].view(x.shape)  # starts 2 bytes past an aligned address
    xm.copy_(x)
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device="cuda")
    drafts = dict(x=xm, dt=dev["dt"][0], Bm=dev["Bm"][0], Cm=dev["Cm"][0], A=A.cuda(),
                  D=D.cuda())
    with pytest.raises(rs.ReplayError, match="aligned"):
        rs.replayssm_verify_commit(layer, state, None, drafts, y)
    assert state.status() == 0 and int(state.len.sum()) == 0


def test_verify_accept_none_keeps_checkpoint_bit_exact():
    w, A, D, S0, rd = _draw(6, B=2, H=16, G=2)
    acc0 = torch.zeros_like(rd["acc"])
    layer, state, y, lens = _gpu_rounds(w, A, D, S0, rd, acc=acc0)
    assert torch.equal(state.h0.cpu(), S0)
    assert np.all(lens == 0)


def test_snapshot_restore_on_gpu_matches_oracle():
    """The conventional comparison: snapshot the full state, step through the
    drafts with the full-state kernel, restore, replay the accepted ones."""
    w, A, D, S0, rd = _draw(8, B=3, H=16, G=2)
    layer = _gpu.layer_for(w, draft_max=0)
    S = S0.clone().cuda()
    snap = torch.empty_like(S)
    dev = _gpu.to_dev(rd)
    R = rd["x"].shape[0]
    y = torch.empty(R, w.B, w.n_draft, w.H, w.P, device="cuda")
    Ad, Dd = A.cuda(), D.cuda()
    for r in range(R):
        snap.copy_(S)
        for d in range(w.n_draft):
            inp = dict(x=dev["x"][r][:, d], dt=dev["dt"][r][:, d], Bm=dev["Bm"][r][:, d],
                       Cm=dev["Cm"][r][:, d], A=Ad, D=Dd)
            rs.replayssm_full_decode_step(layer, S, inp, y[r][:, d])
        S.copy_(snap)
        for d in range(w.n_draft):
            inp = dict(x=dev["x"][r][:, d], dt=dev["dt"][r][:, d], Bm=dev["Bm"][r][:, d],
                       Cm=dev["Cm"][r][:, d], A=Ad, D=Dd)
            junk = torch.empty(w.B, w.H, w.P, device="cuda")
            rs.replayssm_full_decode_step(layer, S, inp, junk, limit=dev["acc"][r], step_index=d)
    torch.cuda.synchronize()
    ys, Ss, _ = oracle.m2_verify_snapshot(S0, rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D,
                                          rd["acc"])
    yg = y.cpu().numpy()
    assert per_step_rel_err(yg.reshape(-1, *yg.shape[3:]), ys.reshape(-1, *ys.shape[3:])) < TOL
    assert rel_err(_gpu.f64(S), Ss) < TOL


def test_verify_bad_acceptance_sets_status():
    w, A, D, S0, rd = _draw(2, B=2, H=16, G=2)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    dev = _gpu.to_dev(rd)
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device="cuda")
    drafts = dict(x=dev["x"][0], dt=dev["dt"][0], Bm=dev["Bm"][0], Cm=dev["Cm"][0], A=A.cuda(),
                  D=D.cuda())
    rs.replayssm_verify_commit(layer, state, None, drafts, y)
    bad = torch.tensor([5, 1], dtype=torch.int32, device="cuda")  # 5 > draft_max
    rs.replayssm_verify_commit(layer, state, bad, drafts, y)
    assert state.status() == 9
    assert int(state.len[0, 0]) == 0 and int(state.len[1, 0]) == 1
    with pytest.raises(rs.ReplayError, match="capacity"):
        big = {k: (v.repeat_interleave(2, dim=1) if v.dim() > 1 else v) for k, v in drafts.items()}
        rs.replayssm_verify_commit(layer, state, None, big, torch.empty(w.B, 8, w.H, w.P,
                                                                         device="cuda"))


def test_decode_after_verify_rounds_with_ragged_lengths():
    """Speculative rounds leave sequences at different buffer lengths, so in
    the decode steps that follow different sequences flush on different steps
    of one launch.  6 verify rounds at batch 16, the last acceptance
    committed, then 40 decode steps; lengths and buffered records bit-exact,
    outputs and checkpoints within the fp32 tolerance."""
    w, A, D, S0, rd = _draw(6, B=16, H=16, G=2)
    layer, state, y, lens = _gpu_rounds(w, A, D, S0, rd)
    g = wl.Generator(w)
    g.initial_state()
    g.rounds(6)
    st = g.steps(40)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, cap=w.L + w.n_draft - 1)
    orc.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, rd["acc"])
    # the oracle's rounds commit each round's acceptance; close the last one
    assert np.array_equal(lens[-1], orc.len)
    start = orc.len[:, 0].copy()
    assert len(set(start.tolist())) >= 4, start  # genuinely ragged
    yo, lt, ft = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    dev = _gpu.to_dev(st)
    Ad, Dd = A.cuda(), D.cuda()
    yg = torch.empty(40, w.B, w.H, w.P, device="cuda")
    lg = torch.empty(40, w.B, w.H, dtype=torch.int32, device="cuda")
    for t in range(40):
        inp = dict(x=dev["x"][t], dt=dev["dt"][t], Bm=dev["Bm"][t], Cm=dev["Cm"][t], A=Ad, D=Dd)
        rs.replayssm_decode_step(layer, state, inp, yg[t])
        lg[t] = state.len
    torch.cuda.synchronize()
    assert state.status() == 0
    assert np.array_equal(lg.cpu().numpy(), lt)
    # flushes happen on different steps for different sequences
    first_flush = [int(np.argmax(ft[:, b, 0])) for b in range(w.B)]
    assert len(set(first_flush)) >= 4, first_flush
    assert per_step_rel_err(yg.cpu().numpy(), yo) < TOL
    assert rel_err(_gpu.f64(state.h0), orc.h0) < TOL
    assert _gpu.m2_buffer_matches(state, orc, w.H // w.G)
