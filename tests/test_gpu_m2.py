"""Mamba-2 parity on the GPU: the CUDA path (through the C ABI) against the
fp64 CPU oracle on the same seeded inputs.

Bars: buffer lengths, flush schedule and buffered slots bit-exact; outputs and
checkpoints within max relative error 1e-4 (element error over
max(|ref|, 1e-2 rms(ref)), per step)."""
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


def _draw(name, T, seqs=None, **kw):
    w = wl.make(name, **kw)
    g = wl.Generator(w, seqs)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(T)
    if seqs is not None:
        w = w.with_(B=len(seqs))
    return w, A, D, S0, st


def _oracle_replay(w, A, D, S0, st, **kw):
    orc = oracle.M2Replay(S0, G=w.G, L=w.L, **kw)
    y, lt, ft = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    return orc, y, lt, ft


@pytest.mark.parametrize("name,T,kw", [
    ("m2_tiny", 64, {}),                       # 4 flushes, fp32 inputs
    ("m2_serving", 40, {"B": 3}),              # bf16, 16 groups, ragged batch
    ("m2_serving", 24, {"B": 2, "P": 128, "N": 64, "H": 16, "G": 4}),
    ("m2_serving", 36, {"B": 2, "P": 128, "H": 16, "G": 2}),  # 128 x 128 tiles, 2 folds
])
def test_m2_replay_decode_matches_oracle(name, T, kw):
    w, A, D, S0, st = _draw(name, T, **kw)
    got = _gpu.m2_replay_run(w, A, D, S0, st, check_h0_untouched=True)
    orc, y, lt, ft = _oracle_replay(w, A, D, S0, st)
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt), "buffer length trace differs"
    assert got["untouched"], "a non-flush step wrote the checkpoint"
    assert worst_step_err(got["y"], y) < TOL
    assert _gpu.m2_buffer_matches(got["state"], orc, w.H // w.G)
    if T >= w.L:
        assert rel_err(got["state"].h0.cpu().double().numpy(), orc.h0) < TOL


def test_m2_conventional_step_matches_oracle():
    for name, T, kw in [("m2_tiny", 64, {}), ("m2_serving", 20, {"B": 2})]:
        w, A, D, S0, st = _draw(name, T, **kw)
        y_gpu, S_gpu = _gpu.m2_full_run(w, A, D, S0, st)
        y, S, _, _ = oracle.m2_conventional(S0, st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
        assert per_step_rel_err(y_gpu, y) < TOL
        assert rel_err(S_gpu, S) < TOL


def test_m2_materialize_and_forced_flush():
    """20 steps leave 4 records buffered: materialising gives the conventional
    state; a forced flush folds them into h0 and decoding continues."""
    w, A, D, S0, st = _draw("m2_serving", 40, B=2)
    first = {k: v[:20] for k, v in st.items()}
    rest = {k: v[20:] for k, v in st.items()}
    got = _gpu.m2_replay_run(w, A, D, S0, first)
    layer, state = got["layer"], got["state"]
    _, S20, _, _ = oracle.m2_conventional(S0, first["x"], first["dt"], first["Bm"], first["Cm"],
                                          A, D)
    S_out = torch.empty_like(state.h0)
    rs.replayssm_materialize(layer, state, S_out, A.cuda())
    assert rel_err(_gpu.f64(S_out), S20) < TOL
    assert torch.equal(state.len, torch.full_like(state.len, 4))
    rs.replayssm_flush(layer, state, A.cuda(), force=False)  # nothing is full: no-op
    assert torch.equal(state.len, torch.full_like(state.len, 4))
    rs.replayssm_flush(layer, state, A.cuda(), force=True)
    assert int(state.len.abs().sum()) == 0
    assert rel_err(_gpu.f64(state.h0), S20) < TOL
    # continue decoding from the flushed state
    dev = _gpu.to_dev(rest)
    y = torch.empty(20, w.B, w.H, w.P, device="cuda")
    for t in range(20):
        inp = dict(x=dev["x"][t], dt=dev["dt"][t], Bm=dev["Bm"][t], Cm=dev["Cm"][t], A=A.cuda(),
                   D=D.cuda())
        rs.replayssm_decode_step(layer, state, inp, y[t])
    yc, _, _, _ = oracle.m2_conventional(S0, st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert per_step_rel_err(y.cpu().numpy(), yc[20:]) < TOL
    assert state.status() == 0


def test_m2_full_batch_sampled():
    """m2_serving at its full batch of 256 (the benchmark's launch shape) over
    40 steps (two flushes); the oracle checks 3 sequences, all 128 heads."""
    T = 40
    w = wl.make("m2_serving")
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(T)
    got = _gpu.m2_replay_run(w, A, D, S0, st)
    seqs = [0, 101, 255]
    sub = {k: v[:, seqs] for k, v in st.items()}
    ws = w.with_(B=len(seqs))
    orc, y, lt, _ = _oracle_replay(ws, A, D, S0[seqs], sub)
    assert per_step_rel_err(got["y"][:, seqs], y) < TOL
    assert np.array_equal(got["len"][:, seqs], lt)
    assert np.all(got["len"] == got["len"][:, :1, :1])
    assert rel_err(got["state"].h0[seqs].cpu().double().numpy(), orc.h0) < TOL
    assert got["state"].status() == 0


def test_m2_bad_buffer_length_sets_status():
    """A corrupted length is caught on the device: the status word reports
    RSSM_ERR_STATE and the affected work items are left untouched."""
    w, A, D, S0, st = _draw("m2_serving", 1, B=2)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    state.len[1, :] = 16          # full buffer on entry: invalid for a decode step
    state.len[0, 3] = 5           # heads of group 0 out of step
    h0_before = state.h0.clone()
    dev = _gpu.to_dev(st)
    y = torch.zeros(w.B, w.H, w.P, device="cuda")
    rs.replayssm_decode_step(layer, state, dict(x=dev["x"][0], dt=dev["dt"][0], Bm=dev["Bm"][0],
                                                Cm=dev["Cm"][0], A=A.cuda(), D=D.cuda()), y)
    assert state.status() == 9
    assert torch.equal(state.len[1], torch.full_like(state.len[1], 16))
    assert torch.equal(state.h0, h0_before)
    assert torch.all(y[1] == 0)
    # the decode work item holding head 3 (heads 0-3) is skipped; the others ran
    assert torch.all(y[0, :4] == 0)
    assert torch.all(state.len[0, :3] == 0) and int(state.len[0, 3]) == 5
    assert torch.all((y[0, 8:] != 0).any(dim=-1))


def test_m2_host_checks():
    w, A, D, S0, st = _draw("m2_tiny", 1, B=1)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    raw = torch.empty(state.h0.numel() + 4, device="cuda")
    state.h0 = raw[1:1 + state.h0.numel()].view_as(state.h0)  # 4-byte offset: misaligned
    with pytest.raises(rs.ReplayError, match="aligned"):
        rs.replayssm_init(layer, state, S0.cuda())
