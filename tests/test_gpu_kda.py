"""Kimi Delta Attention (per-channel decay) parity on the GPU against the fp64
oracle: replay decode with the fused fold, the conventional step, forced
flush and materialisation, 64 folds, and the full batch."""
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


def _draw(T, seqs=None, **kw):
    w = wl.make("kda_serving", **kw)
    g = wl.Generator(w, seqs)
    S0 = g.initial_state()
    st = g.steps(T)
    if seqs is not None:
        w = w.with_(B=len(seqs))
    return w, S0, st


def _orc_decode(w, S0, st):
    orc = oracle.KDAReplay(S0, L=w.L)
    o, lt, ft = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    return orc, o, lt


@pytest.mark.parametrize("T,kw", [(40, {"B": 3, "H": 4}),
                                  (36, {"B": 2, "H": 2, "in_dtype": torch.float32}),
                                  (12, {"B": 2, "H": 2, "L": 5})])
def test_kda_replay_decode_matches_oracle(T, kw):
    w, S0, st = _draw(T, **kw)
    got = _gpu.gdn_replay_run(w, S0, st, check_h0_untouched=True)
    orc, o, lt = _orc_decode(w, S0, st)
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt)
    assert got["untouched"]
    assert per_step_rel_err(got["y"], o) < TOL
    assert rel_err(_gpu.f64(got["state"].h0), orc.h0) < TOL
    n = int(got["state"].len[0, 0])
    for i, rec in enumerate((orc.rec_q, orc.rec_k, orc.rec_v, orc.rec_alpha, orc.rec_beta)):
        assert np.array_equal(_gpu.f64(got["state"].buf[i])[:, :, :n], rec[:, :, :n]), i


def test_kda_conventional_step_matches_oracle():
    w, S0, st = _draw(20, B=2, H=4)
    o_gpu, S_gpu = _gpu.gdn_full_run(w, S0, st)
    o, S, _, _ = oracle.kda_conventional(S0, st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert per_step_rel_err(o_gpu, o) < TOL
    assert rel_err(S_gpu, S) < TOL


def test_kda_materialize_and_forced_flush():
    w, S0, st = _draw(21, B=2, H=4)
    got = _gpu.gdn_replay_run(w, S0, st)
    layer, state = got["layer"], got["state"]
    _, S21, _, _ = oracle.kda_conventional(S0, st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    S_out = torch.empty_like(state.h0)
    rs.replayssm_materialize(layer, state, S_out)
    assert rel_err(_gpu.f64(S_out), S21) < TOL
    assert int(state.len[0, 0]) == 5
    rs.replayssm_flush(layer, state, force=True)
    torch.cuda.synchronize()
    assert int(state.len.abs().sum()) == 0
    assert rel_err(_gpu.f64(state.h0), S21) < TOL


def test_kda_replay_over_64_folds():
    w, S0, st = _draw(1024, B=2, H=2)
    got = _gpu.gdn_replay_run(w, S0, st)
    oc, Sc, _, _ = oracle.kda_conventional(S0, st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    errs = [rel_err(a, b) for a, b in zip(got["y"], oc)]
    assert got["state"].status() == 0
    assert max(errs) < TOL, max(errs)
    assert rel_err(_gpu.f64(got["state"].h0), Sc) < TOL


def test_kda_full_batch_sampled():
    w, S0, st = _draw(20)
    got = _gpu.gdn_replay_run(w, S0, st)
    assert got["state"].status() == 0
    seqs = [0, 97, 255]
    ws, S0s, sts = _draw(20, seqs=seqs)
    orc, o, lt = _orc_decode(ws, S0s, sts)
    assert per_step_rel_err(got["y"][:, seqs], o) < TOL
    assert rel_err(_gpu.f64(got["state"].h0[seqs]), orc.h0) < TOL


def test_kda_bad_buffer_length_sets_status():
    """A corrupted length is caught on the device: RSSM_ERR_STATE in the status
    word, the affected items untouched, every other item decoded as usual.
    320 items on at most 148 CTAs: items of both consumer groups of CTA 0
    (items 0 and 148) are hit."""
    w, S0, st = _draw(1, B=10, H=32)
    layer = _gpu.layer_for(w)
    state = rs.ReplayState(layer)
    rs.replayssm_init(layer, state, S0.cuda())
    bad = [(0, 0), (148 // 32, 148 % 32), (7, 5)]
    for b, h in bad:
        state.len[b, h] = 16  # a full buffer on entry: invalid for a decode step
    h0_before = state.h0.clone()
    dev = _gpu.to_dev(st)
    o = torch.zeros(w.B, w.H, w.P, device="cuda")
    rs.replayssm_decode_step(layer, state, {k: dev[k][0] for k in ("q", "k", "v", "alpha", "beta")}, o)
    torch.cuda.synchronize()
    assert state.status() == 9
    assert torch.equal(state.h0, h0_before)  # a first step folds nothing
    _, oo, _ = _orc_decode(w, S0, {k: v[:1] for k, v in st.items()})
    got = o.cpu().numpy().astype(np.float64)
    good = np.ones((w.B, w.H), dtype=bool)
    for b, h in bad:
        good[b, h] = False
        assert int(state.len[b, h]) == 16
        assert np.all(got[b, h] == 0)
    assert np.all(state.len.cpu().numpy()[good] == 1)
    assert rel_err(got[good], oo[0][good]) < TOL
