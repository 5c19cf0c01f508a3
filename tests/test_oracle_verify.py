"""Pins for speculative verify / commit in the CPU oracle (no GPU)."""
import numpy as np

from ssm_state_storage_b200 import workloads as wl
from tests._util import per_step_rel_err, rel_err


def _setup(B=2, H=16, G=2, R=10):
    w = wl.make("m2_verify", B=B, H=H, G=G)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    rd = g.rounds(R)
    return w, A, D, S0, rd


def test_verify_matches_snapshot_restore(oracle_mod):
    """Output-only evaluation of drafts from checkpoint + buffer gives the same
    draft outputs and the same committed state as snapshot-and-restore decoding
    ([sitech §Reducing state traffic...]; [hamidun §Where the state problem appears])."""
    w, A, D, S0, rd = _setup(R=14)
    ys, Ss, copies = oracle_mod.m2_verify_snapshot(S0, rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A,
                                                   D, rd["acc"])
    cap = w.L + w.n_draft - 1
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L, cap=cap)
    yr, lt = rp.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, rd["acc"])
    assert per_step_rel_err(yr.reshape(-1, *yr.shape[3:]), ys.reshape(-1, *ys.shape[3:])) < 1e-12
    assert rel_err(rp.materialize(A), Ss) < 1e-12
    # committed lengths: running sum of acceptances, folded at >= 16
    acc = rd["acc"].numpy()
    n = np.zeros(w.B, np.int64)
    for r in range(acc.shape[0]):
        n = n + acc[r]
        n = np.where(n >= w.L, 0, n)
        assert np.all(lt[r] == n[:, None])
    assert np.all(copies == 2 * acc.shape[0])


def test_verify_accept_none_changes_nothing(oracle_mod):
    w, A, D, S0, rd = _setup(R=6)
    acc0 = np.zeros_like(rd["acc"].numpy())
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L, cap=w.L + w.n_draft - 1)
    h0 = rp.h0.copy()
    rp.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, acc0)
    np.testing.assert_array_equal(rp.h0, h0)
    assert np.all(rp.len == 0)


def test_verify_accept_all_equals_decode(oracle_mod):
    """Accepting all 4 drafts equals 4 plain decode steps: same outputs, same
    buffer length and the same records in the same slots (no window boundary
    is crossed in the 3 rounds, 12 < 16)."""
    w, A, D, S0, rd = _setup(R=3)
    acc4 = np.full_like(rd["acc"].numpy(), 4)
    cap = w.L + w.n_draft - 1
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L, cap=cap)
    yv, lt = rp.verify(rd["x"], rd["dt"], rd["Bm"], rd["Cm"], A, D, acc4)
    dec = oracle_mod.M2Replay(S0, G=w.G, L=w.L, cap=cap)
    # [R,B,Dn,...] -> [R*Dn,B,...]
    flat = lambda t: np.swapaxes(t.double().numpy(), 1, 2).reshape(-1, *t.shape[1:2], *t.shape[3:])
    yd, ld, _ = dec.decode(flat(rd["x"]), flat(rd["dt"]), flat(rd["Bm"]), flat(rd["Cm"]), A, D)
    assert per_step_rel_err(flat(_t(yv)), yd) < 1e-12
    np.testing.assert_array_equal(rp.len, dec.len)
    n = int(rp.len[0, 0])
    for a, b in ((rp.rec_x, dec.rec_x), (rp.rec_dt, dec.rec_dt), (rp.rec_B, dec.rec_B),
                 (rp.rec_C, dec.rec_C)):
        np.testing.assert_array_equal(a[:, :, :n], b[:, :, :n])
    np.testing.assert_array_equal(rp.h0, dec.h0)


def _t(a):
    import torch
    return torch.from_numpy(a)
