"""Closed-form special cases of the two recurrences, run through the CUDA path
and compared with the fp64 oracle on the same inputs:

  Mamba-2, dt = 0: every decay factor is exp(0) = 1 and every write weight is
      0, so the state never changes: the folds leave h0 bit-identical and
      y = h0 C + D x.
  Mamba-2, A = 0: no decay, the state is the pure sum h0 + sum_i dt_i x_i B_i^T.
  Gated DeltaNet, beta = 0 and alpha = 1: S <- 1 * (I - 0) S + 0, so the state
      never changes: h0 bit-identical after the folds, o = scale h0^T q.

(Standard Mamba-2 and gated-delta-rule recurrences; special cases listed with
the oracle's pins.)"""
import numpy as np
import pytest
import torch

import oracle
from ssm_state_storage_b200 import workloads as wl
from tests import _gpu
from tests._util import per_step_rel_err, rel_err

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _m2(T, **kw):
    w = wl.make("m2_serving", B=3, H=16, G=2, **kw)
    g = wl.Generator(w)
    A, D = g.params()
    return w, A, D, g.initial_state(), g.steps(T)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_m2_dt_zero_keeps_checkpoint_bit_identical(dtype):
    w, A, D, S0, st = _m2(36, in_dtype=dtype)
    st["dt"] = torch.zeros_like(st["dt"])
    got = _gpu.m2_replay_run(w, A, D, S0, st)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L)
    yo, lt, _ = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt)
    assert torch.equal(got["state"].h0.cpu(), S0)  # two folds, state unchanged
    assert per_step_rel_err(got["y"], yo) < TOL


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_m2_no_decay_is_pure_sum(dtype):
    w, A, D, S0, st = _m2(36, in_dtype=dtype)
    A = torch.zeros_like(A)
    got = _gpu.m2_replay_run(w, A, D, S0, st)
    orc = oracle.M2Replay(S0, G=w.G, L=w.L)
    yo, lt, _ = orc.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt)
    assert per_step_rel_err(got["y"], yo) < TOL
    assert rel_err(_gpu.f64(got["state"].h0), orc.h0) < TOL
    # the oracle's pure sum over the 32 folded steps, written out here
    hpg = w.H // w.G
    S = S0.double().clone()
    for t in range(32):
        for h in range(w.H):
            xb = st["x"][t][:, h].double()
            Bb = st["Bm"][t][:, h // hpg].double()
            S[:, h] += st["dt"][t][:, h].double()[:, None, None] * xb[:, :, None] * Bb[:, None, :]
    assert rel_err(_gpu.f64(got["state"].h0), S.numpy()) < TOL


def test_gdn_beta_zero_alpha_one_keeps_checkpoint_bit_identical():
    w = wl.make("gdn_serving", B=2, H=4)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(36)
    st["alpha"] = torch.ones_like(st["alpha"])
    st["beta"] = torch.zeros_like(st["beta"])
    got = _gpu.gdn_replay_run(w, S0, st)
    orc = oracle.GDNReplay(S0, L=w.L)
    o, lt, _ = orc.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert got["state"].status() == 0
    assert np.array_equal(got["len"], lt)
    assert torch.equal(got["state"].h0.cpu(), S0)
    assert per_step_rel_err(got["y"], o) < TOL
    # o = h0^T q exactly as the closed form says
    q = st["q"].double().numpy()
    ref = np.einsum("bhkv,tbhk->tbhv", S0.double().numpy(), q)
    assert per_step_rel_err(got["y"], ref) < TOL
