"""Pins for the Mamba-2 half of the CPU oracle (no GPU).

Each test checks the oracle against something other than itself: hand-derived
values, closed forms of special cases, the replay = conventional identity the
pages state, the traffic counts and the flush schedule the pages state.
"""
import math

import numpy as np
import pytest

from ssm_state_storage_b200 import workloads as wl
from tests._util import per_step_rel_err, read_kv, rel_err


def _tiny_inputs():
    # One head, P=2 rows, N=3 state columns, two tokens.  dt*A = -ln 2 makes
    # every decay factor 1/2, so the expected values are exact dyadics.
    h0 = np.array([[1.0, 1.0, 1.0], [0.0, 0.0, 0.0]]).reshape(1, 1, 2, 3)
    x = np.array([[1.0, 2.0], [0.0, 1.0]]).reshape(2, 1, 1, 2)
    dt = np.array([1.0, 1.0]).reshape(2, 1, 1)
    Bm = np.array([[1.0, 0.0, -1.0], [2.0, 2.0, 2.0]]).reshape(2, 1, 1, 3)
    Cm = np.array([[1.0, 0.0, 0.0], [1.0, 1.0, 1.0]]).reshape(2, 1, 1, 3)
    A = np.array([-math.log(2.0)])
    D = np.array([0.5])
    return h0, x, dt, Bm, Cm, A, D


# Hand derivation (S <- dA S + dt x B^T, y = S C + D x, dA = 1/2):
#   S1 = h0/2 + [1,2]^T [1,0,-1] = [[1.5, .5, -.5], [2, 0, -2]]
#   y1 = S1 [1,0,0]^T + .5 [1,2] = [2, 3]
#   S2 = S1/2 + [0,1]^T [2,2,2]  = [[.75, .25, -.25], [3, 2, 1]]
#   y2 = S2 [1,1,1]^T + .5 [0,1] = [.75, 6.5]
S2_HAND = np.array([[0.75, 0.25, -0.25], [3.0, 2.0, 1.0]])
Y_HAND = np.array([[2.0, 3.0], [0.75, 6.5]])


def test_m2_conventional_hand_two_steps(oracle_mod):
    h0, x, dt, Bm, Cm, A, D = _tiny_inputs()
    y, S, rd, wr = oracle_mod.m2_conventional(h0, x, dt, Bm, Cm, A, D)
    np.testing.assert_allclose(y[:, 0, 0], Y_HAND, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], S2_HAND, rtol=0, atol=1e-14)
    assert rd[0, 0] == 2 and wr[0, 0] == 2


def test_m2_replay_hand_two_steps(oracle_mod):
    h0, x, dt, Bm, Cm, A, D = _tiny_inputs()
    st = oracle_mod.M2Replay(h0, G=1, L=16)
    y, lt, ft = st.decode(x, dt, Bm, Cm, A, D)
    np.testing.assert_allclose(y[:, 0, 0], Y_HAND, rtol=0, atol=1e-14)
    # no flush yet: the checkpoint is untouched, two records are buffered
    np.testing.assert_array_equal(st.h0, h0)
    assert list(lt[:, 0, 0]) == [1, 2] and ft.sum() == 0
    np.testing.assert_allclose(st.materialize(A)[0, 0], S2_HAND, rtol=0, atol=1e-14)
    st.flush(A, force=True)
    np.testing.assert_allclose(st.h0[0, 0], S2_HAND, rtol=0, atol=1e-14)
    assert st.len[0, 0] == 0


def _draw(name, T, seqs=None, **kw):
    w = wl.make(name, **kw)
    g = wl.Generator(w, seqs)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(T)
    return w, A, D, S0, st


@pytest.mark.parametrize("name,T,kw", [
    ("m2_tiny", 64, {}),
    ("m2_serving", 40, {"B": 2}),
])
def test_m2_replay_equals_conventional(oracle_mod, name, T, kw):
    """[sitech §How ReplaySSM works]: outputs match conventional decoding up to
    floating-point differences -- in fp64 that is ~1e-13."""
    w, A, D, S0, st = _draw(name, T, **kw)
    yc, Sc, _, _ = oracle_mod.m2_conventional(S0, st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L)
    yr, lt, ft = rp.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    assert per_step_rel_err(yr, yc) < 1e-12
    assert rel_err(rp.materialize(A), Sc) < 1e-12


def test_m2_pure_sum_when_A_is_zero(oracle_mod):
    """A = 0 gives dA = 1: the state is h0 plus a plain sum of dt x B^T and the
    output needs no decay weights at all."""
    w, A, D, S0, st = _draw("m2_tiny", 12, B=2)
    A0 = np.zeros_like(A.numpy(), dtype=np.float64)
    x, dt, Bm, Cm = (st[k].double().numpy() for k in ("x", "dt", "Bm", "Cm"))
    h0 = S0.double().numpy()
    g = np.arange(w.H) // (w.H // w.G)
    # closed form with einsum over the whole history
    Bh, Ch = Bm[:, :, g], Cm[:, :, g]                     # [T,B,H,N]
    incr = np.einsum("tbh,tbhp,tbhn->tbhpn", dt, x, Bh)   # dt_t x_t B_t^T
    S_t = h0[None] + np.cumsum(incr, axis=0)
    y_ref = np.einsum("tbhpn,tbhn->tbhp", S_t, Ch) + D.double().numpy()[None, None, :, None] * x
    yc, Sc, _, _ = oracle_mod.m2_conventional(S0, x, dt, Bm, Cm, A0, D)
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L)
    yr, _, _ = rp.decode(x, dt, Bm, Cm, A0, D)
    assert per_step_rel_err(yc, y_ref) < 1e-12
    assert per_step_rel_err(yr, y_ref) < 1e-12
    assert rel_err(Sc, S_t[-1]) < 1e-12


def test_m2_dt_zero_leaves_state(oracle_mod):
    """dt = 0: dA = 1 and no input enters; y = h0 C + D x."""
    w, A, D, S0, st = _draw("m2_tiny", 20, B=2)
    x, Bm, Cm = (st[k].double().numpy() for k in ("x", "Bm", "Cm"))
    dt0 = np.zeros(st["dt"].shape)
    yc, Sc, _, _ = oracle_mod.m2_conventional(S0, x, dt0, Bm, Cm, A, D)
    np.testing.assert_array_equal(Sc, S0.double().numpy())
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L)
    yr, _, _ = rp.decode(x, dt0, Bm, Cm, A, D)
    h0 = S0.double().numpy()
    Ch = Cm[:, :, np.arange(w.H) // (w.H // w.G)]
    y_ref = np.einsum("bhpn,tbhn->tbhp", h0, Ch) + D.double().numpy()[None, None, :, None] * x
    assert per_step_rel_err(yc, y_ref) < 1e-13
    assert per_step_rel_err(yr, y_ref) < 1e-13
    np.testing.assert_array_equal(rp.h0, h0)  # the folds at 16 reproduce h0 exactly


def test_m2_unit_vectors_select_columns(oracle_mod):
    """B = e_j writes the input into state column j only; C = e_m reads column m."""
    rng = np.random.default_rng(5)
    P, N = 4, 5
    S0 = rng.standard_normal((1, 1, P, N))
    xv = rng.standard_normal(P)
    j, m, dtv, Av, Dv = 3, 1, 0.7, -1.3, 0.25
    Bv = np.zeros(N); Bv[j] = 1.0
    Cv = np.zeros(N); Cv[m] = 1.0
    y, S, _, _ = oracle_mod.m2_conventional(
        S0, xv.reshape(1, 1, 1, P), np.array([[[dtv]]]), Bv.reshape(1, 1, 1, N),
        Cv.reshape(1, 1, 1, N), np.array([Av]), np.array([Dv]))
    dA = math.exp(dtv * Av)
    exp_S = dA * S0[0, 0].copy()
    exp_S[:, j] += dtv * xv
    np.testing.assert_allclose(S[0, 0], exp_S, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(y[0, 0, 0], exp_S[:, m] + Dv * xv, rtol=1e-15, atol=1e-15)


def test_m2_traffic_per_window(oracle_mod):
    """Counts of whole-state reads and writes over windows of 16 tokens."""
    g = read_kv("window_traffic.txt")
    L = g["window"]
    w, A, D, S0, st = _draw("m2_tiny", 4 * L, B=2)
    _, _, rd, wr = oracle_mod.m2_conventional(S0, st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    rp = oracle_mod.M2Replay(S0, G=w.G, L=L)
    rp.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    windows = 4
    assert np.all(rd == windows * g["conventional_state_reads_per_window"])
    assert np.all(wr == windows * g["conventional_state_writes_per_window"])
    assert np.all(rp.writes == windows * g["replay_checkpoint_writes_per_window"])
    assert np.all(rp.reads == windows * L)


def test_m2_flush_schedule_tiny(oracle_mod):
    """m2_tiny: 64 steps with a 16-record buffer flush on steps 16, 32, 48, 64
    (1-based) and nowhere else; the buffer length after step t is t mod 16."""
    L = read_kv("window_traffic.txt")["window"]
    w, A, D, S0, st = _draw("m2_tiny", 64)
    rp = oracle_mod.M2Replay(S0, G=w.G, L=L)
    _, lt, ft = rp.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    steps = np.arange(1, 65)
    flush_steps = steps[ft[:, 0, 0] == 1]
    assert list(flush_steps) == [16, 32, 48, 64]
    assert np.all(ft == ft[:, :1, :1])
    assert np.all(lt == (steps % L)[:, None, None])


def test_m2_partial_window_flush_and_resume(oracle_mod):
    """Decode 20 steps (len 4), force a flush, decode 20 more: the outputs and
    the materialised state still follow conventional decoding."""
    w, A, D, S0, st = _draw("m2_tiny", 40, B=2)
    yc, Sc, _, _ = oracle_mod.m2_conventional(S0, st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L)
    sl = lambda a, b: [st[k][a:b] for k in ("x", "dt", "Bm", "Cm")]
    y1, lt, _ = rp.decode(*sl(0, 20), A, D)
    assert np.all(rp.len == 4)
    _, Sc20, _, _ = oracle_mod.m2_conventional(S0, *sl(0, 20), A, D)
    assert rel_err(rp.materialize(A), Sc20) < 1e-12
    rp.flush(A, force=True)
    assert np.all(rp.len == 0)
    assert rel_err(rp.h0, Sc20) < 1e-12
    y2, lt2, ft2 = rp.decode(*sl(20, 40), A, D)
    assert per_step_rel_err(np.concatenate([y1, y2]), yc) < 1e-12
    # after the forced flush the window restarts: the next flush is 16 steps later
    assert list(np.nonzero(ft2[:, 0, 0])[0] + 21) == [36]


def test_m2_oracle_rejects_bad_len(oracle_mod):
    w, A, D, S0, st = _draw("m2_tiny", 2, B=1)
    rp = oracle_mod.M2Replay(S0, G=w.G, L=w.L)
    rp.len[:] = 16
    with pytest.raises(ValueError):
        rp.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
