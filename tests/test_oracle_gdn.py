"""Pins for the Gated DeltaNet half of the CPU oracle (no GPU)."""
import numpy as np
import pytest

from ssm_state_storage_b200 import workloads as wl
from tests._util import per_step_rel_err, read_kv, rel_err


def _one(S0, k, v, a, b, q, scale=1.0):
    DK, DV = S0.shape
    return dict(S0=S0.reshape(1, 1, DK, DV), q=q.reshape(1, 1, 1, DK), k=k.reshape(1, 1, 1, DK),
                v=v.reshape(1, 1, 1, DV), alpha=np.array([[[a]]]), beta=np.array([[[b]]]),
                scale=scale)


def _conv(oracle_mod, d):
    return oracle_mod.gdn_conventional(d["S0"], d["q"], d["k"], d["v"], d["alpha"], d["beta"],
                                       d["scale"])


def _replay(oracle_mod, d, L=16):
    rp = oracle_mod.GDNReplay(d["S0"], L=L, scale=d["scale"])
    o, lt, ft = rp.decode(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
    return o, rp


# Hand derivation, S <- a (I - b k k^T) S + b k v^T, o = S^T q:
#   S0 = I, k1 = [1,0], v1 = [2,3], a1 = .5, b1 = 1:
#     S1 = .5 diag(0,1) + [1,0]^T[2,3] = [[2,3],[0,.5]];  q1 = [0,1]: o1 = [0, .5]
#   k2 = [.6,.8], v2 = [1,-1], a2 = 1, b2 = .5:  k2^T S1 = [1.2, 2.2]
#     S2 = S1 + .5 k2 (v2 - [1.2,2.2])^T = [[1.94, 2.04], [-.08, -.78]]
#     q2 = [1,1]: o2 = [1.86, 1.26]
def test_gdn_hand_two_steps(oracle_mod):
    S0 = np.eye(2).reshape(1, 1, 2, 2)
    q = np.array([[0.0, 1.0], [1.0, 1.0]]).reshape(2, 1, 1, 2)
    k = np.array([[1.0, 0.0], [0.6, 0.8]]).reshape(2, 1, 1, 2)
    v = np.array([[2.0, 3.0], [1.0, -1.0]]).reshape(2, 1, 1, 2)
    al = np.array([0.5, 1.0]).reshape(2, 1, 1)
    be = np.array([1.0, 0.5]).reshape(2, 1, 1)
    S2 = np.array([[1.94, 2.04], [-0.08, -0.78]])
    o_hand = np.array([[0.0, 0.5], [1.86, 1.26]])
    o, S, rd, wr = oracle_mod.gdn_conventional(S0, q, k, v, al, be)
    np.testing.assert_allclose(o[:, 0, 0], o_hand, rtol=0, atol=1e-14)
    np.testing.assert_allclose(S[0, 0], S2, rtol=0, atol=1e-14)
    rp = oracle_mod.GDNReplay(S0, L=16)
    o2, _, _ = rp.decode(q, k, v, al, be)
    np.testing.assert_allclose(o2[:, 0, 0], o_hand, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(rp.h0, S0)
    np.testing.assert_allclose(rp.materialize()[0, 0], S2, rtol=0, atol=1e-14)


def test_gdn_delta_rule_invariants(oracle_mod):
    """For a unit key k: S'^T k = a(1-b) S^T k + b v, and S'^T w = a S^T w for
    every w orthogonal to k -- together these fix S' completely."""
    rng = np.random.default_rng(11)
    DK, DV = 8, 6
    S0 = rng.standard_normal((DK, DV))
    k = rng.standard_normal(DK); k /= np.linalg.norm(k)
    v = rng.standard_normal(DV)
    a, b = 0.8, 0.3
    Q, _ = np.linalg.qr(np.column_stack([k, rng.standard_normal((DK, DK - 1))]))
    Q[:, 0] = k  # QR fixes the first column only up to sign
    for col in range(DK):
        qv = Q[:, col]
        d = _one(S0, k, v, a, b, qv)
        o, S, _, _ = _conv(oracle_mod, d)
        o_r, _ = _replay(oracle_mod, d)
        if col == 0:
            exp = a * (1 - b) * (S0.T @ k) + b * v
        else:
            exp = a * (S0.T @ qv)
        np.testing.assert_allclose(o[0, 0, 0], exp, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(o_r[0, 0, 0], exp, rtol=1e-13, atol=1e-13)


def test_gdn_beta_zero(oracle_mod):
    """beta = 0: S <- alpha S; with alpha = 1 as well the state is unchanged exactly."""
    w = wl.make("gdn_serving", B=1, H=2)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(20)
    zb = np.zeros(st["beta"].shape)
    ones = np.ones(st["alpha"].shape)
    o, S, _, _ = oracle_mod.gdn_conventional(S0, st["q"], st["k"], st["v"], ones, zb)
    np.testing.assert_array_equal(S, S0.double().numpy())
    o2, S2, _, _ = oracle_mod.gdn_conventional(S0, st["q"], st["k"], st["v"], st["alpha"], zb)
    decay = np.prod(st["alpha"].double().numpy(), axis=0)
    np.testing.assert_allclose(S2, S0.double().numpy() * decay[..., None, None], rtol=1e-13)
    rp = oracle_mod.GDNReplay(S0, L=16)
    o3, _, _ = rp.decode(st["q"], st["k"], st["v"], ones, zb)
    np.testing.assert_array_equal(rp.h0, S0.double().numpy())
    assert per_step_rel_err(o3, o) < 1e-13


def test_gdn_orthonormal_keys_write_rows(oracle_mod):
    """alpha = beta = 1 with keys e_0..e_{DK-1}: each step overwrites one row of
    the state with its value vector, so after DK steps S = V exactly."""
    rng = np.random.default_rng(3)
    DK, DV, T = 16, 8, 16
    S0 = rng.standard_normal((1, 1, DK, DV))
    k = np.eye(DK)[:T].reshape(T, 1, 1, DK)
    v = rng.standard_normal((T, 1, 1, DV))
    q = rng.standard_normal((T, 1, 1, DK))
    one = np.ones((T, 1, 1))
    o, S, _, _ = oracle_mod.gdn_conventional(S0, q, k, v, one, one)
    np.testing.assert_allclose(S[0, 0], v[:, 0, 0], rtol=0, atol=1e-15)
    rp = oracle_mod.GDNReplay(S0, L=16)
    o2, lt, ft = rp.decode(q, k, v, one, one)
    assert ft[-1, 0, 0] == 1  # the 16th record flushed
    np.testing.assert_allclose(rp.h0[0, 0], v[:, 0, 0], rtol=0, atol=1e-14)
    assert per_step_rel_err(o2, o) < 1e-12


@pytest.mark.parametrize("kw,T", [({"B": 2, "H": 4}, 40), ({"B": 1, "H": 2, "P": 16, "N": 8}, 70)])
def test_gdn_replay_equals_conventional(oracle_mod, kw, T):
    w = wl.make("gdn_serving", **kw)
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = g.steps(T)
    oc, Sc, rd, wr = oracle_mod.gdn_conventional(S0, st["q"], st["k"], st["v"], st["alpha"],
                                                 st["beta"])
    rp = oracle_mod.GDNReplay(S0, L=w.L)
    orr, lt, ft = rp.decode(st["q"], st["k"], st["v"], st["alpha"], st["beta"])
    assert per_step_rel_err(orr, oc) < 1e-11
    assert rel_err(rp.materialize(), Sc) < 1e-11
    # traffic: one checkpoint write per full window, conventional writes every step
    g_ = read_kv("window_traffic.txt")
    assert np.all(rp.writes == T // g_["window"])
    assert np.all(wr == T)
    # the forced flush lands on the conventional state
    rp.flush(force=True)
    assert rel_err(rp.h0, Sc) < 1e-11 and np.all(rp.len == 0)
