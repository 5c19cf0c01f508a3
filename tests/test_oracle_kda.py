"""CPU pins for the Kimi Delta Attention oracle (the gated delta rule with one
decay per key channel, S_t = (I - beta k k^T) Diag(alpha_t) S_{t-1} + beta k v^T,
o = scale S^T q; the layer type named in [hamidun §Why hybrid models became the
norm]).  Pinned to what the mathematics fixes, not to the oracle itself:
equal channels reduce to Gated DeltaNet; the replay form equals stepping the
recurrence [sitech §How ReplaySSM works]; beta = 0 only decays the rows; a
hand-worked two-step case; the delta-rule invariants of one step, which fix
the state completely and tie the decay to the key rows, applied before the
correction."""
import numpy as np
import pytest

import oracle

B, H, DK, DV = 2, 3, 8, 6


def _draw(T, seed, per_channel=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, B, H, DK))
    k = rng.standard_normal((T, B, H, DK))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, B, H, DV))
    z = rng.standard_normal((T, B, H, DK) if per_channel else (T, B, H))
    a = np.exp(-np.log1p(np.exp(z)))
    be = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, B, H))))
    S0 = 0.1 * rng.standard_normal((B, H, DK, DV))
    return S0, q, k, v, a, be


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / np.max(np.abs(b)))


def test_equal_channels_reduce_to_gated_deltanet():
    S0, q, k, v, a, be = _draw(40, 1, per_channel=False)
    a_vec = np.repeat(a[..., None], DK, axis=-1)
    og, Sg, _, _ = oracle.gdn_conventional(S0, q, k, v, a, be)
    ok, Sk, _, _ = oracle.kda_conventional(S0, q, k, v, a_vec, be)
    assert _rel(ok, og) < 1e-13 and _rel(Sk, Sg) < 1e-13
    rg = oracle.GDNReplay(S0, L=16)
    o_rg, _, _ = rg.decode(q, k, v, a, be)
    rk = oracle.KDAReplay(S0, L=16)
    o_rk, _, _ = rk.decode(q, k, v, a_vec, be)
    assert _rel(o_rk, o_rg) < 1e-12 and _rel(rk.h0, rg.h0) < 1e-12


@pytest.mark.parametrize("L", [1, 5, 16])
def test_replay_equals_conventional(L):
    """The pages' identity: outputs from the checkpoint and the buffer equal
    stepping the recurrence, up to rounding; the folds give the same state."""
    T = 40
    S0, q, k, v, a, be = _draw(T, 2 + L)
    oc, Sc, rd, wr = oracle.kda_conventional(S0, q, k, v, a, be)
    rp = oracle.KDAReplay(S0, L=L)
    o, lt, ft = rp.decode(q, k, v, a, be)
    assert _rel(o, oc) < 1e-12
    assert _rel(rp.materialize(), Sc) < 1e-12
    assert np.array_equal(lt[:, 0, 0], (np.arange(1, T + 1) % L))
    assert np.all(rd == T) and np.all(wr == T)            # conventional: every step
    assert np.all(rp.writes == T // L)                    # replay: once per window
    rp.flush(force=True)
    assert _rel(rp.h0, Sc) < 1e-12 and np.all(rp.len == 0)


def test_beta_zero_only_decays_rows():
    S0, q, k, v, a, be = _draw(12, 3)
    _, S, _, _ = oracle.kda_conventional(S0, q, k, v, a, np.zeros_like(be))
    decay = np.prod(a, axis=0)  # [B][H][DK]: per key row
    np.testing.assert_allclose(S, S0 * decay[..., None], rtol=1e-13, atol=0)
    _, S1, _, _ = oracle.kda_conventional(S0, q, k, v, np.ones_like(a), np.zeros_like(be))
    assert np.array_equal(S1, S0)


def test_two_step_hand_case():
    """DK = 2, DV = 1, dyadic values (exact in fp64):
    S0 = [1, 2]; step 1: alpha = (1/2, 1/4), k = (1, 0), v = 3, beta = 1/2:
      Diag(alpha) S0 = [1/2, 1/2], k^T(.) = 1/2, S1 = [1/2 + 1/2 (3 - 1/2), 1/2] = [7/4, 1/2];
    step 2: alpha = (1, 1/2), k = (0, 1), v = -1, beta = 1:
      Diag(alpha) S1 = [7/4, 1/4], k^T(.) = 1/4, S2 = [7/4, 1/4 + (-1 - 1/4)] = [7/4, -1];
    with q = (1, 1): o1 = 9/4, o2 = 3/4."""
    S0 = np.array([1.0, 2.0]).reshape(1, 1, 2, 1)
    q = np.ones((2, 1, 1, 2))
    k = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(2, 1, 1, 2)
    v = np.array([3.0, -1.0]).reshape(2, 1, 1, 1)
    a = np.array([[0.5, 0.25], [1.0, 0.5]]).reshape(2, 1, 1, 2)
    be = np.array([0.5, 1.0]).reshape(2, 1, 1)
    o, S, _, _ = oracle.kda_conventional(S0, q, k, v, a, be)
    assert np.array_equal(S.reshape(-1), [1.75, -1.0])
    assert np.array_equal(o.reshape(-1), [2.25, 0.75])
    rp = oracle.KDAReplay(S0, L=16)
    o_r, _, _ = rp.decode(q, k, v, a, be)
    assert np.array_equal(o_r.reshape(-1), [2.25, 0.75])
    assert np.array_equal(rp.materialize().reshape(-1), [1.75, -1.0])


def test_one_step_invariants_fix_the_state():
    """After one step from S_prev, with D S_prev the rows of S_prev scaled by
    alpha (the key channels): S^T k = (1 - beta) (D S_prev)^T k + beta v
    (|k| = 1), and S^T w = (D S_prev)^T w for every w orthogonal to k.  These
    DK conditions determine S; a decay applied after the correction, or along
    the value axis, breaks them."""
    S0, q, k, v, a, be = _draw(1, 5)
    _, S, _, _ = oracle.kda_conventional(S0, q, k, v, a, be)
    for b in range(B):
        for h in range(H):
            kk, vv, bb = k[0, b, h], v[0, b, h], be[0, b, h]
            DS = S0[b, h] * a[0, b, h][:, None]
            np.testing.assert_allclose(S[b, h].T @ kk, (1 - bb) * (DS.T @ kk) + bb * vv,
                                       rtol=1e-12, atol=1e-14)
            # an orthonormal basis of the complement of k
            Q, _ = np.linalg.qr(np.column_stack([kk, np.eye(DK)[:, :DK - 1]]))
            for c in range(1, DK):
                w = Q[:, c]
                np.testing.assert_allclose(S[b, h].T @ w, DS.T @ w, rtol=1e-11, atol=1e-13)
