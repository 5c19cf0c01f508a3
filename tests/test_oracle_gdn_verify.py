"""Pins for the Gated DeltaNet speculative-verify oracle (replay form) against
what the pages and the mathematics fix: drafts evaluated output-only from the
checkpoint and the buffer give the same outputs as stepping a snapshot of the
full state through them, the committed state equals stepping the accepted
prefix, committing nothing leaves the checkpoint bit-identical, and committing
everything equals plain decoding of the concatenated drafts
[sitech §Reducing state traffic...], [hamidun §Where the state problem appears]."""
import numpy as np
import pytest

import oracle

B, H, DK, DV, DN = 2, 3, 8, 6, 4


def _drafts(R, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((R, B, DN, H, DK))
    k = rng.standard_normal((R, B, DN, H, DK))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((R, B, DN, H, DV))
    alpha = np.exp(-np.log1p(np.exp(rng.standard_normal((R, B, DN, H)))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((R, B, DN, H))))
    S0 = 0.1 * rng.standard_normal((B, H, DK, DV))
    return S0, q, k, v, alpha, beta


@pytest.mark.parametrize("L", [5, 16])
def test_replay_verify_equals_snapshot_and_restore(L):
    R = 14
    S0, q, k, v, a, b = _drafts(R, 7 + L)
    acc = np.random.default_rng(L).integers(0, DN + 1, size=(R, B)).astype(np.int32)
    orc = oracle.GDNReplay(S0, L=L, cap=L + DN - 1)
    o, lt = orc.verify(q, k, v, a, b, acc)
    os_, Ss, copies = oracle.gdn_verify_snapshot(S0, q, k, v, a, b, acc)
    np.testing.assert_allclose(o, os_, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(orc.materialize(), Ss, rtol=1e-10, atol=1e-12)
    assert np.all(copies == 2 * R)          # one snapshot and one restore per round
    # the committed length advances by the accepted count and folds at L
    n = np.zeros((B, H), np.int64)
    for r in range(R):
        n = n + acc[r][:, None]
        n = np.where(n >= L, 0, n)
        assert np.array_equal(lt[r], n)


def test_accept_none_keeps_checkpoint_bit_identical():
    R = 6
    S0, q, k, v, a, b = _drafts(R, 3)
    orc = oracle.GDNReplay(S0, L=5, cap=8)
    o, lt = orc.verify(q, k, v, a, b, np.zeros((R, B), np.int32))
    assert np.array_equal(orc.h0, S0)
    assert np.all(lt == 0)
    # every round's drafts are evaluated from the untouched checkpoint
    os_, _, _ = oracle.gdn_verify_snapshot(S0, q, k, v, a, b, np.zeros((R, B), np.int32))
    np.testing.assert_allclose(o, os_, rtol=1e-10, atol=1e-12)


def test_accept_all_equals_plain_decoding():
    R = 8
    S0, q, k, v, a, b = _drafts(R, 11)
    acc = np.full((R, B), DN, np.int32)
    orc = oracle.GDNReplay(S0, L=5, cap=8)
    o, _ = orc.verify(q, k, v, a, b, acc)
    # the concatenated drafts as T = R * DN ordinary steps: [T][B][H][...]
    seq = lambda x: np.moveaxis(x, 2, 1).reshape(R * DN, B, *x.shape[3:])
    oc, S, _, _ = oracle.gdn_conventional(S0, seq(q), seq(k), seq(v), seq(a), seq(b))
    np.testing.assert_allclose(seq(o), oc, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(orc.materialize(), S, rtol=1e-10, atol=1e-12)


def test_bad_acceptance_is_refused():
    S0, q, k, v, a, b = _drafts(1, 5)
    orc = oracle.GDNReplay(S0, L=5, cap=8)
    with pytest.raises(ValueError):
        orc.verify(q, k, v, a, b, np.full((1, B), DN + 1, np.int32))
