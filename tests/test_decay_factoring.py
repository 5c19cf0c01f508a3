"""The verify kernel forms every draft's decay weights from one exponential per
record by factoring through a reference suffix sum (S = suffix sums of dt,
S_ref = S_{nb+1}):
    exp(A (S_{i+1} - S_{e+1})) = exp(A (S_{i+1} - S_ref)) * exp(A (S_ref - S_{e+1})),
    exp(A (S_0 - S_{e+1}))     = exp(A (S_0 - S_ref))     * exp(A (S_ref - S_{e+1})).
This checks the identity in fp64 against the direct form, including extreme
decay rates and step sizes, and that no factor overflows (only the <= 4 draft
records can make an argument positive)."""
import numpy as np
import pytest


def _direct_and_factored(A, dt, nb, nd):
    K = nb + nd
    S = np.concatenate([np.cumsum(dt[::-1])[::-1], [0.0]])      # S_l = sum_{m >= l} dt_m
    ref = S[nb + 1] if nb + 1 <= K else 0.0
    E = np.exp(A * (S[1:K + 1] - ref))                           # lane l: S_{l+1} - S_ref
    G = np.exp(A * (S[0] - ref))
    out = []
    for d in range(nd):
        e = nb + d
        F = np.exp(A * (ref - S[e + 1]))
        w_fact = E[:e + 1] * F * dt[:e + 1]
        lam_fact = G * F
        w_dir = np.exp(A * (S[1:e + 2] - S[e + 1])) * dt[:e + 1]
        lam_dir = np.exp(A * (S[0] - S[e + 1]))
        out.append((w_fact, lam_fact, w_dir, lam_dir, F, E, G))
    return out


@pytest.mark.parametrize("A", [-16.0, -1.0, -0.01])
@pytest.mark.parametrize("nb", [0, 1, 8, 15])
def test_factored_weights_equal_direct(A, nb):
    rng = np.random.default_rng(int(-A * 100) + nb)
    nd = 4
    dt = np.log1p(np.exp(rng.standard_normal(nb + nd) - 2.0))  # softplus(N(0,1) - 2)
    for w_f, l_f, w_d, l_d, F, E, G in _direct_and_factored(A, dt, nb, nd):
        np.testing.assert_allclose(w_f, w_d, rtol=1e-13, atol=0)
        assert l_f == pytest.approx(l_d, rel=1e-13)


def test_no_factor_overflows_at_extremes():
    """A = -16 with dt = 10 per record: the committed records' factors underflow
    gracefully to 0 and the draft factors stay below exp(16 * 40)."""
    A, nb, nd = -16.0, 15, 4
    dt = np.full(nb + nd, 10.0)
    for w_f, l_f, w_d, l_d, F, E, G in _direct_and_factored(A, dt, nb, nd):
        assert np.all(np.isfinite(E)) and np.isfinite(F) and np.isfinite(G)
        assert np.all(np.isfinite(w_f)) and np.isfinite(l_f)
        np.testing.assert_allclose(w_f, w_d, rtol=1e-12, atol=1e-300)
