"""Pins of the optimizer oracle (oracle/optim.py) against what mathematics
fixes: the Newton-Schulz iteration converges to the SVD polar factor, fixes
orthogonal matrices, and is invariant to scaling its input; AdamW's first
step is lr * sign(g) up to eps; a zero gradient leaves only the decay; and
the groups follow the names the pages give."""
import numpy as np
import pytest

from oracle import optim


def _matrix(rng, n, m, smin, smax):
    """A random n x m matrix with singular values spread over [smin, smax]."""
    U, _ = np.linalg.qr(rng.normal(size=(n, n)))
    V, _ = np.linalg.qr(rng.normal(size=(m, m)))
    k = min(n, m)
    S = np.linspace(smin, smax, k)
    return (U[:, :k] * S) @ V[:, :k].T


@pytest.mark.parametrize("n,m", [(12, 12), (20, 8), (8, 20)])
def test_newton_schulz_reaches_the_polar_factor(n, m):
    rng = np.random.default_rng(n * 100 + m)
    M = _matrix(rng, n, m, 0.3, 2.0)
    P = optim.polar_factor(M)
    np.testing.assert_allclose(optim.newton_schulz(M, 25), P, rtol=0, atol=1e-10)
    # few steps: not there yet, but closer with every step (a planted wrong
    # coefficient would stall or diverge)
    errs = [np.linalg.norm(optim.newton_schulz(M, k) - P) for k in range(0, 12)]
    assert all(b < a for a, b in zip(errs, errs[1:]))
    # the polar factor has orthonormal rows or columns
    k = min(n, m)
    G = P.T @ P if n >= m else P @ P.T
    np.testing.assert_allclose(G, np.eye(k), atol=1e-12)


def test_newton_schulz_fixes_orthogonal_matrices_and_ignores_scale():
    rng = np.random.default_rng(7)
    Q, _ = np.linalg.qr(rng.normal(size=(10, 10)))
    # from Q / |Q|_F every singular value is 1/sqrt(10); the iteration brings them to 1
    np.testing.assert_allclose(optim.newton_schulz(Q * 3.0, 30), Q, atol=1e-12)
    M = _matrix(rng, 9, 6, 0.5, 1.5)
    np.testing.assert_allclose(optim.newton_schulz(M, 8), optim.newton_schulz(37.0 * M, 8), atol=1e-12)


def test_adamw_first_step_and_decay():
    rng = np.random.default_rng(3)
    w, g = rng.normal(size=50), rng.normal(size=50)
    lr, wd, eps = 0.01, 0.1, 1e-8
    w2, m, v = optim.adamw_update(w, g, np.zeros(50), np.zeros(50), 1, lr, 0.9, 0.95, eps, wd)
    # bias-corrected moments of the first step are g and g^2
    np.testing.assert_allclose(w2, w - lr * g / (np.abs(g) + eps) - lr * wd * w, rtol=1e-12)
    np.testing.assert_allclose(m, 0.1 * g, rtol=1e-12)
    np.testing.assert_allclose(v, 0.05 * g * g, rtol=1e-12)
    # a zero gradient with zero moments leaves only the decay
    w3, _, _ = optim.adamw_update(w, np.zeros(50), np.zeros(50), np.zeros(50), 4, lr, 0.9, 0.95, eps, wd)
    np.testing.assert_allclose(w3, w * (1 - lr * wd), rtol=1e-12)


def test_muon_without_momentum_is_the_scaled_polar_factor():
    rng = np.random.default_rng(4)
    w, g = rng.normal(size=(16, 8)), _matrix(rng, 16, 8, 0.5, 1.0)
    w2, buf = optim.muon_update(w, g, np.zeros_like(g), 0.02, 0.0, 0.0, 30)
    np.testing.assert_allclose(buf, g)
    np.testing.assert_allclose(w2, w - 0.02 * optim.polar_factor(g), atol=1e-12)


def test_groups_follow_the_pages():
    assert optim.param_group("wte") == "embed"
    assert optim.param_group("ve4") == "embed"
    assert optim.param_group("lm_head") == "head"
    for n in ("resid_lambdas", "x0_lambdas", "ve_gates"):
        assert optim.param_group(n) == "scalar"
    for n in ("h3.wq", "h3.wk", "h3.wv", "h3.wo", "h3.w1", "h3.w2"):
        assert optim.param_group(n) == "matrix"
