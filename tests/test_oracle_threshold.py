"""Pins of the oracle's rank selection and factorisation against closed forms, optimality
conditions, brute force and the Eckart-Young theorem (no GPU)."""
import math

import numpy as np
import pytest
from scipy.optimize import minimize

import oracle as O
from rank_quantized_kv_decode_b200 import synth


def rot(a):
    return np.array([[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]])


def test_svt_diagonal_closed_form():
    d = np.array([3.0, -1.0, 0.5, 2.0])
    got = O.svt(np.diag(d), 0.75)
    want = np.diag(np.sign(d) * np.maximum(np.abs(d) - 0.75, 0.0))
    np.testing.assert_allclose(got, want, atol=1e-14)


@pytest.mark.parametrize("s1,s2,tau", [(3.0, 1.0, 0.5), (2.0, 0.25, 0.5), (1.0, 0.9, 2.0)])
def test_svt_2x2_known_singular_values(s1, s2, tau):
    a, b = 0.7, -1.9
    W = rot(a) @ np.diag([s1, s2]) @ rot(b).T
    want = rot(a) @ np.diag([max(s1 - tau, 0), max(s2 - tau, 0)]) @ rot(b).T
    np.testing.assert_allclose(O.svt(W, tau), want, atol=1e-13)


def test_svt_prox_optimality_conditions():
    g = np.random.default_rng(3)
    W = g.standard_normal((7, 5))
    tau = 1.1
    X = O.svt(W, tau)
    U, s, Vt = np.linalg.svd(X)
    r = int(np.sum(s > 1e-10))
    assert r == O.kept_rank(np.linalg.svd(W, compute_uv=False), tau)
    Ur, Vr = U[:, :r], Vt[:r].T
    Z = (W - X) / tau - Ur @ Vr.T
    assert np.linalg.norm(Z, 2) <= 1 + 1e-10
    np.testing.assert_allclose(Ur.T @ Z, 0, atol=1e-10)
    np.testing.assert_allclose(Z @ Vr, 0, atol=1e-10)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_svt_brute_force_2x2(seed):
    g = np.random.default_rng(seed)
    W = g.standard_normal((2, 2))
    tau = 0.6

    def obj(v):
        X = v.reshape(2, 2)
        return 0.5 * np.sum((X - W) ** 2) + tau * np.sum(np.linalg.svd(X, compute_uv=False))

    best = None
    for start in [W.ravel(), np.zeros(4), g.standard_normal(4)]:
        res = minimize(obj, start, method="Nelder-Mead",
                       options=dict(xatol=1e-11, fatol=1e-14, maxiter=40000))
        if best is None or res.fun < best.fun:
            best = res
    X = O.svt(W, tau)
    assert obj(X.ravel()) <= best.fun + 1e-10
    np.testing.assert_allclose(X.ravel(), best.x, atol=2e-5)


def test_kept_rank_is_rank_of_svt():
    g = np.random.default_rng(5)
    W = g.standard_normal((9, 6)) @ np.diag([5, 3, 2, 1, 0.5, 0.1])
    s = np.linalg.svd(W, compute_uv=False)
    for tau in [0.0, 0.05, 0.3, 1.0, 2.5, 100.0]:
        X = O.svt(W, tau)
        assert O.kept_rank(s, tau) == np.linalg.matrix_rank(X, tol=1e-9)


def _constructed(n, m, scale, seed):
    g = np.random.default_rng(seed)
    k = min(n, m)
    U = synth.haar_frame(g, n, k)
    V = synth.haar_frame(g, m, k)
    s = synth.spectrum(k, scale)
    return U, s, V, (U * s) @ V.T


def test_eckart_young_workload1_keys():
    # The tiny workload's key projection: 256 x 256, sigma_i = exp(-i/16), rank 64.
    U, s, V, W = _constructed(256, 256, 16.0, 11)
    A, B, sig = O.joint_factors(W, 64)
    E = W - A @ B
    closed = math.sqrt(sum(math.exp(-2 * i / 16) for i in range(64, 256)))
    assert abs(closed - 0.0534315) < 5e-8
    assert abs(np.linalg.norm(E, "fro") - closed) < 1e-12
    assert abs(np.linalg.norm(E, 2) - math.exp(-4)) < 1e-12  # sigma_64
    np.testing.assert_allclose(sig, s, rtol=1e-12, atol=1e-15)
    # the kept singular values are not shrunk: A has column norms sigma_0..sigma_63
    np.testing.assert_allclose(np.linalg.norm(A, axis=0), s[:64], rtol=1e-12)
    # same factors as the known construction, up to the sign of each singular pair
    A2, B2 = O.factors_from_svd(U, s, V, 64)
    sign = np.sign(np.sum(A * A2, axis=0))
    np.testing.assert_allclose(A * sign, A2, atol=1e-10)
    np.testing.assert_allclose(B * sign[:, None], B2, atol=1e-10)


def test_joint_not_worse_than_headwise_at_equal_total_rank():
    # JD has lower approximation error than HD at the same latent size (STAR-KV summary,
    # Methodology §2): the HD reconstruction has rank <= sum of head ranks.
    _, _, _, W = _constructed(64, 64, 8.0, 4)
    H, d, r = 4, 16, 6
    A, B, _ = O.joint_factors(W, H * r)
    ej = np.linalg.norm(W - A @ B)
    parts = O.headwise_factors(W, H, d, [r] * H)
    Wh = np.concatenate([a @ b for a, b, _ in parts], axis=1)
    eh = np.linalg.norm(W - Wh)
    assert ej <= eh + 1e-12


def test_tau_for_mean_rank_hand_example():
    spectra = [np.array([5.0, 4, 3, 2, 1]), np.array([10.0, 1, 0.5])]
    tau, ranks = O.tau_for_mean_rank(spectra, 2.5, 1, 5)
    assert tau == 1.0
    assert list(ranks) == [4, 1]


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_tau_for_mean_rank_brute_force(seed):
    g = np.random.default_rng(seed)
    spectra = [np.sort(g.exponential(size=12))[::-1] for _ in range(5)]
    lo, hi, target = 2, 9, 5.0
    tau, ranks = O.tau_for_mean_rank(spectra, target, lo, hi)

    def mean_at(t):
        return np.mean([np.clip(np.sum(s > t), lo, hi) for s in spectra])

    grid = np.linspace(0, max(s.max() for s in spectra) * 1.01, 20001)
    errs = np.array([abs(mean_at(t) - target) for t in grid])
    best = errs.min()
    assert abs(abs(np.mean(ranks) - target) - best) < 1e-12
    assert list(ranks) == [int(np.clip(np.sum(s > tau), lo, hi)) for s in spectra]
    # ties go to the larger threshold: nothing above tau on the grid is as good
    above = grid[grid > tau + 1e-9]
    assert all(abs(mean_at(t) - target) > best + 1e-12 for t in above if
               mean_at(t) != mean_at(tau))
