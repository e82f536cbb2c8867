"""Pins of the float64 initialisation oracle (oracle/svid.py) against facts fixed outside it.

  * a signed rank-1 matrix g0 (.) S0 (.) h0 is recovered exactly, with and without
    preconditioning (pins the sign rule, the rank-1 step, the preconditioning direction and
    the map-back exponents)                                                 -> svid_init
  * the objective ||W' - sum_i What_i||_F never increases over the (t, i) updates (each update
    is optimal for its path given the others: the sign of the residual, then Eckart-Young
    for |R|)                                                                 -> svid_init
  * the rank-1 step against an independent power iteration written here     -> rank1_abs
  * the reconstruction does not depend on the normalisation of s_in, s_out   -> svid_init
  * the last update is locally optimal: perturbing its scales raises the error -> svid_init
  * a planted mistake in the map-back (wrong exponent sign) is caught by the invariance pin
  * a hand-worked diagonal weight (closed form for 2 and 3 paths) and the zero weight
Source: "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
sec. 4.3 "Stable Initialization for Functional Preservation" (Iterative Residual SVID,
I/O Channel Importance-Scaled Preconditioning), Appendix F.3 (iteration 1 is greedy).
"""
import numpy as np
import pytest

from oracle import svid as osvid
from bit_gemv_rabit_b200 import inputs

ALPHA_IN, ALPHA_OUT = 0.8, 0.65   # the pages' Table 11 intensities for Llama2-7B, 2 bits


def signed_rank1(seed, N, K):
    rng = np.random.default_rng(seed)
    g0 = rng.uniform(0.5, 2.0, N)
    h0 = rng.uniform(0.5, 2.0, K)
    S0 = np.where(rng.random((N, K)) < 0.5, -1, 1).astype(np.int8)
    return g0, S0, h0


@pytest.mark.parametrize("P", [2, 3])
def test_signed_rank1_is_recovered_exactly(P):
    N, K = 24, 40
    g0, S0, h0 = signed_rank1(1, N, K)
    W = g0[:, None] * S0 * h0[None, :]
    ones_k, ones_n = np.ones(K), np.ones(N)
    S, a, b = osvid.svid_init(W, ones_k, ones_n, ALPHA_IN, ALPHA_OUT, P=P, T=3)
    np.testing.assert_array_equal(S[0], S0)
    np.testing.assert_allclose(np.outer(a[0], b[0]), np.outer(g0, h0), rtol=1e-12)
    for i in range(1, P):           # the residual is 0 up to the rounding of the first path
        assert np.max(np.outer(a[i], b[i])) <= 1e-12 * np.max(np.abs(W))
    np.testing.assert_allclose(osvid.reconstruct(S, a, b), W, rtol=1e-12, atol=0)


def test_preconditioned_signed_rank1_maps_back_exactly():
    """W = s_out^-alpha_out (.) (g0 S0 h0) (.) s_in^-alpha_in makes W' signed rank-1; the scales
    mapped back must rebuild W itself."""
    N, K = 30, 52
    g0, S0, h0 = signed_rank1(2, N, K)
    s_in, s_out = inputs.calibration_stats(3, N, K)
    si, so = s_in.astype(np.float64) ** ALPHA_IN, s_out.astype(np.float64) ** ALPHA_OUT
    W = (g0[:, None] * S0 * h0[None, :]) / so[:, None] / si[None, :]
    S, a, b = osvid.svid_init(W, s_in, s_out, ALPHA_IN, ALPHA_OUT, P=2, T=2)
    np.testing.assert_array_equal(S[0], S0)
    np.testing.assert_allclose(osvid.reconstruct(S, a, b), W, rtol=1e-11, atol=0)
    np.testing.assert_allclose(np.outer(a[0], b[0]), W * S0, rtol=1e-11)


@pytest.mark.parametrize("P,precond", [(2, False), (2, True), (3, True)])
def test_objective_never_increases(P, precond):
    N, K = 48, 80
    W = inputs.weight(5, N, K, outlier_frac=0.01)
    s_in, s_out = inputs.calibration_stats(5, N, K) if precond else (np.ones(K), np.ones(N))
    S, a, b, hist = osvid.svid_init(W, s_in, s_out, ALPHA_IN, ALPHA_OUT, P=P, T=8, history=True)
    assert len(hist) == 1 + 8 * P
    h = np.array(hist)
    assert np.all(np.diff(h) <= 1e-12 * h[0])
    assert h[-1] < h[P]           # iterating improves on the greedy (t = 1) decomposition here
    Wp = osvid.precondition(W, s_in, s_out, ALPHA_IN, ALPHA_OUT)
    si = np.asarray(s_in, np.float64) ** ALPHA_IN
    so = np.asarray(s_out, np.float64) ** ALPHA_OUT
    Wh = osvid.reconstruct(S, a * so[None, :], b * si[None, :])
    assert abs(np.linalg.norm(Wp - Wh) - h[-1]) <= 1e-10 * h[0]


def test_diagonal_weight_hand_case():
    """W = diag(3, -2, 1), no preconditioning.  |R| of each update is diagonal, so its leading
    rank-1 part is the largest entry alone: path 1 takes 3 (sigma 3, u = v = e1), path 2 takes
    -2, path 3 takes 1.  Zero residual entries are +1 (sign rule).  By hand:
      P = 3: exact, a_i = b_i = sqrt(sigma_i) e_i;
      P = 2: the entry 1 is left over, ||W - W_hat||_F = 1, at every T (fixed point)."""
    W = np.diag([3.0, -2.0, 1.0])
    ones = np.ones(3)
    S, a, b = osvid.svid_init(W, ones, ones, ALPHA_IN, ALPHA_OUT, P=3, T=1)
    np.testing.assert_allclose(osvid.reconstruct(S, a, b), W, atol=1e-12)
    for i, sig in enumerate([3.0, 2.0, 1.0]):
        e = np.eye(3)[i]
        np.testing.assert_allclose(a[i], np.sqrt(sig) * e, atol=1e-12)
        np.testing.assert_allclose(b[i], np.sqrt(sig) * e, atol=1e-12)
    # -2 is negative in W (path 1) and in R_2 = diag(0, -2, 1) (path 2); R_3 = diag(0, 0, 1)
    assert S[0][1, 1] == -1 and S[1][1, 1] == -1 and np.sum(S == -1) == 2
    for T in (1, 2, 5):
        S2, a2, b2 = osvid.svid_init(W, ones, ones, ALPHA_IN, ALPHA_OUT, P=2, T=T)
        assert abs(np.linalg.norm(W - osvid.reconstruct(S2, a2, b2)) - 1.0) <= 1e-12


def test_zero_weight_gives_zero_scales():
    """W = 0: every residual is 0, so sigma = 0, the scales are 0 and the signs +1."""
    N, K = 5, 7
    s_in, s_out = inputs.calibration_stats(2, N, K)
    S, a, b = osvid.svid_init(np.zeros((N, K)), s_in, s_out, ALPHA_IN, ALPHA_OUT, P=2, T=3)
    assert np.all(S == 1) and not np.any(a) and not np.any(b)


def test_rank1_step_matches_power_iteration():
    rng = np.random.default_rng(7)
    R = rng.standard_normal((37, 61)) * np.exp(rng.standard_normal(61))[None, :]
    sigma, u, v = osvid.rank1_abs(R)
    A = np.abs(R)
    x = np.ones(61)
    for _ in range(2000):
        y = A @ x
        x = A.T @ y
        x /= np.linalg.norm(x)
    y = A @ x
    sig_pi = np.linalg.norm(y)
    assert abs(sigma - sig_pi) <= 1e-10 * sigma
    np.testing.assert_allclose(v, x, atol=1e-9)
    np.testing.assert_allclose(u, y / sig_pi, atol=1e-9)
    assert np.all(u >= 0) and np.all(v >= 0)


def test_reconstruction_is_independent_of_stat_normalisation():
    N, K = 40, 72
    W = inputs.weight(9, N, K)
    s_in, s_out = inputs.calibration_stats(9, N, K)
    S1, a1, b1 = osvid.svid_init(W, s_in, s_out, ALPHA_IN, ALPHA_OUT, P=2, T=4)
    S2, a2, b2 = osvid.svid_init(W, 7.0 * s_in, 0.3 * s_out, ALPHA_IN, ALPHA_OUT, P=2, T=4)
    np.testing.assert_array_equal(S1, S2)
    # the same iteration on inputs scaled by constants: equal up to rounding
    np.testing.assert_allclose(osvid.reconstruct(S2, a2, b2), osvid.reconstruct(S1, a1, b1),
                               rtol=1e-6, atol=0)


def test_last_update_is_locally_optimal():
    N, K = 32, 64
    W = inputs.weight(11, N, K)
    s_in, s_out = inputs.calibration_stats(11, N, K)
    S, a, b = osvid.svid_init(W, s_in, s_out, ALPHA_IN, ALPHA_OUT, P=2, T=5)
    Wp = osvid.precondition(W, s_in, s_out, ALPHA_IN, ALPHA_OUT)
    si = np.asarray(s_in, np.float64) ** ALPHA_IN
    so = np.asarray(s_out, np.float64) ** ALPHA_OUT
    g, h = a * so[None, :], b * si[None, :]
    base = np.linalg.norm(Wp - osvid.reconstruct(S, g, h))
    rng = np.random.default_rng(12)
    for _ in range(20):
        g2, h2 = g.copy(), h.copy()
        g2[1] *= 1 + 1e-3 * rng.standard_normal(N)
        h2[1] *= 1 + 1e-3 * rng.standard_normal(K)
        assert np.linalg.norm(Wp - osvid.reconstruct(S, g2, h2)) >= base * (1 - 1e-12)


def test_planted_map_back_mistake_is_caught(monkeypatch):
    """The invariance pin catches a map-back that multiplies by s^alpha instead of dividing."""
    N, K = 20, 36
    W = inputs.weight(13, N, K)
    s_in, s_out = inputs.calibration_stats(13, N, K)
    real = osvid.svid_init

    def planted(W, s_in, s_out, alpha_in, alpha_out, **kw):
        S, a, b = real(W, s_in, s_out, alpha_in, alpha_out, **kw)
        so = np.asarray(s_out, np.float64) ** alpha_out
        si = np.asarray(s_in, np.float64) ** alpha_in
        return S, a * so[None, :] ** 2, b * si[None, :] ** 2
    monkeypatch.setattr(osvid, "svid_init", planted)
    S1, a1, b1 = osvid.svid_init(W, s_in, s_out, ALPHA_IN, ALPHA_OUT, P=2, T=2)
    S2, a2, b2 = osvid.svid_init(W, 7.0 * s_in, 0.3 * s_out, ALPHA_IN, ALPHA_OUT, P=2, T=2)
    assert not np.allclose(osvid.reconstruct(S2, a2, b2), osvid.reconstruct(S1, a1, b1), rtol=1e-6)


def test_planted_jacobi_order_is_caught_by_the_diagonal_case():
    """Updating every path from the previous iteration's paths (instead of the paths before it
    from this iteration, as the formula states) breaks the hand-worked diagonal case: at t = 1
    every path would see W itself and take its largest entry."""
    W = np.diag([3.0, -2.0, 1.0])
    ones = np.ones(3)

    def jacobi(W, P, T):
        paths = np.zeros((P,) + W.shape)
        for _ in range(T):
            old = paths.copy()
            for i in range(P):
                S, g, h = osvid.svid(W - (old.sum(axis=0) - old[i]))
                paths[i] = g[:, None] * S * h[None, :]
        return paths.sum(axis=0)

    assert np.linalg.norm(jacobi(W, 3, 1) - W) > 1.0
    S, a, b = osvid.svid_init(W, ones, ones, ALPHA_IN, ALPHA_OUT, P=3, T=1)
    assert np.linalg.norm(osvid.reconstruct(S, a, b) - W) < 1e-12
