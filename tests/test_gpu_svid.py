"""GPU parity of the initialisation (Iterative Residual SVID with importance-scaled
preconditioning, RaBiT paper sec. 4.3) against the float64 oracle in oracle/svid.py.

The GPU finds each leading singular pair of |R| by power steps in fp32; the oracle takes it
from a library SVD in float64.  With enough steps (100 here; the error of a step shrinks by
sigma_2/sigma_1, about 0.5 on these inputs) the two agree to fp32 rounding.  Tolerances,
derived from the arithmetic: fp32 sums over K terms (about sqrt(K) * 2^-24 relative) carried
through T iterations stay below 1e-5 in a float32 emulation of the same steps on these
inputs, so the scales and the reconstruction must agree within 1e-4 (Frobenius, relative),
and at most 1e-4 of the signs may differ (residual elements within rounding of 0).  One
such flip moves its element by 2 |a b|, which on a large matrix alone exceeds 1e-4 of the
norm, so the reconstruction is compared where every path's sign agrees.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import svid as osvid
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu
TOL = 1e-4
SIGN_TOL = 1e-4
ALPHA_IN, ALPHA_OUT = 0.8, 0.65   # the pages' Table 11 intensities for Llama2-7B, 2 bits


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from bit_gemv_rabit_b200 import build
    build.build()
    rabit.load()
    rabit.rabit_read_fault(clear=True)
    yield
    assert rabit.rabit_read_fault(clear=True) == 0


def fro(x, ref):
    return float(np.linalg.norm(np.asarray(x, np.float64) - ref) / np.linalg.norm(ref))


def recon_err(S, a, b, So, ao, bo):
    """Relative Frobenius error of the reconstruction where all paths' signs agree."""
    rec, ref = osvid.reconstruct(S, a, b), osvid.reconstruct(So, ao, bo)
    agree = np.all(S == So, axis=0)
    return float(np.linalg.norm((rec - ref)[agree]) / np.linalg.norm(ref))


def gpu_init(W, s_in, s_out, P, T, power_iters=100, ldw=None, power_tol=0.0):
    N, K = W.shape
    if ldw is None:
        Wt = torch.from_numpy(W).cuda()
    else:
        Wt = torch.zeros((N, ldw), device="cuda")
        Wt[:, :K] = torch.from_numpy(W).cuda()
        Wt = Wt[:, :K]
    a = torch.full((P, N), float("nan"), device="cuda")
    b = torch.full((P, K), float("nan"), device="cuda")
    packed = rabit.alloc_packed(N, K, P=P)
    packed.view(torch.int32).fill_(-0x5A5A5A5B)   # 0xA5A5A5A5: every word must be written
    ws = rabit.alloc_svid_init_workspace(N, K, P)
    rabit.rabit_svid_init(Wt, torch.from_numpy(s_in).cuda(), torch.from_numpy(s_out).cuda(), ALPHA_IN,
                          ALPHA_OUT, a, b, packed, ws, P=P, T=T, power_iters=power_iters, power_tol=power_tol)
    torch.cuda.synchronize()
    return a.cpu().numpy(), b.cpu().numpy(), packed.cpu().numpy()


# (1000, 9001): three column sweeps of the power launch, the last ragged; (64, 96): fewer rows
# than CTAs, so some CTAs own no row
@pytest.mark.parametrize("N,K,P,T", [(64, 96, 2, 3), (100, 203, 3, 2), (256, 512, 2, 20),
                                     (256, 512, 3, 20), (1024, 4096, 2, 3), (1000, 9001, 2, 2),
                                     (3000, 257, 3, 2)])
def test_svid_init_matches_oracle(N, K, P, T):
    W = inputs.weight(21 + N, N, K, outlier_frac=0.01)
    s_in, s_out = inputs.calibration_stats(21 + N, N, K)
    So, ao, bo = osvid.svid_init(W, s_in, s_out, ALPHA_IN, ALPHA_OUT, P=P, T=T)
    a, b, packed = gpu_init(W, s_in, s_out, P, T)
    S = oracle.unpack(packed, N, K, P=P)
    assert np.mean(S != So) <= SIGN_TOL
    # every bit that holds no column (padding columns, the 3-path padding word) is 0
    column_bits = oracle.pack(-np.ones_like(So))
    assert not np.any(packed.view(np.uint32) & ~column_bits)
    assert fro(a, ao) <= TOL and fro(b, bo) <= TOL
    assert recon_err(S, a, b, So, ao, bo) <= TOL


def test_svid_init_recovers_preconditioned_signed_rank1():
    """W = s_out^-alpha_out (.) (g0 S0 h0) (.) s_in^-alpha_in: the first path rebuilds W."""
    N, K = 96, 160
    rng = np.random.default_rng(4)
    g0, h0 = rng.uniform(0.5, 2.0, N), rng.uniform(0.5, 2.0, K)
    S0 = np.where(rng.random((N, K)) < 0.5, -1, 1).astype(np.int8)
    s_in, s_out = inputs.calibration_stats(4, N, K)
    si = s_in.astype(np.float64) ** ALPHA_IN
    so = s_out.astype(np.float64) ** ALPHA_OUT
    W = ((g0[:, None] * S0 * h0[None, :]) / so[:, None] / si[None, :]).astype(np.float32)
    a, b, packed = gpu_init(W, s_in, s_out, P=2, T=2, power_iters=40)
    S = oracle.unpack(packed, N, K, P=2)
    np.testing.assert_array_equal(S[0], S0)
    assert fro(osvid.reconstruct(S, a, b), W.astype(np.float64)) <= 1e-5


def test_svid_init_pitched_w_and_repeatability():
    N, K, P, T = 130, 260, 2, 4
    W = inputs.weight(31, N, K)
    s_in, s_out = inputs.calibration_stats(31, N, K)
    a1, b1, p1 = gpu_init(W, s_in, s_out, P, T, power_iters=30)
    a2, b2, p2 = gpu_init(W, s_in, s_out, P, T, power_iters=30, ldw=K + 21)
    np.testing.assert_array_equal(p1, p2)
    np.testing.assert_array_equal(a1, a2)
    np.testing.assert_array_equal(b1, b2)


def test_svid_init_degenerate_cases():
    """W = 0 gives zero scales and all-+1 signs; W = diag(3, -2, 1) with three paths is
    rebuilt exactly, a_i = b_i = sqrt(sigma_i) e_i with sigma = 3, 2, 1 (hand-worked in the
    oracle's pins)."""
    ones3 = np.ones(3, np.float32)
    a, b, packed = gpu_init(np.zeros((5, 7), np.float32), *inputs.calibration_stats(2, 5, 7), P=2, T=3)
    assert not np.any(a) and not np.any(b)
    assert np.all(oracle.unpack(packed, 5, 7, P=2) == 1)
    W = np.diag([3.0, -2.0, 1.0]).astype(np.float32)
    a, b, packed = gpu_init(W, ones3, ones3, P=3, T=1)
    S = oracle.unpack(packed, 3, 3, P=3)
    np.testing.assert_array_equal(S[0], np.where(W < 0, -1, 1))
    assert fro(osvid.reconstruct(S, a, b), W.astype(np.float64)) <= 1e-5
    for i, sig in enumerate([3.0, 2.0, 1.0]):
        np.testing.assert_allclose(a[i], np.sqrt(sig) * np.eye(3)[i], atol=1e-5)
        np.testing.assert_allclose(b[i], np.sqrt(sig) * np.eye(3)[i], atol=1e-5)


def test_svid_init_settled_stop_matches_oracle():
    """With a relative tolerance on sigma the power steps stop early; the result still meets
    the oracle's bar, and is deterministic."""
    N, K, P, T = 512, 768, 2, 6
    W = inputs.weight(77, N, K, outlier_frac=0.01)
    s_in, s_out = inputs.calibration_stats(77, N, K)
    So, ao, bo = osvid.svid_init(W, s_in, s_out, ALPHA_IN, ALPHA_OUT, P=P, T=T)
    a, b, packed = gpu_init(W, s_in, s_out, P, T, power_iters=400, power_tol=1e-6)
    a2, b2, p2 = gpu_init(W, s_in, s_out, P, T, power_iters=400, power_tol=1e-6)
    assert np.array_equal(a, a2) and np.array_equal(b, b2) and np.array_equal(packed, p2)
    S = oracle.unpack(packed, N, K, P=P)
    assert np.mean(S != So) <= SIGN_TOL
    assert recon_err(S, a, b, So, ao, bo) <= TOL
