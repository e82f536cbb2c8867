"""GPU parity of the scale gradients (the layer's QAT backward for a and b) against the
float64 oracle: grad_a[k][n] = sum_j G S_k b_k, grad_b[k][j] = sum_n G a_k S_k for a given
G = dL/dW_hat, signs held fixed.  fp32 accumulation in a fixed order: normwise <= 1e-5."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu
TOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from bit_gemv_rabit_b200 import build
    build.build()
    rabit.load()
    yield
    assert rabit.rabit_read_fault(clear=True) == 0


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


# (64, 40000, 3): a CTA's range of boxes spans two column tiles of a one-or-two-box column;
# (32, 80000, 2): ranges would span three column tiles, so the direct-load pass runs
@pytest.mark.parametrize("N,K,P", [(33, 129, 2), (300, 520, 2), (1024, 4096, 2), (200, 1100, 3), (4096, 4096, 3),
                                   (64, 40000, 3), (32, 80000, 2)])
def test_scale_grads_match_oracle(N, K, P):
    seed = 500 + N + P
    W = inputs.weight(seed, N, K)
    a, b = inputs.scales(seed, W, P=P)
    rng = np.random.default_rng(seed)
    M = 16
    dY = rng.standard_normal((M, N)).astype(np.float32)
    X = rng.standard_normal((M, K)).astype(np.float32)
    G = (dY.T.astype(np.float64) @ X.astype(np.float64)).astype(np.float32)   # dL/dW_hat
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    packed = rabit.alloc_packed(N, K, P=P)
    rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed, P=P)
    ga = torch.empty((P, N), device="cuda")
    gb = torch.empty((P, K), device="cuda")
    ws = rabit.alloc_scale_grads_workspace(N, K, P)
    rabit.rabit_scale_grads(torch.from_numpy(G).cuda(), packed, at, bt, N, K, ga, gb, ws, P=P)
    torch.cuda.synchronize()
    S = oracle.derive_signs(W, a, b, P=P)
    ref_a, ref_b = oracle.scale_grads(G, S, a, b)
    assert normwise(ga.cpu().numpy().astype(np.float64), ref_a) <= TOL
    assert normwise(gb.cpu().numpy().astype(np.float64), ref_b) <= TOL


def test_scale_grads_pitched_g_and_repeatability():
    N, K, P = 130, 700, 2
    W = inputs.weight(61, N, K)
    a, b = inputs.scales(61, W)
    G = np.random.default_rng(61).standard_normal((N, K)).astype(np.float32)
    Gp = torch.zeros((N, K + 37), device="cuda")
    Gp[:, :K] = torch.from_numpy(G).cuda()
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    packed = rabit.alloc_packed(N, K)
    rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed)
    ws = rabit.alloc_scale_grads_workspace(N, K, P)
    outs = []
    for _ in range(2):
        ga, gb = torch.empty((P, N), device="cuda"), torch.empty((P, K), device="cuda")
        rabit.rabit_scale_grads(Gp[:, :K], packed, at, bt, N, K, ga, gb, ws)
        outs.append((ga.cpu().numpy(), gb.cpu().numpy()))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])      # fixed summation order
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    ref_a, ref_b = oracle.scale_grads(G, oracle.derive_signs(W, a, b), a, b)
    assert normwise(outs[0][0].astype(np.float64), ref_a) <= TOL
    assert normwise(outs[0][1].astype(np.float64), ref_b) <= TOL
