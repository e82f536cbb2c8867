"""GPU parity of the three-path (3-bit) variant against the float64 oracle.

S3 = sign(W - W_hat_1 - W_hat_2) (RaBiT paper sec. 4.1 stacking with the sec. 4.2 residual
rule), packed three words plus a zero padding word per group (Appendix E.1 "Weight
Packing").  Packing is bit-exact; GEMV and GEMM outputs are within the normwise tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu
TOL_BF16, TOL_F32 = 2e-3, 1e-5


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


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def layer3(seed, N, K, w_bf16=False):
    W = inputs.weight(seed, N, K, outlier_frac=0.001)
    a, b = inputs.scales(seed, W, P=3)
    if w_bf16:
        Wb = inputs.bf16_bits(W)
        Wdev = torch.from_numpy(Wb.view(np.int16)).view(torch.bfloat16).cuda()
        Wref = Wb
    else:
        Wdev = torch.from_numpy(W).cuda()
        Wref = W
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    packed = rabit.alloc_packed(N, K, P=3)
    packed.view(torch.int32).fill_(-0x5A5A5A5B)  # 0xA5A5A5A5: every word, padding included, must be written
    rabit.rabit_derive_pack(Wdev, at, bt, packed, P=3)
    torch.cuda.synchronize()
    S = oracle.derive_signs(Wref, a, b, P=3)
    return S, a, b, at, bt, packed


@pytest.fixture(params=["tc", "dp2a"])
def gemv_kernel(request, monkeypatch):
    """Both decode implementations (rabit_gemv picks one by batch; the environment forces it)."""
    monkeypatch.setenv("RABIT_GEMV_KERNEL", request.param)
    return request.param


@pytest.mark.parametrize("N,K,w_bf16", [(33, 129, False), (300, 520, True), (1024, 4096, False)])
def test_derive_pack_three_paths_bit_exact(N, K, w_bf16):
    S, a, b, at, bt, packed = layer3(80 + N, N, K, w_bf16)
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack(S))


@pytest.mark.parametrize("N,K,batch", [(33, 129, 1), (300, 520, 3), (1024, 4096, 1), (4096, 4096, 4)])
def test_gemv_three_paths_bf16(N, K, batch, gemv_kernel):
    S, a, b, at, bt, packed = layer3(81 + N, N, K)
    x = inputs.activations(81 + N, batch, K)
    y = torch.empty((batch, N), device="cuda")
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    rabit.rabit_gemv(packed, at, bt, N, K, xt, y, P=3)
    torch.cuda.synchronize()
    assert normwise(y.cpu().numpy().astype(np.float64), oracle.layer(S, a, b, x)) <= TOL_BF16


@pytest.mark.parametrize("N,K,batch", [(33, 129, 1), (300, 520, 5)])
def test_gemv_three_paths_fp32(N, K, batch, gemv_kernel):
    S, a, b, at, bt, packed = layer3(82 + N, N, K)
    x = inputs.activations(82 + N, batch, K, dtype="f32")
    y = torch.empty((batch, N), device="cuda")
    rabit.rabit_gemv(packed, at, bt, N, K, torch.from_numpy(x).cuda(), y, P=3)
    torch.cuda.synchronize()
    assert normwise(y.cpu().numpy().astype(np.float64), oracle.layer(S, a, b, x)) <= TOL_F32


@pytest.mark.parametrize("N,K,M", [(200, 520, 96), (512, 1024, 300)])
def test_gemm_three_paths(N, K, M):
    S, a, b, at, bt, packed = layer3(83 + N, N, K)
    x = inputs.activations(83 + N, M, K, channel_outlier_frac=0.01)
    ldx = ((K + 7) // 8) * 8
    xpad = torch.zeros((M, ldx), dtype=torch.bfloat16, device="cuda")
    xpad[:, :K] = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    y = torch.empty((M, N), device="cuda")
    rabit.rabit_gemm(packed, at, bt, N, K, xpad[:, :K], y, rabit.alloc_gemm_workspace(N, K, 3, M), P=3)
    torch.cuda.synchronize()
    assert normwise(y.cpu().numpy().astype(np.float64), oracle.layer(S, a, b, x)) <= TOL_BF16
