"""rabit_gemm_noalloc: the GEMM for callers that may not allocate device memory.

Some callers cannot give rabit_gemm a workspace because they are not allowed to allocate:
a plugin inside an engine that owns all device memory and exposes no allocator, or a
serving loop that must never call cudaMalloc (it can synchronise the device and is illegal
while a stream is being captured in global mode).  rabit_gemm_noalloc takes its scratch from
a fixed buffer inside the library instead.  These tests call it through the C ABI and check
two calls in a row against the float64 oracle and against rabit_gemm on the same inputs,
with two and three paths.

This file is named so that pytest collects it last; it also passes when run on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu

TOL = 2e-3
SCRATCH_LIMIT = 8 << 20   # RABIT_GEMM_NOALLOC_SCRATCH_BYTES in include/rabit.h


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from bit_gemv_rabit_b200 import build
    build.build()
    oracle.build()
    return rabit.load()


def _call_noalloc(lib, packed, a, b, N, K, x, y, P=2):
    st = lib.rabit_gemm_noalloc(ctypes.c_void_p(packed.data_ptr()), ctypes.c_void_p(a.data_ptr()),
                                ctypes.c_void_p(b.data_ptr()), N, K, P, ctypes.c_void_p(x.data_ptr()),
                                x.shape[0], x.stride(0), ctypes.c_void_p(y.data_ptr()), y.stride(0),
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, rabit.STATUS.get(st, st)


# (N, K, M, P): a ragged shape; a two-path shape whose scratch is exactly the buffer size;
# a three-path shape at the largest token count that fits (3 * M * Kp * 2 bytes cannot equal
# 8 MiB exactly, so M = 341 at Kp = 4096 uses 8,380,416 of its 8,388,608 bytes).
@pytest.mark.parametrize("N,K,M,P", [(300, 1000, 200, 2), (256, 4096, 512, 2), (160, 4096, 341, 3)])
def test_noalloc_matches_oracle_and_workspace_gemm_two_calls(lib, N, K, M, P):
    assert rabit.rabit_gemm_workspace_bytes(N, K, P, M) <= SCRATCH_LIMIT
    W = inputs.weight(900 + N, N, K)
    a, b = inputs.scales(900 + N, W, P=P)
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    packed = rabit.alloc_packed(N, K, P=P)
    rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed, P=P)
    S = oracle.derive_signs(W, a, b, P=P)
    ldx = ((K + 7) // 8) * 8
    for call in range(2):
        x = np.zeros((M, ldx), np.uint16)
        x[:, :K] = inputs.activations(950 + call, M, K, channel_outlier_frac=0.01)
        xt = bf16_dev(x)[:, :K]
        y_ref = torch.empty((M, N), device="cuda")
        rabit.rabit_gemm(packed, at, bt, N, K, xt, y_ref, rabit.alloc_gemm_workspace(N, K, P, M), P=P)
        y = torch.full((M, N), float("nan"), device="cuda")
        _call_noalloc(lib, packed, at, bt, N, K, xt, y, P=P)
        torch.cuda.synchronize()
        y64 = y.cpu().numpy().astype(np.float64)
        exact = oracle.layer(S, a, b, x[:, :K])
        err_oracle = normwise(y64, exact)
        err_gemm = normwise(y64, y_ref.cpu().numpy().astype(np.float64))
        assert err_oracle <= TOL, (call, err_oracle)
        assert err_gemm <= TOL, (call, err_gemm)
    assert rabit.rabit_read_fault(clear=True) == 0


def test_noalloc_rejects_scratch_beyond_the_buffer(lib):
    N, K, M = 256, 4096, 513          # needs 2 * 513 * 4096 * 2 bytes > 8 MiB
    assert rabit.rabit_gemm_workspace_bytes(N, K, 2, M) > SCRATCH_LIMIT
    packed = rabit.alloc_packed(N, K)
    a = torch.ones(2, N, device="cuda")
    b = torch.ones(2, K, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, N), device="cuda")
    with pytest.raises(rabit.RabitError) as e:
        rabit.rabit_gemm_noalloc(packed, a, b, N, K, x, y)
    assert e.value.status == -5   # RABIT_ERR_WORKSPACE
    # three paths: one token more than the largest request that fits
    M3 = 342
    assert rabit.rabit_gemm_workspace_bytes(N, K, 3, M3) > SCRATCH_LIMIT
    packed3 = rabit.alloc_packed(N, K, P=3)
    a3, b3 = torch.ones(3, N, device="cuda"), torch.ones(3, K, device="cuda")
    with pytest.raises(rabit.RabitError) as e:
        rabit.rabit_gemm_noalloc(packed3, a3, b3, N, K, x[:M3], y[:M3], P=3)
    assert e.value.status == -5
