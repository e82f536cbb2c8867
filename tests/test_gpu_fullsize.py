"""GPU parity at the full workload sizes, in the launch configurations the benchmark times.

The whole matrix goes through the CUDA path; the oracle checks a seeded sample of rows
(first, last and random ones) one by one: their packed words bit-exactly, their outputs
within the normwise tolerance.  Workloads: the Llama-2-7B decode layer set (batch 1), the
Llama-3-8B decode set with outliers (batch 1/4/8/16), the Llama-3-8B MLP prefill GEMM at
M=2048 and the Llama-3-70B MLP QAT step (derive + GEMM at M=4096).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

TOL = 2e-3


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def sample_rows(N, seed, count=48):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(count, N), replace=False).tolist()) | {0, N - 1}
    return np.array(sorted(rows), dtype=np.int64)


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


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


def derive_and_check(W, a, b, rows, P=2):
    """GPU derive of the whole W; bit-exact check of the sampled rows; returns (packed, S_rows)."""
    N, K = W.shape
    packed = rabit.alloc_packed(N, K, P=P)
    rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), torch.from_numpy(a).cuda(),
                            torch.from_numpy(b).cuda(), packed, P=P)
    torch.cuda.synchronize()
    per_row = oracle.packed_words(1, K, P)
    host = packed.cpu().numpy().reshape(N, per_row)
    S_rows = np.concatenate([oracle.derive_signs(W, a, b, P=P, rows=(int(r), int(r) + 1)) for r in rows], axis=1)
    np.testing.assert_array_equal(host[rows], oracle.pack(S_rows).reshape(len(rows), per_row))
    return packed, S_rows


@pytest.fixture(params=["tc", "dp2a"])
def gemv_kernel(request, monkeypatch):
    """Both decode implementations (rabit_gemv picks one by batch; the environment forces it)."""
    monkeypatch.setenv("RABIT_GEMV_KERNEL", request.param)
    return request.param


def decode_set(workload):
    spec = inputs.WORKLOADS[workload]
    for idx, (name, N, K) in enumerate(spec["set"]):
        seed = inputs.seed_for(spec["cfg"], idx)
        W = inputs.weight(seed, N, K, sigma=spec["sigma"], outlier_frac=spec["w_outliers"])
        a, b = inputs.scales(seed, W)
        yield name, N, K, seed, W, a, b, spec


@pytest.mark.parametrize("workload", ["single_4096x4096_b1", "llama2_7b_decode_b1", "llama3_8b_decode"])
def test_decode_sets_full_size(workload, gemv_kernel):
    for name, N, K, seed, W, a, b, spec in decode_set(workload):
        rows = sample_rows(N, seed)
        packed, S_rows = derive_and_check(W, a, b, rows)
        at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
        for B in spec["batches"]:
            x = inputs.activations(seed, B, K, channel_outlier_frac=spec["x_outliers"])
            y = torch.empty((B, N), device="cuda")
            rabit.rabit_gemv(packed, at, bt, N, K, bf16_dev(x), y)
            torch.cuda.synchronize()
            ref = oracle.layer(S_rows, a, b, x, rows=rows, N=N)
            err = normwise(y.cpu().numpy()[:, rows].astype(np.float64), ref)
            assert err <= TOL, (name, B, err)


@pytest.mark.parametrize("workload", ["llama3_8b_mlp_prefill_m2048", "llama3_70b_mlp_qat_m4096"])
def test_gemm_workloads_full_size(workload):
    for name, N, K, seed, W, a, b, spec in decode_set(workload):
        rows = sample_rows(N, seed, count=16)
        packed, S_rows = derive_and_check(W, a, b, rows)
        M = spec["batches"][0]
        x = inputs.activations(seed, M, K, channel_outlier_frac=spec["x_outliers"])
        y = torch.empty((M, N), device="cuda")
        ws = rabit.alloc_gemm_workspace(N, K, 2, M)
        rabit.rabit_gemm(packed, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), N, K,
                         bf16_dev(x), y, ws)
        torch.cuda.synchronize()
        ref = oracle.layer(S_rows, a, b, x, rows=rows, N=N)
        err = normwise(y.cpu().numpy()[:, rows].astype(np.float64), ref)
        assert err <= TOL, (name, err)


def test_three_path_decode_set_full_size(gemv_kernel):
    """The 3-bit variant on the Llama-2-7B decode set at batch 1 (sampled rows)."""
    spec = inputs.WORKLOADS["llama2_7b_decode_b1"]
    for idx, (name, N, K) in enumerate(spec["set"]):
        seed = inputs.seed_for(spec["cfg"], idx)
        W = inputs.weight(seed, N, K, sigma=spec["sigma"])
        a, b = inputs.scales(seed, W, P=3)
        rows = sample_rows(N, seed, count=24)
        packed = rabit.alloc_packed(N, K, P=3)
        at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
        rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed, P=3)
        x = inputs.activations(seed, 1, K)
        y = torch.empty((1, N), device="cuda")
        rabit.rabit_gemv(packed, at, bt, N, K, bf16_dev(x), y, P=3)
        torch.cuda.synchronize()
        per_row = oracle.packed_words(1, K, 3)
        S_rows = np.concatenate([oracle.derive_signs(W, a, b, P=3, rows=(int(r), int(r) + 1)) for r in rows], axis=1)
        np.testing.assert_array_equal(packed.cpu().numpy().reshape(N, per_row)[rows],
                                      oracle.pack(S_rows).reshape(len(rows), per_row))
        ref = oracle.layer(S_rows, a, b, x, rows=rows, N=N)
        assert normwise(y.cpu().numpy()[:, rows].astype(np.float64), ref) <= TOL, name


@pytest.mark.parametrize("xdtype,B", [("bf16", 3), ("f32", 5)])
def test_gemv_several_passes_and_batch_rows(xdtype, B, gemv_kernel):
    """28672 x 8192 leaves each CTA of the CUDA-core kernel 194 rows of 2 KiB: more than its
    shared memory holds, so the rows go through several passes, each reused by the batch rows
    (sampled rows); fp32 x at batch 5 as well."""
    N, K = 28672, 8192
    seed = 777
    W = inputs.weight(seed, N, K, sigma=0.015)
    a, b = inputs.scales(seed, W)
    rows = sample_rows(N, seed, count=24)
    packed, S_rows = derive_and_check(W, a, b, rows)
    if xdtype == "f32":
        x = inputs.activations(seed, B, K, dtype="f32")
        xt = torch.from_numpy(x).cuda()
    else:
        x = inputs.activations(seed, B, K)
        xt = bf16_dev(x)
    y = torch.empty((B, N), device="cuda")
    rabit.rabit_gemv(packed, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), N, K, xt, y)
    torch.cuda.synchronize()
    ref = oracle.layer(S_rows, a, b, x, rows=rows, N=N)
    assert normwise(y.cpu().numpy()[:, rows].astype(np.float64), ref) <= (1e-5 if xdtype == "f32" else TOL)


@pytest.mark.parametrize("N,K", [(4096, 11008), (4096, 14336)])
def test_gemv_fp32_down_projections_batch5(N, K, gemv_kernel):
    """fp32 activations at batch 5 on the down-projection shapes of the decode sets (outliers
    in W), sampled rows, normwise <= 1e-5."""
    seed = 880 + K
    W = inputs.weight(seed, N, K, sigma=0.02, outlier_frac=0.001)
    a, b = inputs.scales(seed, W)
    rows = sample_rows(N, seed)
    packed, S_rows = derive_and_check(W, a, b, rows)
    x = inputs.activations(seed, 5, K, dtype="f32")
    y = torch.empty((5, N), device="cuda")
    rabit.rabit_gemv(packed, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), N, K,
                     torch.from_numpy(x).cuda(), y)
    torch.cuda.synchronize()
    ref = oracle.layer(S_rows, a, b, x, rows=rows, N=N)
    assert normwise(y.cpu().numpy()[:, rows].astype(np.float64), ref) <= 1e-5


@pytest.mark.parametrize("B", [4, 16])
def test_three_path_llama3_decode_full_size(B, gemv_kernel):
    """The 3-bit variant on the Llama-3-8B decode shapes at batch 4 and 16 (sampled rows)."""
    spec = inputs.WORKLOADS["llama3_8b_decode"]
    for idx, (name, N, K) in enumerate(spec["set"]):
        seed = inputs.seed_for(spec["cfg"], idx)
        W = inputs.weight(seed, N, K, sigma=spec["sigma"], outlier_frac=spec["w_outliers"])
        a, b = inputs.scales(seed, W, P=3)
        rows = sample_rows(N, seed, count=16)
        packed, S_rows = derive_and_check(W, a, b, rows, P=3)
        x = inputs.activations(seed, B, K)
        y = torch.empty((B, N), device="cuda")
        rabit.rabit_gemv(packed, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), N, K, bf16_dev(x), y, P=3)
        torch.cuda.synchronize()
        ref = oracle.layer(S_rows, a, b, x, rows=rows, N=N)
        assert normwise(y.cpu().numpy()[:, rows].astype(np.float64), ref) <= TOL, (name, B)


@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_three_path_gemm_prefill_full_size(N, K):
    """3-path GEMM on the Llama-3-8B MLP prefill shapes at M = 2048 (sampled rows)."""
    spec = inputs.WORKLOADS["llama3_8b_mlp_prefill_m2048"]
    seed = 990 + N
    W = inputs.weight(seed, N, K, sigma=spec["sigma"])
    a, b = inputs.scales(seed, W, P=3)
    rows = sample_rows(N, seed, count=16)
    packed, S_rows = derive_and_check(W, a, b, rows, P=3)
    M = spec["batches"][0]
    x = inputs.activations(seed, M, K, channel_outlier_frac=spec["x_outliers"])
    y = torch.empty((M, N), device="cuda")
    ws = rabit.alloc_gemm_workspace(N, K, 3, M)
    rabit.rabit_gemm(packed, torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda(), N, K, bf16_dev(x), y, ws, P=3)
    torch.cuda.synchronize()
    ref = oracle.layer(S_rows, a, b, x, rows=rows, N=N)
    assert normwise(y.cpu().numpy()[:, rows].astype(np.float64), ref) <= TOL
