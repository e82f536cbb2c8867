"""GPU parity of the grouped GEMM (rabit_gemm_grouped) against the float64 oracle: several
layers with the same token count in one launch, each within the GEMM's bar (normwise
<= 2e-3), including the Llama-3-8B MLP prefill set at M = 2048 (sampled rows)."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from bit_gemv_rabit_b200 import build
    build.build()
    oracle.build()
    rabit.load()
    rabit.rabit_read_fault(clear=True)
    yield
    assert rabit.rabit_read_fault(clear=True) == 0


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def bf16_dev(bits):
    M, K = bits.shape
    padded = np.zeros((M, (K + 7) // 8 * 8), np.uint16)
    padded[:, :K] = bits
    return torch.from_numpy(padded.view(np.int16)).view(torch.bfloat16).cuda()[:, :K]


def sample_rows(N, seed, count=24):
    rng = np.random.default_rng(seed)
    return np.array(sorted(set(rng.choice(N, size=min(count, N), replace=False).tolist()) | {0, N - 1}), np.int64)


@pytest.mark.parametrize("P", [2, 3])
@pytest.mark.parametrize("M", [300, 1024])
def test_grouped_gemm_mixed_shapes(M, P):
    shapes = [(300, 520), (1024, 4096), (77, 256), (640, 1000)]
    layers, refs = [], []
    for i, (N, K) in enumerate(shapes):
        W = inputs.weight(800 + i, N, K)
        a, b = inputs.scales(800 + i, W, P=P)
        S = oracle.derive_signs(W, a, b, P=P)
        x = inputs.activations(810 + i, M, K, channel_outlier_frac=0.01)
        y = torch.full((M, N), float("nan"), device="cuda")
        layers.append((torch.from_numpy(oracle.pack(S)).cuda(), torch.from_numpy(a).cuda(),
                       torch.from_numpy(b).cuda(), N, K, bf16_dev(x), y))
        refs.append(oracle.layer(S, a, b, x))
    ws = rabit.alloc_gemm_grouped_workspace(layers, P)
    rabit.rabit_gemm_grouped(layers, ws, P=P)
    torch.cuda.synchronize()
    for L, ref in zip(layers, refs):
        assert normwise(L[6].cpu().numpy().astype(np.float64), ref) <= TOL, (L[3], L[4])


@pytest.mark.slow
def test_grouped_gemm_llama3_8b_mlp_prefill_full_size():
    spec = inputs.WORKLOADS["llama3_8b_mlp_prefill_m2048"]
    M = spec["batches"][0]
    layers, checks = [], []
    for idx, (name, N, K) in enumerate(spec["set"]):
        seed = inputs.seed_for(spec["cfg"], idx)
        W = inputs.weight(seed, N, K, sigma=spec["sigma"], outlier_frac=spec["w_outliers"])
        a, b = inputs.scales(seed, W)
        at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
        packed = rabit.alloc_packed(N, K)
        rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed)
        x = inputs.activations(seed, M, K, channel_outlier_frac=spec["x_outliers"])
        rows = sample_rows(N, seed)
        S_rows = np.concatenate([oracle.derive_signs(W, a, b, rows=(int(r), int(r) + 1)) for r in rows], axis=1)
        y = torch.empty((M, N), device="cuda")
        layers.append((packed, at, bt, N, K, bf16_dev(x), y))
        checks.append((name, rows, oracle.layer(S_rows, a, b, x, rows=rows, N=N)))
    ws = rabit.alloc_gemm_grouped_workspace(layers)
    rabit.rabit_gemm_grouped(layers, ws)
    torch.cuda.synchronize()
    for L, (name, rows, ref) in zip(layers, checks):
        assert normwise(L[6].cpu().numpy()[:, rows].astype(np.float64), ref) <= TOL, name
