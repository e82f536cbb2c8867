"""GPU parity of the input gradient (the backward of sec. 4.1's stacked layer, signs held
fixed) against the float64 oracle:

  * rabit_transpose_pack: bit-exact against the oracle's packing of S_k^T, canary words
    around the output;
  * rabit_grad_x: normwise <= 2e-3 (the GEMM's bar), on small shapes that span several
    tiles and a ragged tail, and on the Llama-3-70B MLP QAT shape at M = 4096 (sampled
    columns and tokens).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu

TOL = 2e-3
CANARY = 0xDEADBEEF
GUARD = 64


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
    """bf16 rows with a pitch rounded up to 8 elements (the GEMM reads 16-byte rows)."""
    M, N = bits.shape
    padded = np.zeros((M, (N + 7) // 8 * 8), np.uint16)
    padded[:, :N] = bits
    return torch.from_numpy(padded.view(np.int16)).view(torch.bfloat16).cuda()[:, :N]


def layer(seed, N, K, P):
    W = inputs.weight(seed, N, K)
    a, b = inputs.scales(seed, W, P=P)
    return W, a, b


@pytest.mark.parametrize("P", [2, 3])
@pytest.mark.parametrize("N,K", [(1, 1), (33, 129), (300, 520), (257, 4097), (1024, 256)])
def test_transpose_pack_bit_exact(N, K, P):
    W, a, b = layer(500 + N + K, N, K, P)
    S = oracle.derive_signs(W, a, b, P=P)
    packed = torch.from_numpy(oracle.pack(S)).cuda()
    words = oracle.packed_words(K, N, P)
    buf = torch.full((words + 2 * GUARD,), CANARY, dtype=torch.int64).to(torch.uint32).cuda()
    out = buf[GUARD:GUARD + words]
    rabit.rabit_transpose_pack(packed, N, K, out, P=P)
    torch.cuda.synchronize()
    host = buf.cpu().numpy()
    assert np.all(host[:GUARD] == CANARY) and np.all(host[GUARD + words:] == CANARY)
    np.testing.assert_array_equal(host[GUARD:GUARD + words], oracle.pack(np.ascontiguousarray(S.transpose(0, 2, 1))))


@pytest.mark.parametrize("P", [2, 3])
@pytest.mark.parametrize("N,K,M", [(300, 520, 96), (1024, 4096, 300), (520, 300, 2048)])
def test_grad_x_matches_oracle(N, K, M, P):
    W, a, b = layer(600 + N, N, K, P)
    S = oracle.derive_signs(W, a, b, P=P)
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    packed = torch.from_numpy(oracle.pack(S)).cuda()
    packed_t = rabit.alloc_packed(K, N, P=P)
    rabit.rabit_transpose_pack(packed, N, K, packed_t, P=P)
    dy = inputs.activations(601 + K, M, N)
    gx = torch.full((M, K), float("nan"), device="cuda")
    ws = rabit.alloc_gemm_workspace(K, N, P, M)
    rabit.rabit_grad_x(packed_t, at, bt, N, K, bf16_dev(dy), gx, ws, P=P)
    torch.cuda.synchronize()
    ref = oracle.grad_x(S, a, b, dy)
    assert normwise(gx.cpu().numpy().astype(np.float64), ref) <= TOL


@pytest.mark.slow
def test_grad_x_llama3_70b_mlp_full_size():
    """28672 x 8192 layer (the QAT step's shape), M = 4096 tokens: derive, transpose and
    grad_x on the GPU for the whole layer; the oracle checks 16 columns (their transposed
    packed rows bit-exactly) for 64 sampled tokens."""
    spec = inputs.WORKLOADS["llama3_70b_mlp_qat_m4096"]
    _, N, K = spec["set"][0]
    M = spec["batches"][0]
    seed = inputs.seed_for(spec["cfg"], 0) + 7
    W = inputs.weight(seed, N, K, sigma=spec["sigma"])
    a, b = inputs.scales(seed, W)
    at, bt = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    packed = rabit.alloc_packed(N, K)
    rabit.rabit_derive_pack(torch.from_numpy(W).cuda(), at, bt, packed)
    packed_t = rabit.alloc_packed(K, N)
    rabit.rabit_transpose_pack(packed, N, K, packed_t)
    dy = inputs.activations(seed, M, N)
    gx = torch.empty((M, K), device="cuda")
    ws = rabit.alloc_gemm_workspace(K, N, 2, M)
    rabit.rabit_grad_x(packed_t, at, bt, N, K, bf16_dev(dy), gx, ws)
    torch.cuda.synchronize()
    rng = np.random.default_rng(seed)
    cols = np.array(sorted(set(rng.choice(K, 14, replace=False).tolist()) | {0, K - 1}), dtype=np.int64)
    toks = np.array(sorted(set(rng.choice(M, 62, replace=False).tolist()) | {0, M - 1}), dtype=np.int64)
    # signs of the sampled columns for every row, derived by the oracle in row blocks
    Sc = np.concatenate([oracle.derive_signs(W, a, b, rows=(r0, min(N, r0 + 2048)))[:, :, cols]
                         for r0 in range(0, N, 2048)], axis=1)
    per_row = oracle.packed_words(1, N)
    host_t = packed_t.cpu().numpy().reshape(K, per_row)
    np.testing.assert_array_equal(host_t[cols], oracle.pack(np.ascontiguousarray(Sc.transpose(0, 2, 1))).reshape(len(cols), per_row))
    ref = oracle.grad_x(Sc, a, b, dy[toks], cols=cols)
    got = gx.cpu().numpy()[np.ix_(toks, cols)].astype(np.float64)
    assert normwise(got, ref) <= TOL
