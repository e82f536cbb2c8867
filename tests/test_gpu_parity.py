"""GPU parity: the CUDA path, called through the C ABI, against the float64 oracle.

  * packing: bit-exact, padding included, with canary guard words around the output;
  * gemv: normwise error max|y - y_ref| / max|y_ref| <= 2e-3 (bf16 x) and <= 1e-5 (fp32 x);
  * gemm: normwise error <= 2e-3;
on the same seeded inputs (bit_gemv_rabit_b200.inputs), at sizes that span several tiles and
a ragged tail, plus sampled rows at the full workload sizes.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-3
TOL_F32 = 1e-5
CANARY = 0xDEADBEEF
GUARD = 64  # guard words on each side (256 B keeps the payload 16-byte aligned)


def normwise(y, ref):
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.cuda() if dtype is None else t.to(dtype).cuda()


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def guarded_words(n):
    buf = torch.full((n + 2 * GUARD,), CANARY, dtype=torch.int64).to(torch.uint32).cuda()
    return buf, buf[GUARD:GUARD + n]


def check_guards(buf, n):
    h = buf.cpu().numpy()
    assert np.all(h[:GUARD] == CANARY) and np.all(h[GUARD + n:] == CANARY), "write outside output"


def make_layer(seed, N, K, sigma=0.02, outliers=0.0):
    W = inputs.weight(seed, N, K, sigma=sigma, outlier_frac=outliers)
    a, b = inputs.scales(seed, W)
    return W, a, b


def gpu_derive(W, a, b, w_bf16=False, ldw=None):
    N, K = W.shape
    if w_bf16:
        Wh = inputs.bf16_bits(W)
    else:
        Wh = W
    if ldw is not None and ldw > K:
        pad = np.zeros((N, ldw), dtype=Wh.dtype)
        pad[:, :K] = Wh
        Wt = bf16_dev(pad) if w_bf16 else dev(pad)
        Wt = Wt[:, :K]
    else:
        Wt = bf16_dev(Wh) if w_bf16 else dev(Wh)
    nw = rabit.rabit_packed_words(N, K)
    buf, packed = guarded_words(nw)
    rabit.rabit_derive_pack(Wt, dev(a), dev(b), packed)
    torch.cuda.synchronize()
    check_guards(buf, nw)
    return packed.cpu().numpy(), (Wh if w_bf16 else W)


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


# ------------------------------------------------------------------ derive + pack
DERIVE_SHAPES = [(1, 1), (8, 16), (31, 127), (33, 129), (70, 300), (256, 1024), (100, 4096)]


@pytest.mark.parametrize("N,K", DERIVE_SHAPES)
@pytest.mark.parametrize("w_bf16", [False, True])
def test_derive_pack_bit_exact(N, K, w_bf16):
    W, a, b = make_layer(100 + N + K, N, K, outliers=0.01)
    got, Wused = gpu_derive(W, a, b, w_bf16=w_bf16)
    ref = oracle.pack(oracle.derive_signs(Wused, a, b))
    np.testing.assert_array_equal(got, ref)


def test_derive_pack_pitched_weight():
    W, a, b = make_layer(7, 40, 200)
    got, _ = gpu_derive(W, a, b, ldw=264)
    np.testing.assert_array_equal(got, oracle.pack(oracle.derive_signs(W, a, b)))


def test_derive_pack_hand_cases(golden_dir):
    # The hand-derived 8 x 16 cases (+-0, exact ties, one-ulp near ties, subnormals, 3e38).
    from tests.test_oracle_pins import _golden_cases, _case_value
    a1, b1, cases = _golden_cases(golden_dir)
    N, K = 8, 16
    W = np.zeros((N, K), dtype=np.float32)
    e = np.zeros((2, N, K), dtype=np.int8)
    for n in range(N):
        for j in range(K):
            expr, s1, s2 = cases[(j + 3 * n) % 16]
            W[n, j] = _case_value(expr, a1[n] * b1[j])
            e[0, n, j], e[1, n, j] = s1, s2
    a = np.stack([a1, np.ones(N, np.float32)])
    b = np.stack([b1, np.ones(K, np.float32)])
    got, _ = gpu_derive(W, a, b)
    np.testing.assert_array_equal(oracle.unpack(got, N, K), e)


# ------------------------------------------------------------------ gemv
@pytest.fixture(params=["tc", "dp2a"])
def gemv_kernel(request, monkeypatch):
    """Both decode implementations: rabit_gemv picks one by batch; the environment forces it."""
    monkeypatch.setenv("RABIT_GEMV_KERNEL", request.param)
    return request.param


GEMV_SHAPES = [(1, 1), (32, 128), (33, 129), (96, 1000), (300, 520), (1024, 4096)]


@pytest.mark.parametrize("N,K", GEMV_SHAPES)
@pytest.mark.parametrize("batch", [1, 2, 3, 8, 16])
def test_gemv_bf16_matches_oracle(N, K, batch, gemv_kernel):
    W, a, b = make_layer(200 + N, N, K)
    S = oracle.derive_signs(W, a, b)
    packed = dev(oracle.pack(S))
    x = inputs.activations(200 + K, batch, K)
    y = torch.full((batch, N), float("nan"), device="cuda")
    rabit.rabit_gemv(packed, dev(a), dev(b), N, K, bf16_dev(x), y)
    torch.cuda.synchronize()
    ref = oracle.layer(S, a, b, x)
    assert normwise(y.cpu().numpy().astype(np.float64), ref) <= TOL_BF16


@pytest.mark.parametrize("N,K", [(33, 129), (300, 520), (1024, 4096)])
@pytest.mark.parametrize("batch", [1, 5])
def test_gemv_fp32_matches_oracle(N, K, batch, gemv_kernel):
    W, a, b = make_layer(300 + N, N, K)
    S = oracle.derive_signs(W, a, b)
    packed = dev(oracle.pack(S))
    x = inputs.activations(300 + K, batch, K, dtype="f32")
    y = torch.empty((batch, N), device="cuda")
    rabit.rabit_gemv(packed, dev(a), dev(b), N, K, dev(x), y)
    torch.cuda.synchronize()
    ref = oracle.layer(S, a, b, x)
    assert normwise(y.cpu().numpy().astype(np.float64), ref) <= TOL_F32


@pytest.mark.parametrize("P", [2, 3])
@pytest.mark.parametrize("N,K,batch", [(300, 520, 2), (300, 520, 7), (1024, 4096, 4), (4096, 4096, 6),
                                       (1000, 1000, 16)])
def test_gemv_each_batch_row_matches_oracle(N, K, batch, P, gemv_kernel):
    """Batch rows of magnitudes 2^-6 .. 2^+6 apart: every row is checked on its own, so a row
    scaled with another row's z scale, or left unwritten, fails."""
    W, a, b = make_layer(400 + N + batch, N, K)
    a3, b3 = inputs.scales(400 + N, W, P=P)
    S = oracle.derive_signs(W, a3, b3, P=P)
    x = inputs.activations(401 + K, batch, K)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    xf = xf * np.float32(2.0) ** np.array([(3 * beta) % 13 - 6 for beta in range(batch)],
                                          np.float32)[:, None]
    xb = (xf.view(np.uint32) >> 16).astype(np.uint16)      # power-of-two scaling is exact in bf16
    y = torch.full((batch, N), float("nan"), device="cuda")
    rabit.rabit_gemv(dev(oracle.pack(S)), dev(a3), dev(b3), N, K, bf16_dev(xb), y, P=P)
    torch.cuda.synchronize()
    ref = oracle.layer(S, a3, b3, xb)
    yh = y.cpu().numpy().astype(np.float64)
    for beta in range(batch):
        assert normwise(yh[beta], ref[beta]) <= TOL_BF16, beta


def test_gemv_pitched_io(gemv_kernel):
    N, K, batch = 70, 300, 4
    W, a, b = make_layer(9, N, K)
    S = oracle.derive_signs(W, a, b)
    x = inputs.activations(9, batch, K)
    xpad = np.zeros((batch, K + 40), np.uint16)
    xpad[:, :K] = x
    xt = bf16_dev(xpad)[:, :K]
    yt = torch.full((batch, N + 17), 7.0, device="cuda")
    rabit.rabit_gemv(dev(oracle.pack(S)), dev(a), dev(b), N, K, xt, yt[:, :N])
    torch.cuda.synchronize()
    yh = yt.cpu().numpy()
    assert np.all(yh[:, N:] == 7.0)
    assert normwise(yh[:, :N].astype(np.float64), oracle.layer(S, a, b, x)) <= TOL_BF16


def test_derive_then_gemv_end_to_end():
    N, K = 520, 1000
    W, a, b = make_layer(11, N, K, outliers=0.001)
    Wt = dev(W)
    packed = rabit.alloc_packed(N, K)
    rabit.rabit_derive_pack(Wt, dev(a), dev(b), packed)
    x = inputs.activations(11, 2, K)
    y = torch.empty((2, N), device="cuda")
    rabit.rabit_gemv(packed, dev(a), dev(b), N, K, bf16_dev(x), y)
    torch.cuda.synchronize()
    ref = oracle.layer(oracle.derive_signs(W, a, b), a, b, x)
    assert normwise(y.cpu().numpy().astype(np.float64), ref) <= TOL_BF16


# ------------------------------------------------------------------ gemm
GEMM_SHAPES = [(128, 64, 1), (128, 128, 256), (200, 200, 300), (256, 512, 512), (384, 1024, 100),
               (1000, 700, 777)]


@pytest.mark.parametrize("N,K,M", GEMM_SHAPES)
def test_gemm_matches_oracle(N, K, M):
    W, a, b = make_layer(400 + N + K, N, K)
    S = oracle.derive_signs(W, a, b)
    packed = dev(oracle.pack(S))
    x = inputs.activations(400 + M, M, K, channel_outlier_frac=0.01)
    ldx = ((K + 7) // 8) * 8
    xpad = np.zeros((M, ldx), np.uint16)
    xpad[:, :K] = x
    xt = bf16_dev(xpad)
    y = torch.full((M, N), float("nan"), device="cuda")
    ws = rabit.alloc_gemm_workspace(N, K, 2, M)
    rabit.rabit_gemm(packed, dev(a), dev(b), N, K, xt[:, :K], y, ws)
    torch.cuda.synchronize()
    ref = oracle.layer(S, a, b, x)
    err = normwise(y.cpu().numpy().astype(np.float64), ref)
    assert err <= TOL_BF16, err


def test_gemm_more_tiles_than_sms_matches_oracle():
    # 16 x 10 = 160 tiles on a 148-SM part: a second, partial round of the persistent tile
    # loop; every output is compared.
    N, K, M = 2048, 512, 2560
    W = inputs.weight(171, N, K)
    a, b = inputs.scales(171, W)
    x = inputs.activations(171, M, K, channel_outlier_frac=0.01)
    at, bt = dev(a), dev(b)
    packed = rabit.alloc_packed(N, K)
    rabit.rabit_derive_pack(dev(W), at, bt, packed)
    y = torch.full((M, N), float("nan"), device="cuda")
    rabit.rabit_gemm(packed, at, bt, N, K, bf16_dev(x), y, rabit.alloc_gemm_workspace(N, K, 2, M))
    torch.cuda.synchronize()
    ref = oracle.layer(oracle.derive_signs(W, a, b), a, b, x)
    assert normwise(y.cpu().numpy().astype(np.float64), ref) <= TOL_BF16


def test_gemm_matches_gemv_bitwise_inputs():
    # The two decode/prefill paths compute the same layer: compare them on one input.
    N, K, M = 256, 1024, 16
    W, a, b = make_layer(17, N, K)
    packed = rabit.alloc_packed(N, K)
    rabit.rabit_derive_pack(dev(W), dev(a), dev(b), packed)
    x = bf16_dev(inputs.activations(17, M, K))
    y1 = torch.empty((M, N), device="cuda")
    y2 = torch.empty((M, N), device="cuda")
    rabit.rabit_gemv(packed, dev(a), dev(b), N, K, x, y1)
    rabit.rabit_gemm(packed, dev(a), dev(b), N, K, x, y2, rabit.alloc_gemm_workspace(N, K, 2, M))
    torch.cuda.synchronize()
    assert normwise(y2.cpu().numpy().astype(np.float64), y1.cpu().numpy().astype(np.float64)) <= TOL_BF16


# ------------------------------------------------------------------ error paths on a GPU
def test_arch_mismatch_hook(monkeypatch):
    monkeypatch.setenv("RABIT_TEST_FORCE_ARCH_MISMATCH", "1")
    with pytest.raises(rabit.RabitError) as e:
        rabit.rabit_derive_pack(torch.zeros(4, 4, device="cuda"), torch.ones(2, 4, device="cuda"),
                                torch.ones(2, 4, device="cuda"), rabit.alloc_packed(4, 4))
    assert e.value.status == -6
