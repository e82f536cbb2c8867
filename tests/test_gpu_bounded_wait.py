"""A device wait that runs out is reported, not hung on.

Host-side test switches withhold one event a kernel waits for:
  - RABIT_TEST_SKIP_ONE_ARRIVE: the GEMM's expansion warps skip their first arrival;
  - RABIT_TEST_GEMV_WITHHOLD_COPY: the decode kernel's producer never issues its first copy;
  - RABIT_TEST_SCALE_GRADS_WITHHOLD_COPY: the scale-gradient producer never issues its first box;
  - RABIT_TEST_SVID_WITHHOLD_ARRIVAL: CTA 0 of each SVID power launch skips its first
    grid-barrier arrival.
The bounded wait that depends on it expires (after RABIT_WAIT_TIMEOUT_MS); the kernel drains
its in-flight copies, frees tensor memory and returns; the host reads RABIT_ERR_TIMEOUT with
that wait's fault bit, and the next call on the same context is correct.  No GPU fault is
involved: the failure is a missing event that a flag withholds.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import inputs
from bit_gemv_rabit_b200 import rabit

pytestmark = pytest.mark.gpu

# the GEMM's wait bits: TMA producer, MMA issuer, expansion, epilogue.  Every one of them
# ends up waiting on the withheld arrival; whichever runs out first records its bit and the
# others see the abort flag.
FAULT_GEMM_WAITS = (1 << 0) | (1 << 1) | (1 << 2) | (1 << 3)
# the decode kernel's waits: copies (producer, expansion) and the MMA issuer / epilogue /
# expansion-group barrier; the MMA issuer starts waiting first, so its bit is usually the one
FAULT_GEMV_WAITS = (1 << 5) | (1 << 6)
FAULT_SCALE_GRADS_WAIT = 1 << 7
FAULT_SVID_BARRIER = 1 << 8
RABIT_ERR_TIMEOUT = -8


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


def _case(N=256, K=512, M=256, seed=4242):
    W = inputs.weight(seed, N, K)
    a, b = inputs.scales(seed, W)
    x = inputs.activations(seed, M, K)
    dev = lambda v: torch.from_numpy(np.ascontiguousarray(v)).cuda()
    at, bt = dev(a), dev(b)
    packed = rabit.alloc_packed(N, K)
    rabit.rabit_derive_pack(dev(W), at, bt, packed)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return W, a, b, x, at, bt, packed, xt


def test_gemm_wait_expiry_is_reported_and_the_context_survives(monkeypatch):
    N, K, M = 256, 512, 256
    W, a, b, x, at, bt, packed, xt = _case(N, K, M)
    ws = rabit.alloc_gemm_workspace(N, K, 2, M)
    y = torch.zeros((M, N), device="cuda")
    monkeypatch.setenv("RABIT_TEST_SKIP_ONE_ARRIVE", "1")
    monkeypatch.setenv("RABIT_WAIT_TIMEOUT_MS", "50")
    rabit.rabit_gemm(packed, at, bt, N, K, xt, y, ws)
    flags = ctypes.c_uint32(0)
    st = rabit.load().rabit_read_fault(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                        ctypes.byref(flags), 1)
    assert st == RABIT_ERR_TIMEOUT
    assert flags.value & FAULT_GEMM_WAITS
    monkeypatch.delenv("RABIT_TEST_SKIP_ONE_ARRIVE")
    monkeypatch.delenv("RABIT_WAIT_TIMEOUT_MS")
    # the same context runs the same call correctly afterwards
    rabit.rabit_gemm(packed, at, bt, N, K, xt, y, ws)
    torch.cuda.synchronize()
    assert rabit.rabit_read_fault(clear=True) == 0
    S = oracle.derive_signs(W, a, b)
    ref = oracle.layer(S, a, b, x)
    err = float(np.max(np.abs(y.cpu().numpy() - ref)) / np.max(np.abs(ref)))
    assert err <= 2e-3


def _read_fault():
    flags = ctypes.c_uint32(0)
    st = rabit.load().rabit_read_fault(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                        ctypes.byref(flags), 1)
    return st, flags.value


@pytest.mark.parametrize("N,K,batch", [(256, 512, 1), (4096, 4096, 4)])
def test_gemv_copy_wait_expiry_is_reported_and_the_context_survives(monkeypatch, N, K, batch):
    W, a, b, x, at, bt, packed, xt = _case(N, K, batch, seed=4300 + N)
    ws = rabit.alloc_gemv_workspace(N, K, 2, batch)
    y = torch.zeros((batch, N), device="cuda")
    monkeypatch.setenv("RABIT_GEMV_KERNEL", "tc")     # the tensor-core path has the copy waits
    monkeypatch.setenv("RABIT_TEST_GEMV_WITHHOLD_COPY", "1")
    monkeypatch.setenv("RABIT_WAIT_TIMEOUT_MS", "50")
    rabit.rabit_gemv(packed, at, bt, N, K, xt, y, workspace=ws)
    st, flags = _read_fault()
    assert st == RABIT_ERR_TIMEOUT
    assert flags & FAULT_GEMV_WAITS
    monkeypatch.delenv("RABIT_TEST_GEMV_WITHHOLD_COPY")
    monkeypatch.delenv("RABIT_WAIT_TIMEOUT_MS")
    # after a fault the workspace is zeroed again (its tile counters may be mid-count)
    ws.zero_()
    rabit.rabit_gemv(packed, at, bt, N, K, xt, y, workspace=ws)
    torch.cuda.synchronize()
    assert rabit.rabit_read_fault(clear=True) == 0
    ref = oracle.layer(oracle.derive_signs(W, a, b), a, b, x)
    err = float(np.max(np.abs(y.cpu().numpy() - ref)) / np.max(np.abs(ref)))
    assert err <= 2e-3


def test_scale_grads_copy_wait_expiry_is_reported_and_the_context_survives(monkeypatch):
    N, K = 512, 1024
    W, a, b, x, at, bt, packed, xt = _case(N, K, 1, seed=4400)
    G = torch.from_numpy(np.random.default_rng(4401).standard_normal((N, K)).astype(np.float32)).cuda()
    ga, gb = torch.empty((2, N), device="cuda"), torch.empty((2, K), device="cuda")
    ws = rabit.alloc_scale_grads_workspace(N, K, 2)
    monkeypatch.setenv("RABIT_TEST_SCALE_GRADS_WITHHOLD_COPY", "1")
    monkeypatch.setenv("RABIT_WAIT_TIMEOUT_MS", "50")
    rabit.rabit_scale_grads(G, packed, at, bt, N, K, ga, gb, ws)
    st, flags = _read_fault()
    assert st == RABIT_ERR_TIMEOUT
    assert flags & FAULT_SCALE_GRADS_WAIT
    monkeypatch.delenv("RABIT_TEST_SCALE_GRADS_WITHHOLD_COPY")
    monkeypatch.delenv("RABIT_WAIT_TIMEOUT_MS")
    rabit.rabit_scale_grads(G, packed, at, bt, N, K, ga, gb, ws)
    torch.cuda.synchronize()
    assert rabit.rabit_read_fault(clear=True) == 0
    S = oracle.derive_signs(W, a, b)
    ref_a, ref_b = oracle.scale_grads(G.cpu().numpy(), S, a, b)
    for got, ref in ((ga, ref_a), (gb, ref_b)):
        err = float(np.max(np.abs(got.cpu().numpy() - ref)) / np.max(np.abs(ref)))
        assert err <= 1e-5


def test_svid_barrier_expiry_is_reported_and_the_context_survives(monkeypatch):
    from oracle import svid as osvid
    N, K, P, T = 192, 320, 2, 2
    W = inputs.weight(4500, N, K, outlier_frac=0.01)
    s_in, s_out = inputs.calibration_stats(4500, N, K)
    dev = lambda v: torch.from_numpy(np.ascontiguousarray(v)).cuda()
    Wt, si, so = dev(W), dev(s_in), dev(s_out)
    a, b = torch.empty((P, N), device="cuda"), torch.empty((P, K), device="cuda")
    packed = rabit.alloc_packed(N, K, P=P)
    ws = rabit.alloc_svid_init_workspace(N, K, P)
    monkeypatch.setenv("RABIT_TEST_SVID_WITHHOLD_ARRIVAL", "1")
    monkeypatch.setenv("RABIT_WAIT_TIMEOUT_MS", "50")
    rabit.rabit_svid_init(Wt, si, so, 0.8, 0.65, a, b, packed, ws, P=P, T=T, power_iters=20)
    st, flags = _read_fault()
    assert st == RABIT_ERR_TIMEOUT
    assert flags & FAULT_SVID_BARRIER
    monkeypatch.delenv("RABIT_TEST_SVID_WITHHOLD_ARRIVAL")
    monkeypatch.delenv("RABIT_WAIT_TIMEOUT_MS")
    rabit.rabit_svid_init(Wt, si, so, 0.8, 0.65, a, b, packed, ws, P=P, T=T, power_iters=100)
    torch.cuda.synchronize()
    assert rabit.rabit_read_fault(clear=True) == 0
    So, ao, bo = osvid.svid_init(W, s_in, s_out, 0.8, 0.65, P=P, T=T)
    S = oracle.unpack(packed.cpu().numpy(), N, K, P=P)
    rec, ref = osvid.reconstruct(S, a.cpu().numpy(), b.cpu().numpy()), osvid.reconstruct(So, ao, bo)
    agree = np.all(S == So, axis=0)          # (a residual within rounding of 0 may flip)
    assert np.mean(~agree) <= 1e-4
    assert float(np.linalg.norm((rec - ref)[agree]) / np.linalg.norm(ref)) <= 1e-4
