"""Host-only checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments before touching the GPU.  No kernel is launched here."""
import ctypes
import os
import re

import pytest
import torch

import oracle
from bit_gemv_rabit_b200 import build as rbuild
from bit_gemv_rabit_b200 import rabit

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]

OK, INVALID, ALIGN, SHAPE, UNSUP, WS, ARCH, CUDA = 0, -1, -2, -3, -4, -5, -6, -7
FAKE = 0x10000  # never dereferenced: every call below fails validation first
P = ctypes.c_void_p


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return rabit.load()


def declared_symbols():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        names |= set(re.findall(r"RABIT_API\s+[\w\s\*]+?\b(rabit_\w+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert {"rabit_derive_pack", "rabit_gemv", "rabit_gemm"} <= names
    for name in names:
        assert hasattr(lib, name), name
    assert names == {s[0] for s in rabit.SIGNATURES}


def test_packed_words_matches_layout_definition(lib):
    for N, K in [(1, 1), (32, 128), (33, 129), (4096, 4096), (11008, 4096), (4096, 14336)]:
        assert lib.rabit_packed_words(N, K, 2) == oracle.packed_words(N, K, 2)
    for N, K in [(1, 1), (33, 129), (4096, 4096)]:
        assert lib.rabit_packed_words(N, K, 3) == oracle.packed_words(N, K, 3)
    assert lib.rabit_packed_words(0, 5, 2) == 0
    assert lib.rabit_gemm_workspace_bytes(4096, 4096, 2, 2048) == 2 * 2048 * 4096 * 2
    assert lib.rabit_gemm_workspace_bytes(10, 200, 2, 3) == 2 * 3 * 256 * 2
    assert lib.rabit_gemm_workspace_bytes(10, 200, 3, 3) == 3 * 3 * 256 * 2


def test_status_strings(lib):
    assert rabit.rabit_status_string(0) == "RABIT_OK"
    assert rabit.rabit_status_string(-8) == "RABIT_ERR_TIMEOUT"
    assert rabit.rabit_status_string(123) == "RABIT_ERR_UNKNOWN"


def test_derive_pack_validation(lib):
    f = lib.rabit_derive_pack
    assert f(P(FAKE), 7, 4, 4, 4, 2, P(FAKE), P(FAKE), P(FAKE), None) == INVALID   # dtype
    assert f(None, 0, 4, 4, 4, 2, P(FAKE), P(FAKE), P(FAKE), None) == INVALID      # null W
    assert f(P(FAKE), 0, 4, 4, 4, 2, P(FAKE), P(FAKE), None, None) == INVALID      # null out
    assert f(P(FAKE), 0, 0, 4, 4, 2, P(FAKE), P(FAKE), P(FAKE), None) == SHAPE     # N = 0
    assert f(P(FAKE), 0, 4, 4, 3, 2, P(FAKE), P(FAKE), P(FAKE), None) == SHAPE     # ldw < K
    assert f(P(FAKE), 0, 4, 4, 4, 4, P(FAKE), P(FAKE), P(FAKE), None) == UNSUP     # P = 4
    assert f(P(FAKE), 0, 4, 4, 4, 1, P(FAKE), P(FAKE), P(FAKE), None) == UNSUP     # P = 1
    assert f(P(FAKE), 0, 4, 4, 4, 2, P(FAKE), P(FAKE), P(FAKE + 4), None) == ALIGN


def test_gemv_validation(lib):
    f = lib.rabit_gemv
    need = lib.rabit_gemv_workspace_bytes(8, 8, 2, 1)
    args = lambda **kw: [P(kw.get("packed", FAKE)), P(FAKE), P(FAKE), kw.get("N", 8), kw.get("K", 8),
                         kw.get("P", 2), P(kw.get("x", FAKE)), kw.get("xd", 1), kw.get("batch", 1),
                         kw.get("ldx", 8), P(kw.get("y", FAKE)), kw.get("ldy", 8), P(kw.get("ws", FAKE)),
                         kw.get("wsb", need), None]
    assert f(*args(xd=5)) == INVALID
    assert f(*args(packed=0)) == INVALID
    assert f(*args(y=0)) == INVALID
    assert f(*args(batch=0)) == SHAPE
    assert f(*args(batch=17)) == SHAPE
    assert f(*args(ldx=7)) == SHAPE
    assert f(*args(ldy=7)) == SHAPE
    assert f(*args(K=0)) == SHAPE
    assert f(*args(P=4)) == UNSUP
    assert f(*args(packed=FAKE + 8)) == ALIGN
    assert f(*args(x=FAKE + 1)) == ALIGN
    assert f(*args(y=FAKE + 2)) == ALIGN
    assert f(*args(ws=0)) == WS
    assert f(*args(wsb=need - 1)) == WS
    assert f(*args(ws=FAKE + 8)) == ALIGN           # workspace 16-byte alignment


PARTIAL_BYTES = 160 * 2 * 16 * 256 * 4     # partial sums: largest grid x 2 tiles x 16 rows x 256


def test_gemv_workspace_layout(lib):
    # partial sums, then the counters (4 bytes per row tile), the scales (4 bytes per path and
    # batch row) and the block maxima (4 bytes per path, batch row and 1024 columns), each
    # rounded up to 1 KiB, then the digit images: per 256 columns and path, 128 bytes per digit
    # row (12 per batch row for fp32 x, rounded up to 8 rows)
    assert lib.rabit_gemv_workspace_bytes(4096, 4096, 2, 1) == PARTIAL_BYTES + 3 * 1024 + 16 * 2 * 16 * 128
    assert lib.rabit_gemv_workspace_bytes(300, 1000, 3, 3) == PARTIAL_BYTES + 3 * 1024 + 4 * 3 * 40 * 128
    for N, K, P, batch in [(1, 1, 2, 1), (14336, 4096, 2, 4), (4096, 11008, 2, 16), (4096, 4096, 3, 16)]:
        w = lib.rabit_gemv_workspace_bytes(N, K, P, batch)
        pairs = -(-K // 256)
        assert w >= PARTIAL_BYTES + 4 * -(-N // 128) + 4 * P * batch + pairs * P * 128 * 12 * batch
        assert w <= PARTIAL_BYTES + 4 * -(-N // 128) + 3072 + 4 * P * batch * (1 + pairs) + pairs * P * 128 * 24 * batch
    assert lib.rabit_gemv_workspace_bytes(8, 8, 2, 0) == 0
    assert lib.rabit_gemv_workspace_bytes(8, 8, 2, 17) == 0


def test_gemm_validation(lib):
    f = lib.rabit_gemm
    need = lib.rabit_gemm_workspace_bytes(8, 16, 2, 4)
    args = lambda **kw: [P(kw.get("packed", FAKE)), P(FAKE), P(FAKE), kw.get("N", 8), kw.get("K", 16),
                         kw.get("P", 2), P(kw.get("x", FAKE)), kw.get("M", 4), kw.get("ldx", 16),
                         P(FAKE), kw.get("ldy", 8), P(kw.get("ws", FAKE)), kw.get("wsb", need), None]
    assert f(*args(x=0)) == INVALID
    assert f(*args(M=0)) == SHAPE
    assert f(*args(ldx=8)) == SHAPE
    assert f(*args(ldy=4)) == SHAPE
    assert f(*args(P=1)) == UNSUP
    assert f(*args(x=FAKE + 8)) == ALIGN            # x must be 16-byte aligned
    assert f(*args(ldx=20)) == ALIGN                # pitch must keep rows 16-byte aligned
    assert f(*args(ws=0)) == WS
    assert f(*args(wsb=need - 1)) == WS
    assert f(*args(ws=FAKE + 16)) == ALIGN          # workspace 256-byte alignment


def test_scale_grads_validation(lib):
    f = lib.rabit_scale_grads
    need = lib.rabit_scale_grads_workspace_bytes(8, 16, 2)
    # row sums: one column tile x 8 rows; column sums: the larger of one row block x 16
    # columns (tile pass) and 160 CTAs x 2 runs x 256 columns (stream-K pass)
    assert need == 2 * (1 * 8 + max(1 * 16, 160 * 2 * 256)) * 4
    args = lambda **kw: [P(kw.get("G", FAKE)), kw.get("ldg", 16), P(kw.get("packed", FAKE)), P(FAKE), P(FAKE),
                         kw.get("N", 8), kw.get("K", 16), kw.get("P", 2), P(FAKE), P(FAKE),
                         P(kw.get("ws", FAKE)), kw.get("wsb", need), None]
    assert f(*args(G=0)) == INVALID
    assert f(*args(ldg=15)) == SHAPE
    assert f(*args(N=0)) == SHAPE
    assert f(*args(P=4)) == UNSUP
    assert f(*args(packed=FAKE + 4)) == ALIGN
    assert f(*args(wsb=need - 1)) == WS
    assert f(*args(ws=FAKE + 4)) == ALIGN


def test_svid_init_validation(lib):
    f = lib.rabit_svid_init
    need = lib.rabit_svid_init_workspace_bytes(8, 16, 2)
    assert need >= 8 * 16 * 4                         # the residual alone
    assert lib.rabit_svid_init_workspace_bytes(8, 16, 4) == 0
    args = lambda **kw: [P(kw.get("W", FAKE)), kw.get("N", 8), kw.get("K", 16), kw.get("ldw", 16), kw.get("P", 2),
                         kw.get("T", 20), kw.get("iters", 40), kw.get("tol", 0.0), P(FAKE), P(FAKE), kw.get("ai", 0.8),
                         kw.get("ao", 0.65), P(FAKE), P(FAKE), P(kw.get("packed", FAKE)),
                         P(kw.get("ws", FAKE)), kw.get("wsb", need), None]
    assert f(*args(W=0)) == INVALID
    assert f(*args(ai=float("nan"))) == INVALID
    assert f(*args(ao=float("inf"))) == INVALID
    assert f(*args(tol=-1e-6)) == INVALID
    assert f(*args(tol=float("nan"))) == INVALID
    assert f(*args(tol=float("inf"))) == INVALID
    assert f(*args(N=0)) == SHAPE
    assert f(*args(ldw=15)) == SHAPE
    assert f(*args(T=0)) == SHAPE
    assert f(*args(T=1001)) == SHAPE
    assert f(*args(iters=0)) == SHAPE
    assert f(*args(P=4)) == UNSUP
    assert f(*args(packed=FAKE + 4)) == ALIGN
    assert f(*args(wsb=need - 1)) == WS
    assert f(*args(ws=0)) == WS
    assert f(*args(ws=FAKE + 16)) == ALIGN


@pytest.mark.skipif(torch.cuda.is_available(), reason="valid arguments would launch on a GPU")
def test_valid_arguments_without_gpu_fail_cleanly(lib):
    st = lib.rabit_derive_pack(P(FAKE), 0, 4, 4, 4, 2, P(FAKE), P(FAKE), P(FAKE), None)
    assert st in (CUDA, ARCH)
    flags = ctypes.c_uint32(0)
    assert lib.rabit_read_fault(None, ctypes.byref(flags), 0) in (CUDA, ARCH)
    need = lib.rabit_svid_init_workspace_bytes(8, 16, 2)
    st = lib.rabit_svid_init(P(FAKE), 8, 16, 16, 2, 20, 40, 0.0, P(FAKE), P(FAKE), 0.8, 0.65, P(FAKE), P(FAKE),
                             P(FAKE), P(FAKE), need, None)
    assert st in (CUDA, ARCH)


def test_gemv_grouped_validation(lib):
    L = rabit.GemvLayer
    good = dict(packed=FAKE, a=FAKE, b=FAKE, N=8, K=8, x=FAKE, ldx=8, y=FAKE, ldy=8)
    def arr(**kw):
        d = dict(good, **kw)
        a = (L * 2)(L(**good), L(**d))
        return ctypes.cast(a, ctypes.c_void_p)
    need = lib.rabit_gemv_grouped_workspace_bytes(arr(), 2, 2, 1, 1)
    # two one-tile, one-unit layers, bf16 x, batch 1: 8 digit rows of 128 bytes per path
    assert need == PARTIAL_BYTES + 3 * 1024 + 2 * 2 * 8 * 128
    assert lib.rabit_gemv_grouped_workspace_bytes(arr(), 2, 4, 1, 1) == 0
    assert lib.rabit_gemv_grouped_workspace_bytes(arr(), 2, 2, 7, 1) == 0
    assert lib.rabit_gemv_grouped_workspace_bytes(arr(), 2, 2, 1, 17) == 0
    f = lib.rabit_gemv_grouped
    assert f(None, 2, 2, 1, 1, P(FAKE), need, None) == INVALID
    assert f(arr(), 0, 2, 1, 1, P(FAKE), need, None) == INVALID
    assert f(arr(), 9, 2, 1, 1, P(FAKE), need, None) == INVALID
    assert f(arr(), 2, 2, 7, 1, P(FAKE), need, None) == INVALID       # dtype
    assert f(arr(), 2, 2, 1, 17, P(FAKE), need, None) == SHAPE        # batch
    assert f(arr(y=0), 2, 2, 1, 1, P(FAKE), need, None) == INVALID
    assert f(arr(K=0), 2, 2, 1, 1, P(FAKE), need, None) == SHAPE
    assert f(arr(ldy=7), 2, 2, 1, 1, P(FAKE), need, None) == SHAPE
    assert f(arr(packed=FAKE + 4), 2, 2, 1, 1, P(FAKE), need, None) == ALIGN
    assert f(arr(), 2, 4, 1, 1, P(FAKE), need, None) == UNSUP
    assert f(arr(), 2, 2, 1, 1, P(FAKE), need - 1, None) == WS
    assert f(arr(), 2, 2, 1, 1, P(FAKE + 8), need, None) == ALIGN


def test_transpose_pack_and_grad_x_validation(lib):
    f = lib.rabit_transpose_pack
    assert f(None, 4, 4, 2, P(FAKE), None) == INVALID
    assert f(P(FAKE), 0, 4, 2, P(FAKE), None) == SHAPE
    assert f(P(FAKE), 4, 0, 2, P(FAKE), None) == SHAPE
    assert f(P(FAKE), 4, 4, 4, P(FAKE), None) == UNSUP
    assert f(P(FAKE + 4), 4, 4, 2, P(FAKE), None) == ALIGN
    assert f(P(FAKE), 4, 4, 2, P(FAKE + 4), None) == ALIGN
    g = lib.rabit_grad_x
    need = lib.rabit_gemm_workspace_bytes(16, 8, 2, 8)      # the transposed layer: K x N
    assert need > 0
    assert g(None, P(FAKE), P(FAKE), 8, 16, 2, P(FAKE), 8, 8, P(FAKE), 16, P(FAKE), need, None) == INVALID
    assert g(P(FAKE), P(FAKE), P(FAKE), 8, 16, 2, P(FAKE), 8, 7, P(FAKE), 16, P(FAKE), need, None) == SHAPE  # ldd < N
    assert g(P(FAKE), P(FAKE), P(FAKE), 8, 16, 2, P(FAKE), 8, 8, P(FAKE), 15, P(FAKE), need, None) == SHAPE  # ldg < K
    assert g(P(FAKE), P(FAKE), P(FAKE), 8, 16, 2, P(FAKE), 8, 8, P(FAKE), 16, P(FAKE), need - 1, None) == WS


def test_gemm_grouped_validation(lib):
    L = rabit.GemvLayer
    good = dict(packed=FAKE, a=FAKE, b=FAKE, N=8, K=16, x=FAKE, ldx=16, y=FAKE, ldy=8)
    def arr(**kw):
        d = dict(good, **kw)
        a = (L * 2)(L(**good), L(**d))
        return ctypes.cast(a, ctypes.c_void_p)
    need = lib.rabit_gemm_grouped_workspace_bytes(arr(), 2, 2, 8)
    # each layer's X' ([P][M][Kp] fp16) in its own 256-byte aligned region
    assert need == 2 * (2 * 8 * 128 * 2)
    assert lib.rabit_gemm_grouped_workspace_bytes(arr(), 5, 2, 8) == 0
    assert lib.rabit_gemm_grouped_workspace_bytes(arr(), 2, 4, 8) == 0
    f = lib.rabit_gemm_grouped
    assert f(None, 2, 2, 8, P(FAKE), need, None) == INVALID
    assert f(arr(), 5, 2, 8, P(FAKE), need, None) == INVALID
    assert f(arr(y=0), 2, 2, 8, P(FAKE), need, None) == INVALID
    assert f(arr(ldx=8), 2, 2, 8, P(FAKE), need, None) == SHAPE
    assert f(arr(ldx=20), 2, 2, 8, P(FAKE), need, None) == ALIGN
    assert f(arr(x=FAKE + 8), 2, 2, 8, P(FAKE), need, None) == ALIGN
    assert f(arr(), 2, 4, 8, P(FAKE), need, None) == UNSUP
    assert f(arr(), 2, 2, 8, P(FAKE), need - 1, None) == WS
    assert f(arr(), 2, 2, 8, P(FAKE + 128), need, None) == ALIGN


def test_prepared_gemv_group_marshals_the_plain_call(lib):
    """GemvGroup builds the same layer array as the plain grouped call, keeps its tensors,
    and sizes the workspace with rabit_gemv_grouped_workspace_bytes (no launch here)."""
    layers = []
    for N, K in ((64, 256), (130, 520)):
        x = torch.zeros((3, K), dtype=torch.bfloat16)
        y = torch.zeros((3, N), dtype=torch.float32)
        layers.append((torch.zeros(rabit.rabit_packed_words(N, K, 2), dtype=torch.int32).view(torch.uint32),
                       torch.ones((2, N)), torch.ones((2, K)), N, K, x, y))
    group = rabit.GemvGroup(layers)
    want = rabit._layer_array(layers)
    for got, ref in zip(group._arr, want):
        for field, _ in rabit.GemvLayer._fields_:
            assert getattr(got, field) == getattr(ref, field)
    assert group._scalars == (2, 2, rabit.RABIT_BF16, 3)
    assert group.workspace.numel() == rabit.rabit_gemv_grouped_workspace_bytes(layers) > 0
    assert group.layers[0][5] is layers[0][5]
