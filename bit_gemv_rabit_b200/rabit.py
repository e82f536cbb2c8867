"""Python binding of librabit: argument marshalling only.

Every function here has the name of a C entry point in include/rabit.h, takes torch CUDA
tensors, passes their data pointers, sizes and torch's current CUDA stream to the C call,
and raises :class:`RabitError` on a non-zero status.  No step of the layer runs here, and
there is no fallback: if ``librabit.so`` is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librabit.so")

RABIT_F32, RABIT_BF16 = 0, 1
STATUS = {0: "RABIT_OK", -1: "RABIT_ERR_INVALID_ARG", -2: "RABIT_ERR_ALIGNMENT",
          -3: "RABIT_ERR_SHAPE", -4: "RABIT_ERR_UNSUPPORTED", -5: "RABIT_ERR_WORKSPACE",
          -6: "RABIT_ERR_ARCH", -7: "RABIT_ERR_CUDA", -8: "RABIT_ERR_TIMEOUT"}

# (name, restype, argtypes) of every symbol include/rabit.h declares.
_c, _p, _i, _sz = ctypes, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = [
    ("rabit_packed_words", _sz, [_i, _i, _i]),
    ("rabit_derive_pack", _i, [_p, _i, _i, _i, _i, _i, _p, _p, _p, _p]),
    ("rabit_gemv_workspace_bytes", _sz, [_i, _i, _i, _i]),
    ("rabit_gemv", _i, [_p, _p, _p, _i, _i, _i, _p, _i, _i, _i, _p, _i, _p, _sz, _p]),
    ("rabit_gemv_grouped_workspace_bytes", _sz, [_p, _i, _i, _i, _i]),
    ("rabit_gemv_grouped", _i, [_p, _i, _i, _i, _i, _p, _sz, _p]),
    ("rabit_gemm_workspace_bytes", _sz, [_i, _i, _i, _i]),
    ("rabit_gemm", _i, [_p, _p, _p, _i, _i, _i, _p, _i, _i, _p, _i, _p, _sz, _p]),
    ("rabit_gemm_noalloc", _i, [_p, _p, _p, _i, _i, _i, _p, _i, _i, _p, _i, _p]),
    ("rabit_gemm_grouped_workspace_bytes", _sz, [_p, _i, _i, _i]),
    ("rabit_gemm_grouped", _i, [_p, _i, _i, _i, _p, _sz, _p]),
    ("rabit_transpose_pack", _i, [_p, _i, _i, _i, _p, _p]),
    ("rabit_grad_x", _i, [_p, _p, _p, _i, _i, _i, _p, _i, _i, _p, _i, _p, _sz, _p]),
    ("rabit_scale_grads_workspace_bytes", _sz, [_i, _i, _i]),
    ("rabit_scale_grads", _i, [_p, _i, _p, _p, _p, _i, _i, _i, _p, _p, _p, _sz, _p]),
    ("rabit_svid_init_workspace_bytes", _sz, [_i, _i, _i]),
    ("rabit_svid_init", _i, [_p, _i, _i, _i, _i, _i, _i, ctypes.c_float, _p, _p, ctypes.c_float,
                             ctypes.c_float, _p, _p, _p, _p, _sz, _p]),
    ("rabit_read_fault", _i, [_p, ctypes.POINTER(ctypes.c_uint32), _i]),
    ("rabit_last_cuda_error", _i, []),
    ("rabit_status_string", ctypes.c_char_p, [_i]),
]

_lib = None


class RabitError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        extra = ""
        if status == -7 and _lib is not None:
            extra = f" (cudaError {_lib.rabit_last_cuda_error()})"
        super().__init__(f"{where}: {STATUS.get(status, status)}{extra}")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load librabit.so (raises OSError if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError(f"{path} not found: build it with `python -m bit_gemv_rabit_b200.build`")
        lib = ctypes.CDLL(path)
        for name, res, args in SIGNATURES:
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise RabitError(status, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dptr(t: torch.Tensor | None) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RABIT_F32
    if t.dtype == torch.bfloat16:
        return RABIT_BF16
    return 99  # rejected by the C layer as RABIT_ERR_INVALID_ARG


def rabit_packed_words(N: int, K: int, P: int = 2) -> int:
    return int(load().rabit_packed_words(N, K, P))


def rabit_gemm_workspace_bytes(N: int, K: int, P: int, M: int) -> int:
    return int(load().rabit_gemm_workspace_bytes(N, K, P, M))


def rabit_derive_pack(W: torch.Tensor, a: torch.Tensor, b: torch.Tensor, packed: torch.Tensor,
                      P: int = 2, stream=None) -> torch.Tensor:
    """W [N][K] (row pitch W.stride(0)) fp32/bf16; a [P][N], b [P][K] fp32; packed uint32 out."""
    N, K = W.shape
    _check(load().rabit_derive_pack(_dptr(W), _dtype_code(W), N, K, W.stride(0), P, _dptr(a),
                                    _dptr(b), _dptr(packed), _stream(stream)), "rabit_derive_pack")
    return packed


def rabit_gemv_workspace_bytes(N: int, K: int, P: int = 2, batch: int = 1) -> int:
    return int(load().rabit_gemv_workspace_bytes(N, K, P, batch))


def alloc_gemv_workspace(N: int, K: int, P: int = 2, batch: int = 16, device=None) -> torch.Tensor:
    """A workspace for rabit_gemv, large enough for batch rows of either x type; reusable by
    later calls on the same stream (every call writes what it reads)."""
    return torch.zeros(rabit_gemv_workspace_bytes(N, K, P, batch), dtype=torch.uint8,
                       device=device or "cuda")


def rabit_gemv(packed: torch.Tensor, a: torch.Tensor, b: torch.Tensor, N: int, K: int,
               x: torch.Tensor, y: torch.Tensor, P: int = 2, workspace: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """x [batch][K] bf16/fp32 (pitch x.stride(0)); y [batch][N] fp32 out (pitch y.stride(0)).
    workspace: from alloc_gemv_workspace (needs no initialisation); when None, a fresh one is
    allocated for this call."""
    batch = x.shape[0]
    if workspace is None:
        workspace = alloc_gemv_workspace(N, K, P, batch, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().rabit_gemv(_dptr(packed), _dptr(a), _dptr(b), N, K, P, _dptr(x), _dtype_code(x),
                             batch, x.stride(0), _dptr(y), y.stride(0), _dptr(workspace), ws_bytes,
                             _stream(stream)),
           "rabit_gemv")
    return y


class GemvLayer(ctypes.Structure):
    """struct rabit_gemv_layer of include/rabit.h."""
    _fields_ = [("packed", ctypes.c_void_p), ("a", ctypes.c_void_p), ("b", ctypes.c_void_p),
                ("N", ctypes.c_int), ("K", ctypes.c_int), ("x", ctypes.c_void_p), ("ldx", ctypes.c_int),
                ("y", ctypes.c_void_p), ("ldy", ctypes.c_int)]


def _layer_array(layers):
    arr = (GemvLayer * len(layers))()
    for i, (packed, a, b, N, K, x, y) in enumerate(layers):
        arr[i] = GemvLayer(packed.data_ptr(), a.data_ptr(), b.data_ptr(), N, K, x.data_ptr(), x.stride(0),
                           y.data_ptr(), y.stride(0))
    return arr


def rabit_gemv_grouped_workspace_bytes(layers, P: int = 2) -> int:
    """layers: sequence of (packed, a, b, N, K, x, y) tuples; every x has the same batch and
    dtype."""
    arr = _layer_array(layers)
    x0 = layers[0][5]
    return int(load().rabit_gemv_grouped_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), len(layers), P,
                                                         _dtype_code(x0), x0.shape[0]))


def alloc_gemv_grouped_workspace(layers, P: int = 2, device=None) -> torch.Tensor:
    return torch.empty(rabit_gemv_grouped_workspace_bytes(layers, P), dtype=torch.uint8, device=device or "cuda")


def rabit_gemv_grouped(layers, P: int = 2, workspace: torch.Tensor | None = None, stream=None):
    """layers: sequence of (packed, a, b, N, K, x, y); every x has the same batch and dtype.
    One launch computes rabit_gemv for each layer."""
    arr = _layer_array(layers)
    x0 = layers[0][5]
    if workspace is None:
        workspace = alloc_gemv_grouped_workspace(layers, P, device=x0.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().rabit_gemv_grouped(ctypes.cast(arr, ctypes.c_void_p), len(layers), P, _dtype_code(x0),
                                     x0.shape[0], _dptr(workspace), ws_bytes, _stream(stream)),
           "rabit_gemv_grouped")
    return [layer[6] for layer in layers]


class GemvGroup:
    """A prepared rabit_gemv_grouped call over fixed tensors: the layer array, the scalar
    arguments and the workspace are marshalled once, and run() only enqueues.  The layers'
    tensors (kept referenced here) must stay the same objects; their contents may change
    between runs (new x every step, say)."""

    def __init__(self, layers, P: int = 2, workspace: torch.Tensor | None = None):
        self.layers = list(layers)
        self._arr = _layer_array(self.layers)
        self._ptr = ctypes.cast(self._arr, ctypes.c_void_p)
        x0 = self.layers[0][5]
        self._scalars = (len(self.layers), P, _dtype_code(x0), x0.shape[0])
        if workspace is None:
            workspace = alloc_gemv_grouped_workspace(self.layers, P, device=x0.device)
        self.workspace = workspace
        self._ws = (_dptr(workspace), workspace.numel() * workspace.element_size())
        self._fn = load().rabit_gemv_grouped

    def run(self, stream=None):
        _check(self._fn(self._ptr, *self._scalars, *self._ws, _stream(stream)), "rabit_gemv_grouped")
        return [layer[6] for layer in self.layers]


def rabit_gemm(packed: torch.Tensor, a: torch.Tensor, b: torch.Tensor, N: int, K: int,
               x: torch.Tensor, y: torch.Tensor, workspace: torch.Tensor, P: int = 2,
               stream=None) -> torch.Tensor:
    """x [M][K] bf16 (pitch x.stride(0)); y [M][N] fp32 out; workspace: caller scratch."""
    M = x.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().rabit_gemm(_dptr(packed), _dptr(a), _dptr(b), N, K, P, _dptr(x), M, x.stride(0),
                             _dptr(y), y.stride(0), _dptr(workspace), ws_bytes, _stream(stream)),
           "rabit_gemm")
    return y


def rabit_gemm_grouped_workspace_bytes(layers, P: int = 2) -> int:
    """layers: sequence of (packed, a, b, N, K, x, y) with x bf16 [M][K] (the same M)."""
    arr = _layer_array(layers)
    return int(load().rabit_gemm_grouped_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), len(layers), P,
                                                         layers[0][5].shape[0]))


def alloc_gemm_grouped_workspace(layers, P: int = 2, device=None) -> torch.Tensor:
    return torch.empty(rabit_gemm_grouped_workspace_bytes(layers, P), dtype=torch.uint8, device=device or "cuda")


def rabit_gemm_grouped(layers, workspace: torch.Tensor, P: int = 2, stream=None):
    """layers: sequence of (packed, a, b, N, K, x, y); one launch computes rabit_gemm for each."""
    arr = _layer_array(layers)
    M = layers[0][5].shape[0]
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().rabit_gemm_grouped(ctypes.cast(arr, ctypes.c_void_p), len(layers), P, M, _dptr(workspace),
                                     ws_bytes, _stream(stream)),
           "rabit_gemm_grouped")
    return [layer[6] for layer in layers]


def rabit_transpose_pack(packed: torch.Tensor, N: int, K: int, packed_t: torch.Tensor, P: int = 2,
                         stream=None) -> torch.Tensor:
    """packed: signs of N x K; packed_t (alloc_packed(K, N, P)) receives those of the transpose."""
    _check(load().rabit_transpose_pack(_dptr(packed), N, K, P, _dptr(packed_t), _stream(stream)),
           "rabit_transpose_pack")
    return packed_t


def rabit_grad_x(packed_t: torch.Tensor, a: torch.Tensor, b: torch.Tensor, N: int, K: int,
                 dy: torch.Tensor, grad_x: torch.Tensor, workspace: torch.Tensor, P: int = 2,
                 stream=None) -> torch.Tensor:
    """dy [M][N] bf16; grad_x [M][K] fp32 out; packed_t from rabit_transpose_pack; workspace
    from alloc_gemm_workspace(K, N, P, M)."""
    M = dy.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().rabit_grad_x(_dptr(packed_t), _dptr(a), _dptr(b), N, K, P, _dptr(dy), M, dy.stride(0),
                               _dptr(grad_x), grad_x.stride(0), _dptr(workspace), ws_bytes, _stream(stream)),
           "rabit_grad_x")
    return grad_x


def rabit_gemm_noalloc(packed: torch.Tensor, a: torch.Tensor, b: torch.Tensor, N: int, K: int,
                       x: torch.Tensor, y: torch.Tensor, P: int = 2, stream=None) -> torch.Tensor:
    """rabit_gemm without a workspace, for callers that may not allocate device memory: the
    scratch is the library's fixed buffer (RABIT_GEMM_NOALLOC_SCRATCH_BYTES per device).
    Calls that may overlap on the GPU race on that buffer; order them on one stream."""
    M = x.shape[0]
    _check(load().rabit_gemm_noalloc(_dptr(packed), _dptr(a), _dptr(b), N, K, P, _dptr(x), M,
                                     x.stride(0), _dptr(y), y.stride(0), _stream(stream)),
           "rabit_gemm_noalloc")
    return y


def rabit_scale_grads_workspace_bytes(N: int, K: int, P: int = 2) -> int:
    return int(load().rabit_scale_grads_workspace_bytes(N, K, P))


def rabit_scale_grads(G: torch.Tensor, packed: torch.Tensor, a: torch.Tensor, b: torch.Tensor,
                      N: int, K: int, grad_a: torch.Tensor, grad_b: torch.Tensor,
                      workspace: torch.Tensor, P: int = 2, stream=None):
    """G [N][K] fp32 (pitch G.stride(0)) = dL/dW_hat; grad_a [P][N], grad_b [P][K] fp32 out."""
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().rabit_scale_grads(_dptr(G), G.stride(0), _dptr(packed), _dptr(a), _dptr(b), N, K, P,
                                    _dptr(grad_a), _dptr(grad_b), _dptr(workspace), ws_bytes,
                                    _stream(stream)), "rabit_scale_grads")
    return grad_a, grad_b


def alloc_scale_grads_workspace(N: int, K: int, P: int = 2, device=None) -> torch.Tensor:
    return torch.empty(rabit_scale_grads_workspace_bytes(N, K, P), dtype=torch.uint8,
                       device=device or "cuda")


def rabit_svid_init_workspace_bytes(N: int, K: int, P: int = 2) -> int:
    return int(load().rabit_svid_init_workspace_bytes(N, K, P))


def alloc_svid_init_workspace(N: int, K: int, P: int = 2, device=None) -> torch.Tensor:
    return torch.empty(rabit_svid_init_workspace_bytes(N, K, P), dtype=torch.uint8,
                       device=device or "cuda")


def rabit_svid_init(W: torch.Tensor, s_in: torch.Tensor, s_out: torch.Tensor, alpha_in: float,
                    alpha_out: float, a: torch.Tensor, b: torch.Tensor, packed: torch.Tensor,
                    workspace: torch.Tensor, P: int = 2, T: int = 20, power_iters: int = 40,
                    power_tol: float = 0.0, stream=None):
    """W [N][K] fp32 (pitch W.stride(0)); s_in [K], s_out [N] fp32; a [P][N], b [P][K] fp32 and
    packed (the final signs) out.  Iterative Residual SVID initialisation; each update takes
    at most `power_iters` power steps, fewer once a step moves the unit vectors u and v by at
    most `power_tol` (Euclidean norm)."""
    N, K = W.shape
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().rabit_svid_init(_dptr(W), N, K, W.stride(0), P, T, power_iters, float(power_tol), _dptr(s_in),
                                  _dptr(s_out), float(alpha_in), float(alpha_out), _dptr(a), _dptr(b),
                                  _dptr(packed), _dptr(workspace), ws_bytes, _stream(stream)),
           "rabit_svid_init")
    return a, b, packed


def rabit_read_fault(clear: bool = True, stream=None) -> int:
    """Synchronise and return the device fault word (0 = no bounded wait expired)."""
    flags = ctypes.c_uint32(0)
    st = load().rabit_read_fault(_stream(stream), ctypes.byref(flags), 1 if clear else 0)
    if st not in (0, -8):
        raise RabitError(st, "rabit_read_fault")
    return int(flags.value)


def rabit_status_string(status: int) -> str:
    return load().rabit_status_string(status).decode()


def alloc_packed(N: int, K: int, P: int = 2, device=None) -> torch.Tensor:
    """A uint32 tensor of rabit_packed_words(N, K, P) words (torch allocates, 16 B aligned)."""
    return torch.empty(rabit_packed_words(N, K, P), dtype=torch.uint32, device=device or "cuda")


def alloc_gemm_workspace(N: int, K: int, P: int, M: int, device=None) -> torch.Tensor:
    return torch.empty(rabit_gemm_workspace_bytes(N, K, P, M), dtype=torch.uint8,
                       device=device or "cuda")
