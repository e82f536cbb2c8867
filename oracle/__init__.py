"""Float64 CPU oracle for the RaBiT residual-binary linear layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``; nothing on the product path may import it.  It shares no
code with the CUDA library (``bit_gemv_rabit_b200``) and never imports it.

The arithmetic lives in ``rabit_oracle.c`` (plain float64 loops); this module only
marshals numpy arrays.  Definitions follow "RaBiT: Residual-Aware Binarization Training for
Accurate and Efficient LLMs" (arXiv 2602.05367): sec. 4.1 (binary building block and
stacking), sec. 4.2 "The Coupled Forward Pass" (path derivation), Appendix E.1 "Weight
Packing" (bit convention).  The per-function docstrings name the passage each follows.

Every function here is pinned by ``tests/test_oracle_pins.py`` against hand-written
expectations, brute force, closed-form identities and a numpy matmul.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rabit_oracle.c")
_LIB_PATH = os.path.join(_HERE, "librabit_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP) into oracle/librabit_oracle.so."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
               "-shared", "-std=c11", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_derive_signs.argtypes = [p, i64, i64, i64, ctypes.c_int, p, p, i64, i64, p]
        lib.oracle_derive_signs.restype = None
        lib.oracle_padded_cols.argtypes = [i64]
        lib.oracle_padded_cols.restype = i64
        lib.oracle_packed_words.argtypes = [i64, i64, ctypes.c_int]
        lib.oracle_packed_words.restype = i64
        lib.oracle_word_index.argtypes = [ctypes.c_int, i64, i64, i64, ctypes.c_int]
        lib.oracle_word_index.restype = i64
        lib.oracle_pack.argtypes = [p, i64, i64, ctypes.c_int, p]
        lib.oracle_pack.restype = None
        lib.oracle_unpack.argtypes = [p, i64, i64, ctypes.c_int, p]
        lib.oracle_unpack.restype = None
        lib.oracle_layer.argtypes = [p, i64, p, i64, i64, ctypes.c_int, p, p, p, i64, i64, p]
        lib.oracle_layer.restype = None
        lib.oracle_scale_grads.argtypes = [p, i64, i64, p, ctypes.c_int, p, p, p, p]
        lib.oracle_scale_grads.restype = None
        lib.oracle_grad_x.argtypes = [p, i64, i64, ctypes.c_int, p, p, p, i64, i64, p]
        lib.oracle_grad_x.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def widen(values: np.ndarray) -> np.ndarray:
    """Exact widening to float64.  ``uint16`` arrays are read as bf16 bit patterns."""
    values = np.asarray(values)
    if values.dtype == np.uint16:
        return (values.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if values.dtype in (np.float32, np.float64):
        return values.astype(np.float64)
    raise TypeError(f"unsupported dtype {values.dtype}")


def num_threads() -> int:
    """OpenMP threads the oracle's row loops use."""
    return int(_load().oracle_num_threads())


def derive_signs(W: np.ndarray, a: np.ndarray, b: np.ndarray, P: int = 2,
                 rows: tuple[int, int] | None = None) -> np.ndarray:
    """Sec. 4.2 coupled forward pass: S_1 = sign(W), S_p = sign(W - sum_{i<p} a_i S_i b_i).

    W: [N][K] float32 or bf16 (uint16 bits); a: [P][N]; b: [P][K] (float32).
    Returns int8 [P][n1-n0][K] of +1/-1 for rows [n0, n1) (default: all rows).
    sign(v) = +1 unless v < 0.
    """
    Wd = np.ascontiguousarray(widen(W))
    N, K = Wd.shape
    ad = np.ascontiguousarray(widen(a)).reshape(-1, N)
    bd = np.ascontiguousarray(widen(b)).reshape(-1, K)
    assert ad.shape[0] >= P and bd.shape[0] >= P
    n0, n1 = rows if rows is not None else (0, N)
    S = np.empty((P, n1 - n0, K), dtype=np.int8)
    _load().oracle_derive_signs(_ptr(Wd), N, K, K, P, _ptr(ad), _ptr(bd), n0, n1, _ptr(S))
    return S


def padded_cols(K: int) -> int:
    return int(_load().oracle_padded_cols(K))


def packed_words(N: int, K: int, P: int = 2) -> int:
    return int(_load().oracle_packed_words(N, K, P))


def word_index(k: int, n: int, w: int, K: int, P: int = 2) -> int:
    """Position of (path k, row n, 32-column word w) in the RABIT_LAYOUT_V2 buffer."""
    return int(_load().oracle_word_index(k, n, w, K, P))


def pack(S: np.ndarray) -> np.ndarray:
    """Appendix E.1 packing of int8 signs [P][N][K] into RABIT_LAYOUT_V2 uint32 words."""
    S = np.ascontiguousarray(S, dtype=np.int8)
    P, N, K = S.shape
    out = np.empty(packed_words(N, K, P), dtype=np.uint32)
    _load().oracle_pack(_ptr(S), N, K, P, _ptr(out))
    return out


def unpack(packed: np.ndarray, N: int, K: int, P: int = 2) -> np.ndarray:
    """Inverse of :func:`pack`: int8 [P][N][K] with bit 1 -> -1, bit 0 -> +1."""
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    assert packed.size >= packed_words(N, K, P)
    S = np.empty((P, N, K), dtype=np.int8)
    _load().oracle_unpack(_ptr(packed), N, K, P, _ptr(S))
    return S


def layer(S: np.ndarray, a: np.ndarray, b: np.ndarray, x: np.ndarray,
          rows: np.ndarray | None = None, N: int | None = None) -> np.ndarray:
    """Sec. 4.1 stacked layer: y[beta][i] = sum_k a_k[n_i] sum_j S_k[i][j] b_k[j] x[beta][j].

    S: int8 [P][R][K] signs of R rows (row i is output row rows[i], or i if rows is None);
    a: [P][N]; b: [P][K]; x: [B][K] (float32, float64 or bf16 bits).  Returns float64 [B][R].
    """
    S = np.ascontiguousarray(S, dtype=np.int8)
    P, R, K = S.shape
    xd = np.ascontiguousarray(widen(x))
    if xd.ndim == 1:
        xd = xd[None, :]
    B = xd.shape[0]
    assert xd.shape[1] == K
    ad = np.ascontiguousarray(widen(a))
    N = ad.shape[-1] if N is None else N
    ad = ad.reshape(-1, N)
    bd = np.ascontiguousarray(widen(b)).reshape(-1, K)
    y = np.empty((B, R), dtype=np.float64)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    _load().oracle_layer(_ptr(S), R, None if rows_arr is None else _ptr(rows_arr), N, K, P,
                         _ptr(ad), _ptr(bd), _ptr(xd), B, K, _ptr(y))
    return y


def scale_grads(G: np.ndarray, S: np.ndarray, a: np.ndarray, b: np.ndarray):
    """Scale gradients for G = dL/dW_hat with the signs held fixed (chain rule on sec. 4.1's
    W_hat = sum_k a_k S_k b_k): ga[k][n] = sum_j G S_k b_k, gb[k][j] = sum_n G a_k S_k.
    Returns float64 (ga [P][N], gb [P][K])."""
    S = np.ascontiguousarray(S, dtype=np.int8)
    P, N, K = S.shape
    Gd = np.ascontiguousarray(widen(G)).reshape(N, K)
    ad = np.ascontiguousarray(widen(a)).reshape(-1, N)
    bd = np.ascontiguousarray(widen(b)).reshape(-1, K)
    ga = np.empty((P, N), dtype=np.float64)
    gb = np.empty((P, K), dtype=np.float64)
    _load().oracle_scale_grads(_ptr(Gd), N, K, _ptr(S), P, _ptr(ad), _ptr(bd), _ptr(ga), _ptr(gb))
    return ga, gb


def grad_x(S: np.ndarray, a: np.ndarray, b: np.ndarray, dY: np.ndarray,
           cols: np.ndarray | None = None) -> np.ndarray:
    """Input gradient of sec. 4.1's stacked layer with the signs held fixed:
    gx[m][c] = sum_n dY[m][n] W_hat[n][j_c], W_hat = sum_k a_k S_k b_k.

    S: int8 [P][N][C], the signs of the C columns j_c (cols, or all K columns when cols is
    None); a: [P][N]; b: [P][K]; dY: [M][N] (float32, float64 or bf16 bits).
    Returns float64 [M][C]."""
    S = np.ascontiguousarray(S, dtype=np.int8)
    P, N, C = S.shape
    ad = np.ascontiguousarray(widen(a)).reshape(-1, N)
    bd = np.ascontiguousarray(widen(b)).reshape(P, -1)
    bc = np.ascontiguousarray(bd if cols is None else bd[:, np.asarray(cols)])
    assert bc.shape == (P, C)
    dYd = np.ascontiguousarray(widen(dY))
    if dYd.ndim == 1:
        dYd = dYd[None, :]
    M = dYd.shape[0]
    assert dYd.shape[1] == N
    gx = np.empty((M, C), dtype=np.float64)
    _load().oracle_grad_x(_ptr(S), N, C, P, _ptr(ad), _ptr(bc), _ptr(dYd), M, N, _ptr(gx))
    return gx
