"""Float64 CPU oracle of the RaBiT initialisation (Iterative Residual SVID with I/O channel
importance-scaled preconditioning).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by ``tests/`` and by the
CPU-baseline leg of ``bench.py``; nothing on the product path may import it, and it shares
no code with the CUDA library.

Definitions follow "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient
LLMs", sec. 4.3 "Stable Initialization for Functional Preservation":

* Preconditioning (sec. 4.3, item 2):  W' = s_out^alpha_out (.) W (.) s_in^alpha_in, with s_out
  per output row and s_in per input column (positive calibration statistics).
* Iterative Residual SVID (sec. 4.3, item 1), for t = 1..T and paths i = 1..P in order:
      R_i^(t) = W' - sum_{j<i} What_j^(t) - sum_{j>i} What_j^(t-1)
      (B_i, g_i', h_i') = SVID(R_i^(t)),   What_i^(t) = g_i' (.) B_i (.) h_i'
  with What_j^(0) = 0, so that t = 1 is the greedy decomposition (Appendix F.3 calls
  iteration 1 "Greedy SVID").
* Scales mapped back (sec. 4.3, after the preconditioning formula):
      g_i = s_out^-alpha_out (.) g_i',   h_i = s_in^-alpha_in (.) h_i'.

SVID is not defined on the pages; the reading taken here is the sign-value-independent
decomposition of the cited prior work: B = sign(R) (+1 unless R < 0, the sign rule used
everywhere in this repository) and g' h'^T the best rank-1 approximation of |R| in the
Frobenius norm, i.e. its leading singular triplet (sigma, u, v) with u, v >= 0 (Perron
vectors of the nonnegative |R|), split evenly: g' = sqrt(sigma) u, h' = sqrt(sigma) v.  A
library SVD supplies the triplet.  Only the product g' h'^T enters What, so the split does
not change the reconstruction.

Pinned by ``tests/test_oracle_svid.py`` (exact recovery of signed rank-1 matrices, with and
without preconditioning; monotone decrease of the objective over the updates; the SVD step
against an independent power iteration; invariance to the normalisation of s_in and s_out;
optimality of the last update).
"""
from __future__ import annotations

import numpy as np


def sign(R: np.ndarray) -> np.ndarray:
    """+1 unless R < 0 (so +0, -0 and NaN give +1), as int8."""
    return np.where(R < 0, -1, 1).astype(np.int8)


def rank1_abs(R: np.ndarray) -> tuple[float, np.ndarray, np.ndarray]:
    """Leading singular triplet of |R| with nonnegative vectors (the rank-1 part of SVID)."""
    A = np.abs(np.asarray(R, dtype=np.float64))
    if not np.any(A):
        N, K = A.shape
        return 0.0, np.zeros(N), np.zeros(K)
    U, s, Vt = np.linalg.svd(A, full_matrices=False)
    u, v = U[:, 0], Vt[0]
    if u.sum() < 0:          # the singular pair is defined up to a common sign
        u, v = -u, -v
    return float(s[0]), np.maximum(u, 0.0), np.maximum(v, 0.0)


def svid(R: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """SVID(R) = (sign R, g', h') with g' h'^T the best rank-1 approximation of |R|."""
    sigma, u, v = rank1_abs(R)
    r = np.sqrt(sigma)
    return sign(R), r * u, r * v


def precondition(W: np.ndarray, s_in: np.ndarray, s_out: np.ndarray,
                 alpha_in: float, alpha_out: float) -> np.ndarray:
    """W' = s_out^alpha_out (.) W (.) s_in^alpha_in (sec. 4.3, item 2), float64."""
    W = np.asarray(W, dtype=np.float64)
    so = np.asarray(s_out, dtype=np.float64) ** float(alpha_out)
    si = np.asarray(s_in, dtype=np.float64) ** float(alpha_in)
    return so[:, None] * W * si[None, :]


def svid_init(W: np.ndarray, s_in: np.ndarray, s_out: np.ndarray, alpha_in: float,
              alpha_out: float, P: int = 2, T: int = 20, history: bool = False):
    """Iterative Residual SVID on the preconditioned W, scales mapped back (sec. 4.3).

    W [N][K] (any float dtype); s_in [K] > 0; s_out [N] > 0.  Returns (S, a, b) with
    S int8 [P][N][K] the final binary cores B_i^(T), a float64 [P][N] = g_i and b float64
    [P][K] = h_i in the original domain; the reconstruction is sum_i a_i (.) S_i (.) b_i.
    With history=True also returns the list of ||W' - sum_j What_j||_F after every
    (t, i) update, starting with the value before the first update.
    """
    Wp = precondition(W, s_in, s_out, alpha_in, alpha_out)
    N, K = Wp.shape
    S = np.ones((P, N, K), dtype=np.int8)
    gp = np.zeros((P, N))
    hp = np.zeros((P, K))
    paths = np.zeros((P, N, K))          # What_i of the latest update of each path
    hist = [float(np.linalg.norm(Wp))] if history else None
    for _t in range(T):
        for i in range(P):
            # paths j < i hold this iteration's update, paths j > i the previous iteration's
            R = Wp - (paths.sum(axis=0) - paths[i])
            S[i], gp[i], hp[i] = svid(R)
            paths[i] = gp[i][:, None] * S[i] * hp[i][None, :]
            if history:
                hist.append(float(np.linalg.norm(Wp - paths.sum(axis=0))))
    so = np.asarray(s_out, dtype=np.float64) ** float(alpha_out)
    si = np.asarray(s_in, dtype=np.float64) ** float(alpha_in)
    a = gp / so[None, :]
    b = hp / si[None, :]
    return (S, a, b, hist) if history else (S, a, b)


def reconstruct(S: np.ndarray, a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """sum_i a_i (.) S_i (.) b_i (sec. 4.1 stacking), float64."""
    return np.einsum("pn,pnk,pk->nk", np.asarray(a, np.float64), S.astype(np.float64),
                     np.asarray(b, np.float64))
