"""Seeded synthetic inputs for the residual-binary linear layer.

This module draws random numbers and shapes them; it holds none of the layer's arithmetic
(no sign, residual, packing or product), so both the float64 oracle's tests and the CUDA
path's tests and benchmark can take their inputs from here.

Recipe (one function per workload item):
  * W ~ N(0, sigma^2) fp32, [N][K] row-major (out features x in features, like
    ``nn.Linear.weight``); optionally a fraction of entries, drawn uniformly without
    replacement, multiplied by an outlier factor.
  * scales, per path k: a_k[n] = u_n * sqrt(m_k), b_k[j] = v_j * sqrt(m_k) with
    u, v ~ U(0.5, 1.5) i.i.d., so a_k[n] * b_k[j] is about U*U*m_k with mean m_k.
    m_1 = mean|W| (a statistic of the drawn W).  m_2 = KAPPA * m_1 with KAPPA = 0.6, the
    closed-form ratio E|R_1| / E|W| for Gaussian W when the first path's scale equals
    E|W| (E||Z| - c| / E|Z| at c = sqrt(2/pi)); it stands in for "mean|.|" of the
    first-path residual without computing that residual here.
  * x ~ N(0, 1) rounded to bf16 (round-to-nearest-even), [B][K]; optionally a fraction of
    the K channels (the same channels for every token) multiplied by a factor.
  * calibration statistics for the initialisation's preconditioning: s_in [K] stands for
    the per-channel max |activation| (log-normal, sigma 0.5, with 1% of the channels x10)
    and s_out [N] for the per-row max |output gradient| (log-normal, sigma 0.3); each is
    divided by its mean.  No calibration data is used.
"""
from __future__ import annotations

import numpy as np

KAPPA = 0.6


def rng_for(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def bf16_bits(values: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    f = np.ascontiguousarray(values, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    rounded = ((u + 0x7FFF + lsb) >> 16).astype(np.uint32)
    nan = np.isnan(f)
    if nan.any():
        rounded = np.where(nan, (f.view(np.uint32) >> 16) | 0x40, rounded)
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def weight(seed: int, N: int, K: int, sigma: float = 0.02, outlier_frac: float = 0.0,
           outlier_scale: float = 20.0) -> np.ndarray:
    """Shared full-precision weight W, fp32 [N][K]."""
    rng = rng_for(seed)
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(sigma)
    if outlier_frac > 0.0:
        count = int(round(outlier_frac * N * K))
        idx = rng.choice(N * K, size=count, replace=False)
        W.reshape(-1)[idx] *= np.float32(outlier_scale)
    return W


def scales(seed: int, W: np.ndarray, P: int = 2) -> tuple[np.ndarray, np.ndarray]:
    """Per-output a [P][N] and per-input b [P][K] fp32 scales for W (see module recipe)."""
    N, K = W.shape
    rng = rng_for(seed + 7919)
    m = float(np.mean(np.abs(W), dtype=np.float64))
    a = np.empty((P, N), dtype=np.float32)
    b = np.empty((P, K), dtype=np.float32)
    for k in range(P):
        mk = m * (KAPPA ** k)
        a[k] = rng.uniform(0.5, 1.5, N) * np.sqrt(mk)
        b[k] = rng.uniform(0.5, 1.5, K) * np.sqrt(mk)
    return a, b


def activations(seed: int, B: int, K: int, channel_outlier_frac: float = 0.0,
                channel_outlier_scale: float = 10.0, dtype: str = "bf16") -> np.ndarray:
    """x [B][K]: bf16 bit patterns (uint16) by default, or fp32 with dtype='f32'."""
    rng = rng_for(seed + 104729)
    x = rng.standard_normal((B, K), dtype=np.float32)
    if channel_outlier_frac > 0.0:
        count = max(1, int(round(channel_outlier_frac * K)))
        ch = rng.choice(K, size=count, replace=False)
        x[:, ch] *= np.float32(channel_outlier_scale)
    if dtype == "bf16":
        return bf16_bits(x)
    if dtype == "f32":
        return x
    raise ValueError(dtype)


def calibration_stats(seed: int, N: int, K: int, outlier_frac: float = 0.01,
                      outlier_scale: float = 10.0) -> tuple[np.ndarray, np.ndarray]:
    """(s_in [K], s_out [N]) fp32, positive, each with mean 1 (see module recipe)."""
    rng = rng_for(seed + 15485863)
    s_in = np.exp(0.5 * rng.standard_normal(K))
    if outlier_frac > 0.0:
        count = max(1, int(round(outlier_frac * K)))
        s_in[rng.choice(K, size=count, replace=False)] *= outlier_scale
    s_out = np.exp(0.3 * rng.standard_normal(N))
    return (s_in / s_in.mean()).astype(np.float32), (s_out / s_out.mean()).astype(np.float32)


# Workload shapes, named by what they are.  Each entry: (name, N, K).
LLAMA2_7B_DECODE_SET = [
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008),
]
LLAMA3_8B_DECODE_SET = [
    ("q_proj", 4096, 4096), ("k_proj", 1024, 4096), ("v_proj", 1024, 4096),
    ("gate_proj", 14336, 4096), ("up_proj", 14336, 4096), ("down_proj", 4096, 14336),
]
LLAMA3_8B_MLP_PREFILL = [("gate_proj", 14336, 4096), ("up_proj", 14336, 4096),
                         ("down_proj", 4096, 14336)]
LLAMA3_70B_MLP_QAT = [("gate_proj", 28672, 8192)]

WORKLOADS = {
    # name: dict(matrices, batch sizes or tokens, weight sigma, outliers, x outliers)
    "single_4096x4096_b1": dict(set=[("layer", 4096, 4096)], batches=[1], sigma=0.02,
                                w_outliers=0.0, x_outliers=0.0, cfg=1),
    "llama2_7b_decode_b1": dict(set=LLAMA2_7B_DECODE_SET, batches=[1], sigma=0.02,
                                w_outliers=0.0, x_outliers=0.0, cfg=2),
    "llama3_8b_decode": dict(set=LLAMA3_8B_DECODE_SET, batches=[1, 4, 8, 16], sigma=0.02,
                             w_outliers=0.001, x_outliers=0.0, cfg=3),
    "llama3_8b_mlp_prefill_m2048": dict(set=LLAMA3_8B_MLP_PREFILL, batches=[2048],
                                        sigma=0.02, w_outliers=0.0, x_outliers=0.01, cfg=4),
    "llama3_70b_mlp_qat_m4096": dict(set=LLAMA3_70B_MLP_QAT, batches=[4096], sigma=0.015,
                                     w_outliers=0.0, x_outliers=0.0, cfg=5),
}


def seed_for(cfg: int, matrix_index: int) -> int:
    return 1000 * cfg + matrix_index
