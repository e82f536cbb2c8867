"""Pins of the float64 oracle against facts fixed outside the oracle itself.

Each test names what pins which oracle function:
  * hand-derived sign cases (tests/golden/derive_8x16_cases.txt)         -> derive_signs
  * a hand-computed 2x3 worked example (tests/golden/layer_2x3_worked.txt) -> derive, pack, layer
  * brute-force minimisation of the per-element path-2 error               -> derive_signs (S2)
  * the Frobenius identity ||W-W2||^2 = ||R1||^2 - 2 sum c|R1| + sum c^2   -> derive_signs (S2)
  * hand-built words (all +1, all -1, alternating) and the layout formula   -> pack / unpack
  * numpy matmul of the materialised W_hat, one-hot x, a2 = 0, classic
    per-matrix binarisation, linearity                                      -> layer
Sources: "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
sec. 4.1 (building block, stacking), sec. 4.2 (coupled forward pass), Appendix E.1
(weight packing).
"""
import os

import numpy as np
import pytest

import oracle
from bit_gemv_rabit_b200 import inputs

F32 = np.float32


def _read_kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#") or ":" not in line:
            continue
        k, v = line.split(":", 1)
        out[k.strip()] = v.split()
    return out


def _golden_cases(golden_dir):
    path = os.path.join(golden_dir, "derive_8x16_cases.txt")
    a1 = b1 = None
    cases = {}
    for line in open(path):
        s = line.strip()
        if s.startswith("# a1:"):
            a1 = np.array([float(t) for t in s[5:].split()], dtype=F32)
        elif s.startswith("# b1:"):
            b1 = np.array([float(t) for t in s[5:].split()], dtype=F32)
        elif s and not s.startswith("#"):
            parts = s.split()
            cases[int(parts[0])] = (parts[1], int(parts[2]), int(parts[3]))
    assert a1 is not None and b1 is not None and len(cases) == 16
    return a1, b1, cases


def _case_value(expr, c):
    c = F32(c)
    table = {
        "+0.0": F32(0.0), "-0.0": F32(-0.0), "c": c, "-c": -c,
        "nextup(c)": np.nextafter(c, F32(np.inf)), "nextdown(c)": np.nextafter(c, F32(0)),
        "-nextup(c)": -np.nextafter(c, F32(np.inf)), "-nextdown(c)": -np.nextafter(c, F32(0)),
        "2^-149": F32(2.0 ** -149), "-2^-149": F32(-(2.0 ** -149)),
        "3.0e38": F32(3.0e38), "-3.0e38": F32(-3.0e38),
        "3c": F32(3) * c, "c/2": c / F32(2), "-c/2": -c / F32(2), "-3c": F32(-3) * c,
    }
    return table[expr]


def test_hand_derived_sign_cases(golden_dir):
    a1, b1, cases = _golden_cases(golden_dir)
    N, K = 8, 16
    W = np.zeros((N, K), dtype=F32)
    e1 = np.zeros((N, K), dtype=np.int8)
    e2 = np.zeros((N, K), dtype=np.int8)
    for n in range(N):
        for j in range(K):
            expr, s1, s2 = cases[(j + 3 * n) % 16]
            c = a1[n] * b1[j]
            assert float(c) == float(a1[n]) * float(b1[j])  # dyadic: exact in fp32
            W[n, j] = _case_value(expr, c)
            e1[n, j], e2[n, j] = s1, s2
    assert np.signbit(W[np.where(W == 0)]).any()  # the -0.0 case is really present
    a = np.stack([a1, np.ones(N, F32)])
    b = np.stack([b1, np.ones(K, F32)])
    S = oracle.derive_signs(W, a, b, P=2)
    np.testing.assert_array_equal(S[0], e1)
    np.testing.assert_array_equal(S[1], e2)


def test_worked_layer_example(golden_dir):
    g = _read_kv(os.path.join(golden_dir, "layer_2x3_worked.txt"))
    f = lambda k: np.array([float(t) for t in g[k]], dtype=F32)
    W = np.stack([f("W0"), f("W1")])
    a = np.stack([f("a1"), f("a2")])
    b = np.stack([f("b1"), f("b2")])
    x = np.stack([f("x0"), f("x1")])
    S = oracle.derive_signs(W, a, b)
    np.testing.assert_array_equal(S[0], np.stack([f("S1_0"), f("S1_1")]).astype(np.int8))
    np.testing.assert_array_equal(S[1], np.stack([f("S2_0"), f("S2_1")]).astype(np.int8))
    y = oracle.layer(S, a, b, x)
    np.testing.assert_array_equal(y, np.stack([f("y0"), f("y1")]).astype(np.float64))
    packed = oracle.pack(S)
    assert packed.size == int(g["packed_words"][0])
    expect = np.zeros(packed.size, dtype=np.uint32)
    for item in g["packed"]:
        idx, val = item.split(":")
        expect[int(idx)] = int(val, 16)
    np.testing.assert_array_equal(packed, expect)


def _random_layer(seed, N, K, sigma=0.02, outliers=0.0):
    W = inputs.weight(seed, N, K, sigma=sigma, outlier_frac=outliers)
    a, b = inputs.scales(seed, W)
    return W, a, b


def test_brute_force_path2_minimises_elementwise_error():
    # The path-2 objective separates per element: for each (n, j) the chosen s2 must
    # minimise (R1 - c*s)^2 over s in {+1, -1}, c = a2[n]*b2[j] > 0; ties go to +1.
    rng = np.random.default_rng(5)
    N, K = 8, 16
    W = rng.standard_normal((N, K)).astype(F32)
    a = rng.uniform(0.2, 1.0, (2, N)).astype(F32)
    b = rng.uniform(0.2, 1.0, (2, K)).astype(F32)
    S = oracle.derive_signs(W, a, b)
    for n in range(N):
        for j in range(K):
            w = float(W[n, j])
            best1 = min((+1, -1), key=lambda s: ((w - float(a[0, n]) * float(b[0, j]) * s) ** 2, -s))
            # path 1: sign(W) minimises |W - c1*s| for any c1 > 0
            assert S[0, n, j] == best1
            r1 = w - float(a[0, n]) * S[0, n, j] * float(b[0, j])
            c2 = float(a[1, n]) * float(b[1, j])
            errs = {s: (r1 - c2 * s) ** 2 for s in (+1, -1)}
            best2 = +1 if errs[+1] <= errs[-1] else -1
            assert S[1, n, j] == best2


def test_frobenius_identity_and_error_hierarchy():
    # With c_nj = a2[n] b2[j] > 0 and S2 = sign(R1):
    #   ||W - W_hat2||^2 = ||R1||^2 - 2 sum c |R1| + sum c^2     (exact identity)
    # and ||W - W_hat2|| <= ||W - W_hat1|| holds iff sum c^2 <= 2 sum c |R1|.
    for seed, (N, K) in [(11, (64, 96)), (12, (33, 130))]:
        W, a, b = _random_layer(seed, N, K)
        S = oracle.derive_signs(W, a, b)
        Wd = W.astype(np.float64)
        c1 = np.outer(a[0].astype(np.float64), b[0].astype(np.float64))
        c2 = np.outer(a[1].astype(np.float64), b[1].astype(np.float64))
        W1 = c1 * S[0]
        W2 = W1 + c2 * S[1]
        R1 = Wd - W1
        lhs = np.sum((Wd - W2) ** 2)
        rhs = np.sum(R1 ** 2) - 2 * np.sum(c2 * np.abs(R1)) + np.sum(c2 ** 2)
        assert lhs == pytest.approx(rhs, rel=1e-12)
        assert np.sum(c2 ** 2) <= 2 * np.sum(c2 * np.abs(R1))
        assert np.linalg.norm(Wd - W2) <= np.linalg.norm(Wd - W1)


def test_planted_path2_sign_flip_breaks_identity():
    # A plausible oracle mistake (S2 = sign(W) instead of sign(R1)) must fail the identity.
    W, a, b = _random_layer(13, 32, 64)
    S = oracle.derive_signs(W, a, b)
    Wd = W.astype(np.float64)
    c1 = np.outer(a[0].astype(np.float64), b[0].astype(np.float64))
    c2 = np.outer(a[1].astype(np.float64), b[1].astype(np.float64))
    R1 = Wd - c1 * S[0]
    wrong = S[0]
    lhs = np.sum((R1 - c2 * wrong) ** 2)
    rhs = np.sum(R1 ** 2) - 2 * np.sum(c2 * np.abs(R1)) + np.sum(c2 ** 2)
    assert abs(lhs - rhs) > 1e-6 * rhs


def test_exact_first_path_gives_zero_residual():
    # W = a1 (.) S (.) b1 exactly -> R1 == 0 -> S2 == +1 everywhere, ||W - W_hat1|| = 0.
    rng = np.random.default_rng(3)
    N, K = 16, 40
    a1 = (2.0 ** rng.integers(-4, 2, N)).astype(F32)
    b1 = (2.0 ** rng.integers(-4, 2, K)).astype(F32)
    S = np.where(rng.random((N, K)) < 0.5, -1, 1).astype(F32)
    W = (a1[:, None] * S * b1[None, :]).astype(F32)
    a = np.stack([a1, np.ones(N, F32)])
    b = np.stack([b1, np.ones(K, F32)])
    got = oracle.derive_signs(W, a, b)
    np.testing.assert_array_equal(got[0], S.astype(np.int8))
    assert np.all(got[1] == 1)


def test_gaussian_path_flip_fraction_band():
    # For Gaussian W with c ~ mean|W| the fraction of S2 != S1 is about P(|Z| < 0.798) = 0.575
    # (sanity band, not an exact value).
    N, K = 256, 512
    W = inputs.weight(21, N, K)
    m = float(np.mean(np.abs(W)))
    a = np.full((2, N), np.sqrt(m), dtype=F32)
    b = np.full((2, K), np.sqrt(m), dtype=F32)
    S = oracle.derive_signs(W, a, b)
    frac = float(np.mean(S[0] != S[1]))
    assert 0.55 < frac < 0.60


def test_pack_hand_built_words():
    N, K, P = 32, 128, 2
    S = np.ones((P, N, K), dtype=np.int8)
    S[1] = -1
    S[0, 5, :32] = np.where(np.arange(32) % 2 == 1, -1, 1)  # alternating: bits 1,3,5,... set
    packed = oracle.pack(S)
    assert packed.size == P * N * K // 32
    assert packed[oracle.word_index(0, 0, 0, K)] == 0x00000000
    assert packed[oracle.word_index(1, 7, 3, K)] == 0xFFFFFFFF
    assert packed[oracle.word_index(0, 5, 0, K)] == 0xAAAAAAAA
    # column 0 is the least significant bit
    S2 = np.ones((1, 1, 1), dtype=np.int8)
    S2[0, 0, 0] = -1
    p2 = oracle.pack(S2)
    assert p2[0] == 1 and np.count_nonzero(p2) == 1


def test_layout_formula_hand_offsets():
    # N=40, K=200 -> Kp=256: 8 groups of 32 columns per row, 2 words (paths) per group.
    N, K = 40, 200
    assert oracle.padded_cols(K) == 256
    assert oracle.packed_words(N, K, 2) == 40 * 8 * 2
    # (k, n, w) -> (n*8 + w)*2 + k, evaluated by hand:
    assert oracle.word_index(0, 0, 0, K) == 0
    assert oracle.word_index(1, 0, 0, K) == 1
    assert oracle.word_index(0, 0, 3, K) == 6
    assert oracle.word_index(0, 1, 0, K) == 16
    assert oracle.word_index(0, 33, 5, K) == 538
    assert oracle.word_index(1, 39, 7, K) == 639      # the last word of the buffer
    # three paths: groups of 4 words (one padding word), (n*8 + w)*4 + k
    assert oracle.packed_words(N, K, 3) == 40 * 8 * 4
    assert oracle.word_index(2, 1, 2, K, P=3) == 42


def test_pack_unpack_roundtrip_and_padding_zero():
    rng = np.random.default_rng(9)
    for (N, K) in [(1, 1), (31, 127), (33, 129), (64, 256), (70, 300)]:
        S = np.where(rng.random((2, N, K)) < 0.5, -1, 1).astype(np.int8)
        packed = oracle.pack(S)
        np.testing.assert_array_equal(oracle.unpack(packed, N, K), S)
        # every set bit must belong to a real (row, column); padding stays 0
        ones = int(sum(bin(int(v)).count("1") for v in packed))
        assert ones == int(np.sum(S == -1))


def test_layer_matches_numpy_matmul_of_materialised_weight():
    for seed, (N, K, B) in [(31, (48, 160, 3)), (32, (64, 256, 1))]:
        W, a, b = _random_layer(seed, N, K)
        S = oracle.derive_signs(W, a, b)
        x = inputs.bf16_to_f32(inputs.activations(seed, B, K)).astype(np.float64)
        W_hat = sum(np.outer(a[k].astype(np.float64), b[k].astype(np.float64)) * S[k] for k in range(2))
        ref = x @ W_hat.T
        y = oracle.layer(S, a, b, x)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_layer_special_cases():
    W, a, b = _random_layer(41, 24, 96)
    S = oracle.derive_signs(W, a, b)
    K = W.shape[1]
    # one-hot x = e_j gives column j of W_hat exactly
    for j in (0, 17, K - 1):
        x = np.zeros((1, K))
        x[0, j] = 1.0
        y = oracle.layer(S, a, b, x)[0]
        col = sum(a[k].astype(np.float64) * S[k][:, j] * float(b[k, j]) for k in range(2))
        np.testing.assert_array_equal(y, col)
    # a2 = 0 -> path 1 only
    x = np.random.default_rng(1).standard_normal((2, K))
    a0 = a.copy()
    a0[1] = 0
    y_full = oracle.layer(S, a0, b, x)
    y_p1 = oracle.layer(S[:1], a0[:1], b[:1], x)
    np.testing.assert_allclose(y_full, y_p1, rtol=1e-13)
    # b == 1, a == mean|W|, one path: classic per-matrix binarisation mean|W| * sign(W) x
    m = float(np.mean(np.abs(W)))
    a1 = np.full((1, W.shape[0]), m)
    b1 = np.ones((1, K))
    S1 = oracle.derive_signs(W, np.vstack([a1, a1]).astype(F32), np.vstack([b1, b1]).astype(F32), P=1)
    y = oracle.layer(S1, a1, b1, x)
    ref = x @ (m * np.where(W < 0, -1.0, 1.0)).T
    np.testing.assert_allclose(y, ref, rtol=1e-12)
    # linearity in x
    x2 = np.random.default_rng(2).standard_normal((2, K))
    np.testing.assert_allclose(oracle.layer(S, a, b, 2 * x + x2),
                               2 * oracle.layer(S, a, b, x) + oracle.layer(S, a, b, x2),
                               rtol=1e-11, atol=1e-12)


def test_layer_row_subset_matches_full():
    W, a, b = _random_layer(51, 64, 128)
    S = oracle.derive_signs(W, a, b)
    x = np.random.default_rng(4).standard_normal((3, 128))
    full = oracle.layer(S, a, b, x)
    rows = np.array([0, 5, 63])
    Ssub = oracle.derive_signs(W, a, b, rows=(5, 6))
    np.testing.assert_array_equal(Ssub[:, 0], S[:, 5])
    sub = oracle.layer(S[:, rows], a, b, x, rows=rows)
    np.testing.assert_array_equal(sub, full[:, rows])


def test_bf16_weight_widens_exactly():
    W = inputs.weight(61, 8, 64)
    Wb = inputs.bf16_bits(W)
    a, b = inputs.scales(61, W)
    S_bits = oracle.derive_signs(Wb, a, b)
    S_f32 = oracle.derive_signs(inputs.bf16_to_f32(Wb), a, b)
    np.testing.assert_array_equal(S_bits, S_f32)


# ---- three paths: the residual rule applied once more (S_3 = sign(W - W_hat_1 - W_hat_2)),
# grouped as three words plus a zero padding word (Appendix E.1 "Weight Packing", PackedBits3).

def _three_path_layer(seed, N, K):
    W = inputs.weight(seed, N, K)
    a, b = inputs.scales(seed, W, P=3)
    return W, a, b


def test_three_path_signs_follow_the_residual_rule():
    # brute force per element on a small case, written out in float64 here
    rng = np.random.default_rng(71)
    N, K = 8, 24
    W = rng.standard_normal((N, K)).astype(F32)
    a = rng.uniform(0.1, 0.9, (3, N)).astype(F32)
    b = rng.uniform(0.1, 0.9, (3, K)).astype(F32)
    S = oracle.derive_signs(W, a, b, P=3)
    S2 = oracle.derive_signs(W, a, b, P=2)
    np.testing.assert_array_equal(S[:2], S2)          # the first two paths do not change
    for n in range(N):
        for j in range(K):
            r = float(W[n, j])
            for k in range(3):
                c = float(a[k, n]) * float(b[k, j])
                errs = {s: (r - c * s) ** 2 for s in (+1, -1)}
                best = +1 if errs[+1] <= errs[-1] else -1
                assert S[k, n, j] == best
                r -= c * best


def test_three_path_frobenius_identity_and_hierarchy():
    W, a, b = _three_path_layer(72, 48, 160)
    S = oracle.derive_signs(W, a, b, P=3)
    Wd = W.astype(np.float64)
    c = [np.outer(a[k].astype(np.float64), b[k].astype(np.float64)) for k in range(3)]
    W2 = c[0] * S[0] + c[1] * S[1]
    W3 = W2 + c[2] * S[2]
    R2 = Wd - W2
    lhs = np.sum((Wd - W3) ** 2)
    rhs = np.sum(R2 ** 2) - 2 * np.sum(c[2] * np.abs(R2)) + np.sum(c[2] ** 2)
    assert lhs == pytest.approx(rhs, rel=1e-12)
    assert np.linalg.norm(Wd - W3) <= np.linalg.norm(Wd - W2)


def test_three_path_pack_groups_and_roundtrip():
    rng = np.random.default_rng(73)
    N, K = 5, 200                                      # Kp = 256: 8 groups of 4 words per row
    S = np.where(rng.random((3, N, K)) < 0.5, -1, 1).astype(np.int8)
    packed = oracle.pack(S)
    assert packed.size == N * 8 * 4
    np.testing.assert_array_equal(oracle.unpack(packed, N, K, P=3), S)
    assert np.all(packed.reshape(N, 8, 4)[:, :, 3] == 0)    # the padding word of every group
    # hand check: path 3 (k=2), row 4, column 37 -> word (4*8 + 1)*4 + 2 = 134, bit 5
    S1 = np.ones((3, N, K), dtype=np.int8)
    S1[2, 4, 37] = -1
    p1 = oracle.pack(S1)
    assert p1[134] == 1 << 5 and np.count_nonzero(p1) == 1


def test_three_path_layer_matches_numpy_matmul():
    W, a, b = _three_path_layer(74, 40, 130)
    S = oracle.derive_signs(W, a, b, P=3)
    x = inputs.bf16_to_f32(inputs.activations(74, 3, 130)).astype(np.float64)
    W_hat = sum(np.outer(a[k].astype(np.float64), b[k].astype(np.float64)) * S[k] for k in range(3))
    np.testing.assert_allclose(oracle.layer(S, a, b, x), x @ W_hat.T, rtol=1e-12, atol=1e-14)


# ---- scale gradients (the layer's backward for a and b with the signs held fixed)

def test_scale_grads_match_finite_differences_of_the_layer():
    # L(a, b) = sum_{m,n} dY[m][n] * y[m][n] is linear in each a_k[n] and each b_k[j], so a
    # difference quotient of the pinned layer is exact up to float64 rounding.
    N, K, M = 12, 70, 5
    W, a, b = _three_path_layer(91, N, K)
    S = oracle.derive_signs(W, a, b, P=3)
    rng = np.random.default_rng(91)
    x = rng.standard_normal((M, K))
    dY = rng.standard_normal((M, N))
    G = dY.T @ x                                             # dL/dW_hat for y = x W_hat^T
    ga, gb = oracle.scale_grads(G, S, a, b)
    ad, bd = a.astype(np.float64), b.astype(np.float64)
    L = lambda a_, b_: float(np.sum(dY * oracle.layer(S, a_, b_, x)))
    base = L(ad, bd)
    for k, n in [(0, 0), (1, 5), (2, N - 1)]:
        a2 = ad.copy(); a2[k, n] += 1.0
        assert L(a2, bd) - base == pytest.approx(ga[k, n], rel=1e-9, abs=1e-9)
    for k, j in [(0, 3), (1, K - 1), (2, 40)]:
        b2 = bd.copy(); b2[k, j] += 1.0
        assert L(ad, b2) - base == pytest.approx(gb[k, j], rel=1e-9, abs=1e-9)


def test_scale_grads_hand_case():
    # N=1, K=2, one path: W_hat = a*[s0*b0, s1*b1]; G = [g0, g1]
    S = np.array([[[1, -1]]], dtype=np.int8)
    a = np.array([[2.0]]); b = np.array([[3.0, 5.0]])
    G = np.array([[7.0, 11.0]])
    ga, gb = oracle.scale_grads(G, S, a, b)
    assert ga[0, 0] == 7 * 3 - 11 * 5              # -34
    np.testing.assert_array_equal(gb[0], [7 * 2, -11 * 2])


def test_grad_x_matches_finite_differences_of_the_layer():
    # L(x) = sum_{m,n} dY[m][n] * y[m][n] is linear in every x[m][j], so a unit step of the
    # pinned layer gives dL/dx[m][j] exactly up to float64 rounding.
    for P in (2, 3):
        N, K, M = 13, 70, 4
        W, a, b = _three_path_layer(93, N, K) if P == 3 else (None, None, None)
        if P == 2:
            rng0 = np.random.default_rng(92)
            W = rng0.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
            a, b = inputs.scales(92, W)
        S = oracle.derive_signs(W, a, b, P=P)
        rng = np.random.default_rng(93 + P)
        x = rng.standard_normal((M, K))
        dY = rng.standard_normal((M, N))
        gx = oracle.grad_x(S, a, b, dY)
        L = lambda x_: float(np.sum(dY * oracle.layer(S, a, b, x_)))
        base = L(x)
        for m, j in [(0, 0), (1, 17), (M - 1, K - 1), (2, 40)]:
            x2 = x.copy(); x2[m, j] += 1.0
            assert L(x2) - base == pytest.approx(gx[m, j], rel=1e-9, abs=1e-9), (P, m, j)


def test_grad_x_hand_case_and_column_subset():
    # N=2, K=2, one path: W_hat = [[a0 s00 b0, a0 s01 b1], [a1 s10 b0, a1 s11 b1]]
    S = np.array([[[1, -1], [-1, -1]]], dtype=np.int8)
    a = np.array([[2.0, 3.0]]); b = np.array([[5.0, 7.0]])
    dY = np.array([[1.0, 10.0]])
    gx = oracle.grad_x(S, a, b, dY)
    np.testing.assert_array_equal(gx[0], [1 * 2 * 5 - 10 * 3 * 5, -1 * 2 * 7 - 10 * 3 * 7])
    # the column path: signs and b of columns (1,) only
    g1 = oracle.grad_x(S[:, :, [1]], a, b, dY, cols=np.array([1]))
    assert g1[0, 0] == gx[0, 1]


def test_grad_x_is_the_transposed_layer():
    # W_hat^T = sum_k b_k S_k^T a_k: the layer of the transposed signs with a and b exchanged
    N, K, M = 9, 45, 3
    rng = np.random.default_rng(95)
    W = rng.standard_normal((N, K)).astype(np.float32) * np.float32(0.02)
    a, b = inputs.scales(95, W)
    S = oracle.derive_signs(W, a, b)
    dY = rng.standard_normal((M, N))
    np.testing.assert_allclose(oracle.grad_x(S, a, b, dY),
                               oracle.layer(np.ascontiguousarray(S.transpose(0, 2, 1)), b, a, dY),
                               rtol=1e-12, atol=1e-12)
