/*
 * rabit_oracle.c -- float64 CPU oracle for the RaBiT residual-binary linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct statement of what
 * the librabit CUDA path must compute.  It is used by tests/, by the smoke check and by
 * bench.py's CPU-baseline leg, and by nothing else.  It shares no code, header, table or
 * constant with the CUDA library and includes nothing from it.
 *
 * Source of every definition: "RaBiT: Residual-Aware Binarization Training for Accurate
 * and Efficient LLMs" (You et al., arXiv 2602.05367):
 *   - sec. 4.1, "Binary Building Blocks":  W_hat = g (.) B (.) h, B in {+-1}^{dout x din},
 *     g per output row, h per input column (sec. 4.3 maps g to s_out and h to s_in);
 *   - sec. 4.1, "Multi-bit Approximation via Stacking": W_hat^(k) = sum_i g_i (.) B_i (.) h_i;
 *   - sec. 4.2, "The Coupled Forward Pass", steps 1-3: B_1 = sign(W_FP),
 *     R_1 = W_FP - W_hat_1, B_2 = sign(R_1);
 *   - Appendix E.1, "Weight Packing": 32 columns per uint32, +1 -> bit 0, -1 -> bit 1,
 *     the paths' words of one 32-column group grouped together (uint2 for 2 bits).
 * In this library's names a_k is the per-output scale (g_k) and b_k the per-input scale (h_k).
 *
 * Readings where the pages are silent:
 *   - sign(v) = +1 unless v < 0, so +0, -0 and NaN binarize to +1 (the pages map only +-1);
 *   - column j of a 32-column group sits at bit (j % 32), least significant bit first;
 *   - the arrangement is the RABIT_LAYOUT_V2 formula below: rows one after another, each
 *     row's 32-column groups in order, each group holding the P paths' words side by side.
 *     (The pages also interleave rows in warp-sized groups for a kernel that maps lanes to
 *     rows; the kernel this oracle checks maps lanes to column groups, so rows stay whole.)
 *
 * Precision: every input is an fp32 (or bf16, widened exactly) value; the product a*b of
 * two fp32 values is exact in binary64, so the residual W - a*s*b is rounded once and its
 * sign is exact.  Layer outputs are plain float64 sums.
 *
 * Parallelism: the outer loops over rows carry an OpenMP pragma so that the timed CPU
 * baseline uses the host's cores; each output element is still one plain sequential sum.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* sign as the pages use it, with the tie/zero reading stated above */
static inline int8_t oracle_sign(double v) { return (v < 0.0) ? (int8_t)-1 : (int8_t)1; }

/*
 * Coupled forward derivation (sec. 4.2, steps 1-3), for rows [n0, n1) of W.
 *   W   : float64 [*][ldw], row n at W + n*ldw (values widened exactly from fp32/bf16)
 *   a   : float64 [P][N]   per-output scales a_k (only paths 1..P-1 are read)
 *   b   : float64 [P][K]   per-input scales  b_k (only paths 1..P-1 are read)
 *   S   : int8    [P][n1-n0][K] output signs (+1/-1), row n stored at (n - n0)
 * Path 1 binarizes W; path p binarizes the residual left after paths 1..p-1
 * (sec. 4.1 stacking applied to the sec. 4.2 residual rule; P = 2 is the paper's 2-bit case).
 */
ORACLE_API void oracle_derive_signs(const double *W, int64_t N, int64_t K, int64_t ldw,
                                    int P, const double *a, const double *b,
                                    int64_t n0, int64_t n1, int8_t *S)
{
    const int64_t rows = n1 - n0;
    #pragma omp parallel for schedule(static)
    for (int64_t n = n0; n < n1; ++n) {
        for (int64_t j = 0; j < K; ++j) {
            double r = W[n * ldw + j];                 /* R_0 = W_FP */
            for (int p = 0; p < P; ++p) {
                int8_t s = oracle_sign(r);              /* B_{p+1} = sign(R_p) */
                S[((int64_t)p * rows + (n - n0)) * K + j] = s;
                /* R_{p+1} = R_p - a_{p+1}[n] * s * b_{p+1}[j] */
                r = r - a[(int64_t)p * N + n] * (double)s * b[(int64_t)p * K + j];
            }
        }
    }
}

/* Padded column count of the packed layout: columns to a multiple of 128.  Rows are not padded. */
ORACLE_API int64_t oracle_padded_cols(int64_t K) { return ((K + 127) / 128) * 128; }

/* Words of one 32-column group: the P paths' words side by side, padded to a power of two
   (P = 2 -> 2 words, the "uint2" grouping of Appendix E.1). */
static int64_t oracle_group_words(int P) { return P <= 1 ? 1 : (P == 2 ? 2 : 4); }

ORACLE_API int64_t oracle_packed_words(int64_t N, int64_t K, int P)
{
    return N * (oracle_padded_cols(K) / 32) * oracle_group_words(P);
}

/*
 * RABIT_LAYOUT_V2 word index of (path k, row n, 32-column word w), P paths:
 *   index = (n * (Kp/32) + w) * G + k,   G = words per group (2 for P = 2)
 * i.e. rows are stored one after another; inside a row, each 32-column group holds the
 * P paths' words next to each other (Appendix E.1 groups the 2-bit case's words as uint2).
 */
ORACLE_API int64_t oracle_word_index(int k, int64_t n, int64_t w, int64_t K, int P)
{
    return (n * (oracle_padded_cols(K) / 32) + w) * oracle_group_words(P) + k;
}

/*
 * Pack signs (Appendix E.1 "Weight Packing"): bit (j % 32) of word j/32 is 1 iff S = -1.
 * Padding columns (and the padding word of a 3-path group) stay 0.  S is [P][N][K]; out has oracle_packed_words().
 */
ORACLE_API void oracle_pack(const int8_t *S, int64_t N, int64_t K, int P, uint32_t *out)
{
    memset(out, 0, sizeof(uint32_t) * (size_t)oracle_packed_words(N, K, P));
    for (int k = 0; k < P; ++k)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < K; ++j)
                if (S[((int64_t)k * N + n) * K + j] == -1)
                    out[oracle_word_index(k, n, j / 32, K, P)] |= (uint32_t)1u << (j % 32);
}

/* Inverse of oracle_pack: bit 1 -> -1, bit 0 -> +1.  S is [P][N][K]. */
ORACLE_API void oracle_unpack(const uint32_t *packed, int64_t N, int64_t K, int P, int8_t *S)
{
    for (int k = 0; k < P; ++k)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t j = 0; j < K; ++j) {
                uint32_t word = packed[oracle_word_index(k, n, j / 32, K, P)];
                S[((int64_t)k * N + n) * K + j] = ((word >> (j % 32)) & 1u) ? (int8_t)-1 : (int8_t)1;
            }
}

/*
 * Residual-binary linear layer (sec. 4.1 stacking, executed per path as in sec. 4.2's
 * inference note and Appendix E.1's per-path computation):
 *   y[beta][i] = sum_k a_k[n_i] * sum_j S_k[i][j] * b_k[j] * x[beta][j]
 * for the rows whose signs are given.
 *   S    : int8 [P][R][K] signs of R rows; row i of S is output row rows[i] (rows may be
 *          NULL, meaning rows[i] = i)
 *   a    : float64 [P][N], b : float64 [P][K]
 *   x    : float64 [B][ldx] activations (widened exactly from bf16/fp32)
 *   y    : float64 [B][R] output, y[beta][i] belongs to output row rows[i]
 */
ORACLE_API void oracle_layer(const int8_t *S, int64_t R, const int64_t *rows, int64_t N,
                             int64_t K, int P, const double *a, const double *b,
                             const double *x, int64_t B, int64_t ldx, double *y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < R; ++i) {
        const int64_t n = rows ? rows[i] : i;
        for (int64_t beta = 0; beta < B; ++beta) {
            double acc = 0.0;
            for (int k = 0; k < P; ++k) {
                const int8_t *srow = S + ((int64_t)k * R + i) * K;
                const double *bk = b + (int64_t)k * K;
                const double *xb = x + beta * ldx;
                double t = 0.0;
                for (int64_t j = 0; j < K; ++j)
                    t += (double)srow[j] * bk[j] * xb[j];
                acc += a[(int64_t)k * N + n] * t;
            }
            y[beta * R + i] = acc;
        }
    }
}

/*
 * Gradients of the layer's scales for a given gradient G = dL/dW_hat (the straight-through
 * estimator passes G to the shared weight unchanged and holds the signs fixed; the pages'
 * sec. 4.2 update formula is lost in extraction, so this is the plain chain rule applied to
 * sec. 4.1's W_hat = sum_k a_k (.) S_k (.) b_k):
 *   ga[k][n] = sum_j G[n][j] * S_k[n][j] * b_k[j]
 *   gb[k][j] = sum_n G[n][j] * a_k[n] * S_k[n][j]
 *   G  : float64 [N][K];  S : int8 [P][N][K];  a : [P][N];  b : [P][K]
 *   ga : float64 [P][N];  gb : float64 [P][K]
 */
ORACLE_API void oracle_scale_grads(const double *G, int64_t N, int64_t K, const int8_t *S, int P,
                                   const double *a, const double *b, double *ga, double *gb)
{
    for (int k = 0; k < P; ++k) {
        const int8_t *Sk = S + (int64_t)k * N * K;
        #pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            double t = 0.0;
            for (int64_t j = 0; j < K; ++j)
                t += G[n * K + j] * (double)Sk[n * K + j] * b[(int64_t)k * K + j];
            ga[(int64_t)k * N + n] = t;
        }
        #pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < K; ++j) {
            double t = 0.0;
            for (int64_t n = 0; n < N; ++n)
                t += G[n * K + j] * a[(int64_t)k * N + n] * (double)Sk[n * K + j];
            gb[(int64_t)k * K + j] = t;
        }
    }
}

/*
 * Input gradient of the stacked layer (sec. 4.1) with the signs held fixed: for
 * y = W_hat x with W_hat[n][j] = sum_k a_k[n] S_k[n][j] b_k[j],
 *   gx[m][c] = dL/dx[m][j_c] = sum_n dY[m][n] W_hat[n][j_c]
 *            = sum_k b_k[j_c] sum_n dY[m][n] a_k[n] S_k[n][c]
 *   S  : int8 [P][N][C], the signs of the C columns j_c (all rows n)
 *   a  : [P][N];  bc : [P][C] (b_k at the C columns);  dY : float64 [M][ldd]
 *   gx : float64 [M][C]
 */
ORACLE_API void oracle_grad_x(const int8_t *S, int64_t N, int64_t C, int P, const double *a,
                              const double *bc, const double *dY, int64_t M, int64_t ldd, double *gx)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int k = 0; k < P; ++k) {
                const int8_t *Sk = S + (int64_t)k * N * C;
                double t = 0.0;
                for (int64_t n = 0; n < N; ++n)
                    t += dY[m * ldd + n] * a[(int64_t)k * N + n] * (double)Sk[n * C + c];
                acc += bc[(int64_t)k * C + c] * t;
            }
            gx[m * C + c] = acc;
        }
    }
}

/* Number of OpenMP threads the parallel loops above use (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
ORACLE_API int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
ORACLE_API int oracle_num_threads(void) { return 1; }
#endif
