/*
 * rabit.h -- C ABI of librabit, the RaBiT residual-binary linear layer on NVIDIA B200.
 *
 * The layer (RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs,
 * arXiv 2602.05367, sec. 4.1 "Multi-bit Approximation via Stacking"):
 *
 *     y = sum_{k=1..P} a_k (.) ( S_k . ( b_k (.) x ) )
 *
 * S_k in {+1,-1}^{N x K} are sign planes, a_k (length N) a per-output scale and b_k
 * (length K) a per-input scale (the paper's g_k and h_k).  The planes are derived in
 * sequence from one shared full-precision weight W (sec. 4.2 "The Coupled Forward Pass"):
 *     S_1 = sign(W),   R_1 = W - a_1 (.) S_1 (.) b_1,   S_2 = sign(R_1),
 * with sign(v) = +1 unless v < 0 (so +0, -0, NaN and an exact residual tie give +1), and
 * for three paths (the 3-bit case) once more: R_2 = R_1 - a_2 (.) S_2 (.) b_2, S_3 = sign(R_2).
 * P = 2 and P = 3 are implemented.
 *
 * Conventions shared by every call:
 *   - Every pointer argument is DEVICE memory owned by the caller (e.g. a torch tensor's
 *     data_ptr()).  The library allocates no device memory and keeps no per-call state;
 *     its only global state is a per-device fault word (rabit_read_fault), cached device
 *     attributes, and the fixed scratch buffer of rabit_gemm_noalloc (a static device
 *     array, not an allocation).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are asynchronous:
 *     they validate, enqueue and return.  Execution errors surface at the caller's next
 *     synchronisation, as for any CUDA launch.
 *   - Matrices are row-major; `ld*` arguments are row pitches in ELEMENTS.
 *   - Every call returns a rabit_status (0 = success).  Arguments are validated before
 *     anything is enqueued; a call that returns an error has enqueued nothing, except a
 *     RABIT_ERR_CUDA from a launch after the first of a call that enqueues several kernels
 *     (rabit_gemm, rabit_svid_init).  No call aborts, throws or prints.  RABIT_ERR_CUDA leaves the cudaError_t in
 *     rabit_last_cuda_error() (per calling thread).
 *   - The device current on the calling thread must be an sm_100 (B200-class) GPU; any
 *     other device gives RABIT_ERR_ARCH.
 */
#ifndef RABIT_H
#define RABIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define RABIT_API __attribute__((visibility("default")))
#else
#define RABIT_API
#endif

/* Element types accepted for W (derive) and x (gemv). */
typedef enum rabit_dtype { RABIT_F32 = 0, RABIT_BF16 = 1 } rabit_dtype;

typedef enum rabit_status {
    RABIT_OK = 0,
    RABIT_ERR_INVALID_ARG = -1,  /* null pointer, bad enum value */
    RABIT_ERR_ALIGNMENT = -2,    /* a pointer or pitch breaks the stated alignment */
    RABIT_ERR_SHAPE = -3,        /* N, K, M, batch or a pitch out of range */
    RABIT_ERR_UNSUPPORTED = -4,  /* valid request this build does not implement (P other than 2, 3) */
    RABIT_ERR_WORKSPACE = -5,    /* workspace missing or too small */
    RABIT_ERR_ARCH = -6,         /* current device is not sm_100 */
    RABIT_ERR_CUDA = -7,         /* a CUDA runtime call failed; see rabit_last_cuda_error() */
    RABIT_ERR_TIMEOUT = -8       /* reported by rabit_read_fault: a bounded device wait expired */
} rabit_status;

/*
 * Packed sign layout RABIT_LAYOUT_V2 (Appendix E.1 "Weight Packing": 32 columns per
 * uint32 word, +1 -> bit 0, -1 -> bit 1, the 2-bit case's two words grouped as a uint2 and
 * the 3-bit case's three words plus one padding word as a uint4).
 *   Kp = ceil(K/128)*128, Wr = Kp/32 groups of 32 columns per row, G = 2 (P = 2) or 4 (P = 3);
 *   column j sits at bit (j % 32) of group j/32, least significant bit first;
 *   word(k, n, w) = (n*Wr + w)*G + k    (path k < P, row n < N, group w < Wr).
 * Rows are stored one after another, and inside a row the paths' words of each 32-column
 * group sit side by side.  Padding columns (j >= K) and the padding word of a 3-path group
 * are 0; rows are not padded.  The buffer holds G*N*Wr uint32 words (rabit_packed_words)
 * and must be 16-byte aligned.
 */
#define RABIT_LAYOUT_V2 2
RABIT_API size_t rabit_packed_words(int N, int K, int P);

/*
 * rabit_derive_pack -- sec. 4.2 "The Coupled Forward Pass", steps 1-3, followed by the
 * Appendix E.1 packing.  For every n < N, j < K:
 *     s1 = sign(W[n][j]);  r1 = W[n][j] - a[0][n]*s1*b[0][j];  s2 = sign(r1)
 * and for P = 3 the same rule once more (sec. 4.1 stacking):
 *     r2 = r1 - a[1][n]*s2*b[1][j];  s3 = sign(r2)
 * sign(v) = +1 unless v < 0.  With P = 2, r1 is formed with one rounding (fused
 * multiply-add), so its sign is exact whenever the exact residual is nonzero and
 * |a[0][n]*b[0][j]| >= 2^-100.  With P = 3 both residuals are formed in binary64 (each
 * product exact, each subtraction rounded once).  Writes every word of the packed buffer,
 * padding included (so it never needs clearing).  Scales are read, never written: they stay
 * caller-owned learnable parameters.
 *   W       [N][ldw] fp32 (w_dtype RABIT_F32) or bf16 (RABIT_BF16), ldw >= K
 *   a       [P][N] fp32, b [P][K] fp32 (paths 1..P-1 are read; the last path needs no scale)
 *   packed  rabit_packed_words(N, K, P) uint32, 16-byte aligned (output)
 * Errors: INVALID_ARG (null, bad dtype), SHAPE (N, K < 1, ldw < K), UNSUPPORTED (P not 2 or 3),
 *         ALIGNMENT (packed), ARCH, CUDA.
 */
RABIT_API int rabit_derive_pack(const void *W, int w_dtype, int N, int K, int ldw, int P,
                      const float *a, const float *b, uint32_t *packed, void *stream);

/*
 * rabit_gemv -- decode path, batch 1..16 (sec. 4.1 stacking executed per path as in
 * Appendix E.1 "Compute Pipeline": paths computed in parallel, signs applied without
 * multiplication, output scale applied last):
 *     y[beta][n] = sum_k a[k][n] * sum_j S_k[n][j] * b[k][j] * x[beta][j]
 * Two implementations, chosen by batch (RABIT_GEMV_KERNEL=dp2a or =tc in the environment
 * forces one):
 *   batch <= 4: one CUDA-core kernel.  z = b_k * x is quantised per 32-column group to 13
 *     bits (two 13-bit slices for fp32 x) with a power-of-two scale; the signs select which
 *     z enter integer dot products (dp2a), exact in 32-bit.
 *   batch > 4 (and every rabit_gemv_grouped call): the tensor-core path.  The signs enter
 *     tcgen05.mma as 4-bit +-1 values and z as balanced base-4 digits of zq = rint(z * 2^e)
 *     with one power-of-two scale per (path, batch row), |zq| below 2^15 (bf16 x) or 2^23
 *     (fp32 x); the sign sums of zq are exact.  Prep kernels write the digits and scales
 *     to the workspace, then the main kernel streams the signs.
 * Results are deterministic.
 *   packed  RABIT_LAYOUT_V2 buffer of N x K, P paths (input)
 *   a [P][N], b [P][K] fp32
 *   x       [batch][ldx], bf16 (x_dtype RABIT_BF16) or fp32 (RABIT_F32), ldx >= K
 *   y       [batch][ldy] fp32 (output, fully overwritten for n < N), ldy >= N
 *   workspace  at least rabit_gemv_workspace_bytes(N, K, P, batch) bytes (enough for either
 *              x type), 16-byte aligned, caller-owned: about 5.2 MB of partial sums for the
 *              row tiles that several CTAs share, one counter per 128-row tile, the scales,
 *              and the digits (P * K * batch bytes for bf16 x, 1.5 times that for fp32 x,
 *              rounded up).  It needs no initialisation: every call writes what it reads.
 *              Calls that share a workspace must not overlap on the GPU (order them on one
 *              stream).
 * Accuracy (normwise, max|y - y_exact| / max|y_exact|): <= 2e-3 for bf16 x, <= 1e-5 for
 * fp32 x.  Errors: INVALID_ARG, SHAPE (batch outside 1..16, pitches), UNSUPPORTED,
 * ALIGNMENT (packed, workspace), WORKSPACE, ARCH, CUDA.  A device-side wait that expires
 * (it cannot in correct operation) ends the kernel early and is reported by
 * rabit_read_fault as RABIT_ERR_TIMEOUT.
 */
RABIT_API size_t rabit_gemv_workspace_bytes(int N, int K, int P, int batch);
RABIT_API int rabit_gemv(const uint32_t *packed, const float *a, const float *b, int N, int K, int P,
               const void *x, int x_dtype, int batch, int ldx, float *y, int ldy,
               void *workspace, size_t workspace_bytes, void *stream);

/*
 * rabit_gemv_grouped -- rabit_gemv for up to RABIT_GEMV_MAX_GROUP independent layers in one
 * launch, e.g. the projections of a decoder block that read the same activation (query, key
 * and value; gate and up).  Each layer computes exactly what rabit_gemv computes for it; the
 * launch shares the fixed costs (setup, the dependency on the previous kernel, the final
 * sums) and balances all layers' work over the SMs.  The layers share P, the activation type
 * and the batch; each has its own signs, scales, x and y (which must not overlap another
 * layer's y).
 *   layers     host array of `count` descriptions (1 <= count <= RABIT_GEMV_MAX_GROUP); the
 *              pointers inside are device pointers with the layouts of rabit_gemv
 *   workspace  at least rabit_gemv_grouped_workspace_bytes(layers, count, P, x_dtype, batch)
 *              bytes, 16-byte aligned, with the rules of rabit_gemv's workspace (0 from the
 *              size call means invalid arguments)
 * Errors: as rabit_gemv, plus INVALID_ARG for a null `layers` or count out of range.
 */
#define RABIT_GEMV_MAX_GROUP 8
typedef struct rabit_gemv_layer {
    const uint32_t *packed;   /* RABIT_LAYOUT_V2 signs of N x K, P paths */
    const float *a;           /* [P][N] */
    const float *b;           /* [P][K] */
    int N, K;
    const void *x;            /* [batch][ldx] */
    int ldx;
    float *y;                 /* [batch][ldy] */
    int ldy;
} rabit_gemv_layer;
RABIT_API size_t rabit_gemv_grouped_workspace_bytes(const rabit_gemv_layer *layers, int count, int P,
                                                    int x_dtype, int batch);
RABIT_API int rabit_gemv_grouped(const rabit_gemv_layer *layers, int count, int P, int x_dtype, int batch,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * rabit_gemm -- prefill / QAT forward path at large M (sec. 4.2: the forward pass uses
 * W_hat^(2)), the same contraction as rabit_gemv for M tokens:
 *     y[m][n] = sum_k a[k][n] * sum_j S_k[n][j] * b[k][j] * x[m][j]
 * computed on the tensor cores: the signs are expanded to fp16 +-a[k][n] in tensor memory,
 * the activations enter as fp16(x (.) b_k) and products accumulate in fp32.
 *   packed  RABIT_LAYOUT_V2 buffer (input); a [P][N], b [P][K] fp32
 *   x_bf16  [M][ldx] bf16, 16-byte aligned, ldx >= K and ldx % 8 == 0
 *   y       [M][ldy] fp32 (output, fully overwritten for m < M, n < N), ldy >= N
 *   workspace  scratch of at least rabit_gemm_workspace_bytes(N, K, P, M) bytes,
 *              256-byte aligned, owned by the caller; contents need no initialisation
 *              and are garbage afterwards.  Calls that share a workspace must not overlap.
 * Accuracy: <= 2e-3 normwise, provided every |a[k][n]| lies in fp16's normal range
 * [6.2e-5, 65504] and |x*b| < 65504.  Errors: INVALID_ARG, SHAPE, UNSUPPORTED, ALIGNMENT,
 * WORKSPACE, ARCH, CUDA.  A device-side wait that expires (it cannot in correct operation)
 * ends the kernel early and is reported by rabit_read_fault as RABIT_ERR_TIMEOUT.
 */
RABIT_API size_t rabit_gemm_workspace_bytes(int N, int K, int P, int M);
RABIT_API int rabit_gemm(const uint32_t *packed, const float *a, const float *b, int N, int K, int P,
               const uint16_t *x_bf16, int M, int ldx, float *y, int ldy,
               void *workspace, size_t workspace_bytes, void *stream);

/*
 * rabit_gemm_grouped -- rabit_gemm for up to RABIT_GEMM_MAX_GROUP independent layers with the
 * same token count M in one persistent launch (e.g. the gate and up projections of an MLP,
 * which read the same x).  Each layer computes exactly what rabit_gemm computes for it; the
 * layers' tiles share the CTAs, dealt longest contraction first to the least loaded CTA, so
 * the last wave of one layer no longer leaves SMs idle.
 *   layers     host array of `count` descriptions (struct rabit_gemv_layer): packed, a, b, N,
 *              K as for rabit_gemm; x = bf16 [M][ldx] (16-byte aligned, ldx >= K and a
 *              multiple of 8); y = fp32 [M][ldy] (output), ldy >= N
 *   workspace  at least rabit_gemm_grouped_workspace_bytes(layers, count, P, M) bytes,
 *              256-byte aligned (0 from the size call means invalid arguments)
 * Accuracy and errors: those of rabit_gemm, plus INVALID_ARG for a null `layers` or count
 * out of range.
 */
#define RABIT_GEMM_MAX_GROUP 4
RABIT_API size_t rabit_gemm_grouped_workspace_bytes(const rabit_gemv_layer *layers, int count, int P, int M);
RABIT_API int rabit_gemm_grouped(const rabit_gemv_layer *layers, int count, int P, int M, void *workspace,
                                 size_t workspace_bytes, void *stream);

/*
 * rabit_transpose_pack -- the packed sign planes of W^T from those of W, for the input
 * gradient (sec. 4.1: W_hat = sum_k a_k (.) S_k (.) b_k, so W_hat^T = sum_k b_k (.) S_k^T (.) a_k
 * is a stacked layer of the same form, K x N, with a and b exchanged):
 *     packed_t holds S_k^T[j][n] = S_k[n][j] for every path k, j < K, n < N.
 *   packed    RABIT_LAYOUT_V2 buffer of N x K, P paths (input)
 *   packed_t  RABIT_LAYOUT_V2 buffer of K x N, P paths: rabit_packed_words(K, N, P) uint32,
 *             16-byte aligned (output, every word written, padding columns n >= N zero)
 * Bit-exact.  Errors: INVALID_ARG, SHAPE, UNSUPPORTED (P not 2 or 3), ALIGNMENT, ARCH, CUDA.
 */
RABIT_API int rabit_transpose_pack(const uint32_t *packed, int N, int K, int P, uint32_t *packed_t,
                                   void *stream);

/*
 * rabit_grad_x -- input gradient of the layer for M tokens (the backward of sec. 4.1's
 * stacked layer with the signs held fixed):
 *     grad_x[m][j] = sum_n dY[m][n] W_hat[n][j] = sum_k b_k[j] sum_n S_k[n][j] a_k[n] dY[m][n]
 * computed as rabit_gemm of the transposed layer: signs from rabit_transpose_pack, per-output
 * scale b_k, per-input scale a_k, activations dY (on tcgen05, fp32 accumulation).
 *   packed_t  RABIT_LAYOUT_V2 of K x N from rabit_transpose_pack (input)
 *   a [P][N], b [P][K] fp32 (the layer's scales, as for rabit_gemm)
 *   dy_bf16   [M][ldd] bf16, ldd >= N and a multiple of 8, 16-byte aligned
 *   grad_x    [M][ldg] fp32 (output), ldg >= K
 *   workspace at least rabit_gemm_workspace_bytes(K, N, P, M) bytes, 256-byte aligned
 * Accuracy (normwise): <= 2e-3, the bar of rabit_gemm.  Errors: those of rabit_gemm.
 */
RABIT_API int rabit_grad_x(const uint32_t *packed_t, const float *a, const float *b, int N, int K, int P,
                           const uint16_t *dy_bf16, int M, int ldd, float *grad_x, int ldg,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * rabit_gemm_noalloc -- the same computation as rabit_gemm, for callers that are not allowed
 * to allocate device memory and so cannot hand rabit_gemm a workspace.  Examples: a plugin
 * loaded into an inference engine that owns every device allocation and gives the plugin
 * no allocator, or a latency-critical serving loop that must never call cudaMalloc (it can
 * synchronise the whole device and fails while another thread captures a stream in global
 * mode).  The paper has no counterpart to this call; it exists only for such callers.
 *
 * The scratch rabit_gemm would take from `workspace` (the fp16 x (.) b_k operand) lives
 * instead in one fixed device buffer of RABIT_GEMM_NOALLOC_SCRATCH_BYTES inside the
 * library, which every GPU that loads librabit holds until the process exits.  Nothing is
 * allocated by this call.
 *   - Requests that need more scratch than that (rabit_gemm_workspace_bytes(N, K, P, M) >
 *     RABIT_GEMM_NOALLOC_SCRATCH_BYTES, e.g. more than 512 tokens at K = 4096) are rejected
 *     with RABIT_ERR_WORKSPACE before anything is enqueued; use rabit_gemm for them.
 *   - All calls on a device share the one buffer and leave their data in it.  The call
 *     overwrites every byte it reads, so nothing needs clearing, but two calls that can run
 *     at the same time on the GPU (different streams without ordering between them) race on
 *     the buffer and give wrong results: order such calls on one stream or with events.
 *   - The first call on each device looks up the buffer's device address; make that first
 *     call before any stream capture begins.
 * Arguments, accuracy and the other errors are those of rabit_gemm.
 */
#define RABIT_GEMM_NOALLOC_SCRATCH_BYTES (8u << 20)
RABIT_API int rabit_gemm_noalloc(const uint32_t *packed, const float *a, const float *b, int N,
                                 int K, int P, const uint16_t *x_bf16, int M, int ldx, float *y,
                                 int ldy, void *stream);

/*
 * rabit_scale_grads -- backward of the layer's scales for a given G = dL/dW_hat (the QAT
 * backward of sec. 4.2: the shared weight takes G unchanged, the signs are held fixed, and
 * the learnable scales get the chain rule of sec. 4.1's W_hat = sum_k a_k (.) S_k (.) b_k;
 * the page text loses the update formula, so the plain chain rule is taken):
 *     grad_a[k][n] = sum_j G[n][j] * S_k[n][j] * b[k][j]
 *     grad_b[k][j] = sum_n G[n][j] * a[k][n] * S_k[n][j]
 * G itself is the dense product dY^T X of the layer's output gradient and input, which the
 * caller forms (a plain GEMM).  Accumulates in fp32 in a fixed order (deterministic).
 *   G        [N][ldg] fp32, ldg >= K (input)
 *   packed   RABIT_LAYOUT_V2 signs of N x K, P paths (input); a [P][N], b [P][K] fp32
 *   grad_a   [P][N] fp32, grad_b [P][K] fp32 (outputs, fully overwritten)
 *   workspace  at least rabit_scale_grads_workspace_bytes(N, K, P) bytes, 16-byte aligned,
 *              caller-owned; no initialisation needed.  Calls sharing it must not overlap.
 * Errors: INVALID_ARG (null), SHAPE (N, K < 1, ldg < K), UNSUPPORTED (P not 2 or 3),
 *         ALIGNMENT (packed, G, workspace), WORKSPACE, ARCH, CUDA.
 */
RABIT_API size_t rabit_scale_grads_workspace_bytes(int N, int K, int P);
RABIT_API int rabit_scale_grads(const float *G, int ldg, const uint32_t *packed, const float *a,
                                const float *b, int N, int K, int P, float *grad_a, float *grad_b,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * rabit_svid_init -- initialisation of the layer's paths and scales (sec. 4.3 "Stable
 * Initialization for Functional Preservation"): Iterative Residual SVID on the
 * importance-preconditioned weight, scales mapped back to the original domain.
 *     W' = s_out^alpha_out (.) W (.) s_in^alpha_in          (row scale s_out, column scale s_in)
 *     for t = 1..T, i = 1..P:  R_i = W' - sum_{j != i} What_j   (latest update of each path,
 *                                                           What_j = 0 before its first)
 *         B_i = sign(R_i),  g_i' h_i'^T = sigma u v^T, the leading rank-1 part of |R_i|,
 *         g_i' = sqrt(sigma) u,  h_i' = sqrt(sigma) v,  What_i = g_i' (.) B_i (.) h_i'
 *     a[i] = g_i' / s_out^alpha_out,   b[i] = h_i' / s_in^alpha_in
 * SVID is read as the sign-value-independent decomposition (sign plus the best rank-1
 * approximation of |R|), which the pages cite but do not define.  The leading singular
 * pair comes from power steps per update (fp32 sums, double norms, every sum in a fixed
 * order, so the result is deterministic), warm-started from the path's pair of the previous
 * iteration (uniform vectors at t = 1): at most `power_iters` of them, fewer when
 * power_tol > 0 and a step moved both unit vectors u and v by at most power_tol (Euclidean
 * norm): the step after it is the last (power_tol = 0: exactly power_iters steps).  Every
 * step of an update runs inside one cooperative launch (one CTA per SM, two grid barriers
 * per step, each wait bounded: an expired wait sets the fault word, see rabit_read_fault).
 * The pages use T = 20.
 *   W        [N][ldw] fp32, ldw >= K (input)
 *   s_in [K], s_out [N]  positive fp32 calibration statistics (inputs; the reconstruction
 *            sum_i a_i (.) B_i (.) b_i does not depend on their normalisation);
 *            non-positive or non-finite entries give undefined (inf or NaN) outputs
 *   a [P][N], b [P][K] fp32 (outputs, fully overwritten)
 *   packed   RABIT_LAYOUT_V2 buffer of N x K, P paths: the final B_i (output, every word
 *            written, padding included)
 *   workspace  at least rabit_svid_init_workspace_bytes(N, K, P) bytes (about 4*N*K),
 *              256-byte aligned, caller-owned, no initialisation needed.  Calls sharing it
 *              must not overlap.
 * Enqueues 2 + 2 * T * P kernels on `stream` (a residual pass and a power launch per update)
 * and returns.
 * Errors: INVALID_ARG (null, non-finite alpha, power_tol negative or not finite), SHAPE (N, K < 1,
 *         ldw < K, T or power_iters outside 1..RABIT_SVID_MAX_ITERS), UNSUPPORTED (P not 2 or 3),
 *         ALIGNMENT (packed, workspace), WORKSPACE, ARCH, CUDA.
 */
#define RABIT_SVID_MAX_ITERS 1000
RABIT_API size_t rabit_svid_init_workspace_bytes(int N, int K, int P);
RABIT_API int rabit_svid_init(const float *W, int N, int K, int ldw, int P, int T, int power_iters,
                              float power_tol, const float *s_in, const float *s_out, float alpha_in, float alpha_out,
                              float *a, float *b, uint32_t *packed, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * rabit_read_fault -- synchronise `stream` and read the current device's fault word
 * (bit set by a kernel whose bounded wait expired).  Returns RABIT_OK when no fault is
 * recorded, RABIT_ERR_TIMEOUT when one is, RABIT_ERR_CUDA on a CUDA failure.  `flags`
 * (may be NULL) receives the raw word; clear != 0 resets it to 0 afterwards.
 */
RABIT_API int rabit_read_fault(void *stream, uint32_t *flags, int clear);

/* Last cudaError_t seen by a librabit call on this thread (0 if none). */
RABIT_API int rabit_last_cuda_error(void);

/* Static, human-readable name of a rabit_status value. */
RABIT_API const char *rabit_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* RABIT_H */
