// svid.cu -- initialisation of the residual-binary layer: Iterative Residual SVID on the
// importance-preconditioned weight.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs", sec. 4.3
// "Stable Initialization for Functional Preservation":
//     W' = s_out^alpha_out (.) W (.) s_in^alpha_in
//     for t = 1..T, paths i = 1..P in order:
//         R_i = W' - sum_{j != i} What_j        (the latest update of every other path)
//         (B_i, g_i', h_i') = SVID(R_i),   What_i = g_i' (.) B_i (.) h_i'
//     g_i = s_out^-alpha_out (.) g_i',   h_i = s_in^-alpha_in (.) h_i'
// with What_j = 0 before a path's first update (iteration 1 is the greedy decomposition).
// SVID(R) = (sign R, g', h'), g' h'^T the leading rank-1 part sigma u v^T of |R| split as
// sqrt(sigma) u, sqrt(sigma) v; the pages leave SVID to the cited prior work, whose
// sign-value-independent decomposition this is.
//
// Design (HBM-bound passes, CUDA cores):
//  * Residual pass, once per (t, i): a warp per 32-column group reads the group's W values
//    (128 contiguous bytes), the other paths' packed words (one broadcast load each) and
//    scales, writes R (fp32, rows 16-byte aligned) and a ballot of the signs straight into
//    path i of the packed output -- the same layout the decode and prefill kernels read.
//  * Power iteration for (sigma, u, v), warm-started from the path's vectors of the previous
//    iteration.  With G = R and S = sign(R), the scale-gradient kernels compute exactly
//    |R| v (their grad_a: sum_j G S b) and |R|^T u (their grad_b: sum_n G a S), so each
//    power step is one deterministic pass over R by those kernels, followed by a one-CTA
//    kernel that normalises u and v (and on the last step writes sqrt(sigma) u, sqrt(sigma) v).
//  * u and v start positive and |R| is nonnegative, so they stay the Perron vectors.
#include <algorithm>
#include <cmath>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kThreads = 256;
constexpr int kNormThreads = 1024;

__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}

// Workspace carve-up (every part 256-byte aligned).
struct SvidWs {
    float *R;          // [N][ldr] residual of the path being updated
    uint2 *ps;         // [N][Wr] two-path packed words, both = sign(R) (operand of the power step)
    void *sg;          // scale-gradient workspace (two paths)
    float *so, *si;    // s_out^alpha_out [N], s_in^alpha_in [K]
    float *gp, *hp;    // g' [P][N], h' [P][K] in the preconditioned domain
    float *U, *V;      // unit singular vectors per path [P][N], [P][K] (warm starts)
    float *avec, *bvec;      // power-step operands [2][N], [2][K]; the second row stays 0
    float *grad_a, *grad_b;  // power-step results [2][N], [2][K]
    size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

__host__ __device__ inline int64_t residual_pitch(int K) { return (static_cast<int64_t>(K) + 3) / 4 * 4; }

SvidWs svid_layout(void *base, int N, int K, int P) {
    SvidWs w{};
    const int64_t Wr = padded_cols(K) / 32;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return reinterpret_cast<char *>(reinterpret_cast<uintptr_t>(base) + o);
    };
    w.R = reinterpret_cast<float *>(take(static_cast<size_t>(N) * residual_pitch(K) * 4));
    w.ps = reinterpret_cast<uint2 *>(take(static_cast<size_t>(N) * Wr * 8));
    w.sg = take(scale_grads_workspace_bytes(N, K, 2));
    w.so = reinterpret_cast<float *>(take(static_cast<size_t>(N) * 4));
    w.si = reinterpret_cast<float *>(take(static_cast<size_t>(K) * 4));
    w.gp = reinterpret_cast<float *>(take(static_cast<size_t>(P) * N * 4));
    w.hp = reinterpret_cast<float *>(take(static_cast<size_t>(P) * K * 4));
    w.U = reinterpret_cast<float *>(take(static_cast<size_t>(P) * N * 4));
    w.V = reinterpret_cast<float *>(take(static_cast<size_t>(P) * K * 4));
    w.avec = reinterpret_cast<float *>(take(static_cast<size_t>(2) * N * 4));
    w.bvec = reinterpret_cast<float *>(take(static_cast<size_t>(2) * K * 4));
    w.grad_a = reinterpret_cast<float *>(take(static_cast<size_t>(2) * N * 4));
    w.grad_b = reinterpret_cast<float *>(take(static_cast<size_t>(2) * K * 4));
    w.total = off;
    return w;
}

// Preconditioning vectors, zero scales, uniform unit start vectors, zero second operand rows.
__global__ void __launch_bounds__(kThreads)
svid_prep_kernel(const float *__restrict__ s_in, const float *__restrict__ s_out, float alpha_in,
                 float alpha_out, int N, int K, int P, SvidWs w) {
    pdl_enter();
    const float un = 1.0f / sqrtf(static_cast<float>(N)), vk = 1.0f / sqrtf(static_cast<float>(K));
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < N; t += stride) {
        w.so[t] = powf(__ldg(s_out + t), alpha_out);
        for (int p = 0; p < P; ++p) {
            w.gp[p * static_cast<int64_t>(N) + t] = 0.0f;
            w.U[p * static_cast<int64_t>(N) + t] = un;
        }
        w.avec[N + t] = 0.0f;
    }
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < K; t += stride) {
        w.si[t] = powf(__ldg(s_in + t), alpha_in);
        for (int p = 0; p < P; ++p) {
            w.hp[p * static_cast<int64_t>(K) + t] = 0.0f;
            w.V[p * static_cast<int64_t>(K) + t] = vk;
        }
        w.bvec[K + t] = 0.0f;
    }
}

// R_i = W' - sum_{p != i} g_p' (.) B_p (.) h_p', its signs into path i of the packed output and
// into the power-step operand; also loads path i's start vectors into the operand rows.
template <int kP>
__global__ void __launch_bounds__(kThreads)
svid_residual_kernel(const float *__restrict__ W, int ldw, int N, int K, int Wr, int path,
                     uint32_t *__restrict__ packed, SvidWs w) {
    constexpr int G = kP == 2 ? 2 : 4;  // words per 32-column group in the packed layout
    pdl_enter();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t groups = static_cast<int64_t>(N) * Wr;
    const int64_t ldr = residual_pitch(K);
    for (int64_t gi = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; gi < groups;
         gi += nwarps) {
        const int n = static_cast<int>(gi / Wr);
        const int j = static_cast<int>(gi - static_cast<int64_t>(n) * Wr) * 32 + lane;
        const bool ok = j < K;
        float r = 0.0f;
        if (ok) {
            r = w.so[n] * __ldg(W + static_cast<int64_t>(n) * ldw + j) * w.si[j];
#pragma unroll
            for (int p = 0; p < kP; ++p) {
                if (p == path) continue;
                const bool neg = (packed[gi * G + p] >> lane) & 1u;
                const float m = w.gp[p * static_cast<int64_t>(N) + n] * w.hp[p * static_cast<int64_t>(K) + j];
                r = neg ? r + m : r - m;
            }
            w.R[static_cast<int64_t>(n) * ldr + j] = r;
        }
        const uint32_t bits = __ballot_sync(0xffffffffu, ok && r < 0.0f);   // sign(v) = -1 iff v < 0
        if (lane == 0) {
            packed[gi * G + path] = bits;
            if (kP == 3 && path == 0) packed[gi * G + 3] = 0u;                 // padding word
            w.ps[gi] = make_uint2(bits, bits);
        }
    }
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < N; t += stride)
        w.avec[t] = w.U[path * static_cast<int64_t>(N) + t];
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < K; t += stride)
        w.bvec[t] = w.V[path * static_cast<int64_t>(K) + t];
}

// Sum of v over the CTA in a fixed order (deterministic); every thread gets the total.
__device__ double cta_sum(double v, double *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();                        // red may still be read from a previous call
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double s = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) s += red[i];
    return s;
}

// One CTA: u = |R| v / || |R| v ||, v = |R|^T u / || . ||.  On the last power step of a path
// the scales g' = sqrt(sigma) u, h' = sqrt(sigma) v (sigma = || |R| v || for the unit v fed
// in) and the warm-start vectors are stored.  A zero product (R == 0) keeps the old vector
// and gives zero scales.
__global__ void __launch_bounds__(kNormThreads)
svid_normalize_kernel(int N, int K, int path, int last, SvidWs w) {
    __shared__ double red[kNormThreads / 32];
    pdl_enter();
    double sa = 0.0, sb = 0.0;
    for (int n = threadIdx.x; n < N; n += blockDim.x) sa += static_cast<double>(w.grad_a[n]) * w.grad_a[n];
    for (int j = threadIdx.x; j < K; j += blockDim.x) sb += static_cast<double>(w.grad_b[j]) * w.grad_b[j];
    const double na = sqrt(cta_sum(sa, red));
    const double nb = sqrt(cta_sum(sb, red));
    const float ia = na > 0.0 ? static_cast<float>(1.0 / na) : 0.0f;
    const float ib = nb > 0.0 ? static_cast<float>(1.0 / nb) : 0.0f;
    if (!last) {
        if (na > 0.0)
            for (int n = threadIdx.x; n < N; n += blockDim.x) w.avec[n] = w.grad_a[n] * ia;
        if (nb > 0.0)
            for (int j = threadIdx.x; j < K; j += blockDim.x) w.bvec[j] = w.grad_b[j] * ib;
        return;
    }
    const float rs = static_cast<float>(sqrt(na));   // sqrt(sigma)
    float *U = w.U + path * static_cast<int64_t>(N), *gp = w.gp + path * static_cast<int64_t>(N);
    float *V = w.V + path * static_cast<int64_t>(K), *hp = w.hp + path * static_cast<int64_t>(K);
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
        const float u = w.grad_a[n] * ia;
        gp[n] = rs * u;
        if (na > 0.0) U[n] = u;
    }
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
        const float v = w.grad_b[j] * ib;
        hp[j] = nb > 0.0 ? rs * v : 0.0f;
        if (nb > 0.0) V[j] = v;
    }
}

// Scales mapped back to the original domain: a_p = g_p' / s_out^alpha_out, b_p = h_p' / s_in^alpha_in.
__global__ void __launch_bounds__(kThreads)
svid_finish_kernel(int N, int K, int P, float *__restrict__ a, float *__restrict__ b, SvidWs w) {
    pdl_enter();
    const int stride = gridDim.x * blockDim.x;
    for (int p = 0; p < P; ++p) {
        for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < N; n += stride)
            a[p * static_cast<int64_t>(N) + n] = w.gp[p * static_cast<int64_t>(N) + n] / w.so[n];
        for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += stride)
            b[p * static_cast<int64_t>(K) + j] = w.hp[p * static_cast<int64_t>(K) + j] / w.si[j];
    }
}

template <typename... KArgs, typename... Args>
cudaError_t launch(const LaunchCtx &ctx, int grid, int block, void (*kern)(KArgs...), Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(block));
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

size_t svid_workspace_bytes(int N, int K, int P) { return svid_layout(nullptr, N, K, P).total; }

cudaError_t launch_svid_init(const LaunchCtx &ctx, const float *W, int ldw, int N, int K, int P, int T,
                             int power_iters, const float *s_in, const float *s_out, float alpha_in,
                             float alpha_out, float *a, float *b, uint32_t *packed, void *workspace,
                             uint32_t *fault_word, uint64_t timeout_ns) {
    if ((P != 2 && P != 3) || T < 1 || power_iters < 1) return cudaErrorInvalidValue;
    const SvidWs w = svid_layout(workspace, N, K, P);
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    const int64_t vec_len = std::max<int64_t>(N, K);
    const int vec_grid = static_cast<int>(std::min<int64_t>((vec_len + kThreads - 1) / kThreads, ctx.num_sms * 4));
    const int64_t warps = static_cast<int64_t>(N) * Wr;
    const int res_grid = static_cast<int>(std::min<int64_t>((warps * 32 + kThreads - 1) / kThreads,
                                                            static_cast<int64_t>(ctx.num_sms) * 16));
    cudaError_t e = launch(ctx, vec_grid, kThreads, svid_prep_kernel, s_in, s_out, alpha_in, alpha_out, N, K, P, w);
    for (int t = 0; t < T && e == cudaSuccess; ++t) {
        for (int i = 0; i < P && e == cudaSuccess; ++i) {
            e = P == 2 ? launch(ctx, res_grid, kThreads, svid_residual_kernel<2>, W, ldw, N, K, Wr, i, packed, w)
                       : launch(ctx, res_grid, kThreads, svid_residual_kernel<3>, W, ldw, N, K, Wr, i, packed, w);
            for (int s = 0; s < power_iters && e == cudaSuccess; ++s) {
                e = launch_scale_grads(ctx, w.R, static_cast<int>(residual_pitch(K)),
                                       reinterpret_cast<const uint32_t *>(w.ps), w.avec, w.bvec, N, K, 2,
                                       w.grad_a, w.grad_b, w.sg, fault_word, timeout_ns);
                if (e == cudaSuccess)
                    e = launch(ctx, 1, kNormThreads, svid_normalize_kernel, N, K, i, s == power_iters - 1 ? 1 : 0, w);
            }
        }
    }
    if (e == cudaSuccess) e = launch(ctx, vec_grid, kThreads, svid_finish_kernel, N, K, P, a, b, w);
    return e;
}

}  // namespace rabit
