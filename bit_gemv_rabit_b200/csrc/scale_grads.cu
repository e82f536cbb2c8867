// scale_grads.cu -- gradients of the layer's scales for a given G = dL/dW_hat.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs": the shared
// weight takes G unchanged (straight-through) and the scales are learnable (sec. 4.2); the
// page text loses the update formula, so this is the plain chain rule on sec. 4.1's
// W_hat = sum_k a_k (.) S_k (.) b_k with the signs held fixed:
//     grad_a[k][n] = sum_j G[n][j] * S_k[n][j] * b_k[j]
//     grad_b[k][j] = sum_n G[n][j] * a_k[n] * S_k[n][j]
//
// HBM-bound: G (4 bytes per weight) is read once, the packed signs (P bits per weight) once.
// Pass 1: a CTA owns a tile of 128 rows x 512 columns (16 groups); each warp takes 16 rows,
// each lane 16 columns (j = 32 i + lane), so every G load is one coalesced 128-byte line.
// Lanes 0..15 load the row's 16 group words and a shuffle hands word i to all lanes at step i.
// Row sums reduce over the lanes and land in a per-column-tile slot; column sums reduce over
// the warps in shared memory and land in a per-row-block slot.  Pass 2 adds the slots in a
// fixed order, so the result does not depend on scheduling.
#include <algorithm>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kTileRows = 128;
constexpr int kTileGroups = 16;                  // 512 columns
constexpr int kTileCols = kTileGroups * 32;
constexpr int kThreads = 256;                    // 8 warps x 16 rows
constexpr int kRowsPerWarp = kTileRows / (kThreads / 32);

template <int kP>
__global__ void __launch_bounds__(kThreads)
scale_grads_tile_kernel(const float *__restrict__ G, int ldg, const uint32_t *__restrict__ packed,
                        const float *__restrict__ a, const float *__restrict__ b, int N, int K, int Wr,
                        float *__restrict__ ws_a, float *__restrict__ ws_b) {
    constexpr int kG = kP == 2 ? 2 : 4;          // words per 32-column group
    __shared__ float colsum[kThreads / 32][kP][kTileCols];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nct = (K + kTileCols - 1) / kTileCols;
    const int ct = blockIdx.x % nct, rb = blockIdx.x / nct;
    const int g0 = ct * kTileGroups;               // first group of the tile
    const int n_begin = rb * kTileRows + warp * kRowsPerWarp;

    float bcol[kP][kTileGroups], cacc[kP][kTileGroups];
#pragma unroll
    for (int i = 0; i < kTileGroups; ++i) {
        const int j = (g0 + i) * 32 + lane;
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            bcol[k][i] = j < K ? __ldg(b + static_cast<int64_t>(k) * K + j) : 0.0f;
            cacc[k][i] = 0.0f;
        }
    }
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const int n = n_begin + r;
        if (n >= N) break;                         // warp-uniform
        float ak[kP];
#pragma unroll
        for (int k = 0; k < kP; ++k) ak[k] = __ldg(a + static_cast<int64_t>(k) * N + n);
        uint32_t word[kP];
        const bool wl = lane < kTileGroups && g0 + lane < Wr;
#pragma unroll
        for (int k = 0; k < kP; ++k)
            word[k] = wl ? __ldg(packed + (static_cast<int64_t>(n) * Wr + g0 + lane) * kG + k) : 0u;
        const float *grow = G + static_cast<int64_t>(n) * ldg;
        float gv[kTileGroups];
#pragma unroll
        for (int i = 0; i < kTileGroups; ++i) {
            const int j = (g0 + i) * 32 + lane;
            gv[i] = j < K ? __ldg(grow + j) : 0.0f;
        }
        float racc[kP];
#pragma unroll
        for (int k = 0; k < kP; ++k) racc[k] = 0.0f;
#pragma unroll
        for (int i = 0; i < kTileGroups; ++i) {
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                const uint32_t wi = __shfl_sync(0xffffffffu, word[k], i);
                // s = +1 for bit 0, -1 for bit 1: flip the sign bit of G
                const float gs = __uint_as_float(__float_as_uint(gv[i]) ^ (((wi >> lane) & 1u) << 31));
                racc[k] = fmaf(gs, bcol[k][i], racc[k]);
                cacc[k][i] = fmaf(gs, ak[k], cacc[k][i]);
            }
        }
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            float v = racc[k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) ws_a[(static_cast<int64_t>(k) * nct + ct) * N + n] = v;
        }
    }
    // column sums of the tile: over the 8 warps, in a fixed order
#pragma unroll
    for (int k = 0; k < kP; ++k)
#pragma unroll
        for (int i = 0; i < kTileGroups; ++i) colsum[warp][k][i * 32 + lane] = cacc[k][i];
    __syncthreads();
    const int nrb = (N + kTileRows - 1) / kTileRows;
    for (int t = threadIdx.x; t < kP * kTileCols; t += kThreads) {
        const int k = t / kTileCols, c = t % kTileCols;
        const int j = g0 * 32 + c;
        if (j >= K) continue;
        float v = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) v += colsum[w][k][c];
        ws_b[(static_cast<int64_t>(k) * nrb + rb) * K + j] = v;
    }
}

// Pass 2: grad_a[k][n] = sum over column tiles, grad_b[k][j] = sum over row blocks.
__global__ void __launch_bounds__(256)
scale_grads_sum_kernel(const float *__restrict__ ws_a, const float *__restrict__ ws_b, int N, int K,
                       int P, int nct, int nrb, float *__restrict__ grad_a, float *__restrict__ grad_b) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int64_t na = static_cast<int64_t>(P) * N, nb = static_cast<int64_t>(P) * K;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < na + nb;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (t < na) {
            const int64_t k = t / N, n = t % N;
            float v = 0.0f;
            for (int c = 0; c < nct; ++c) v += ws_a[(k * nct + c) * N + n];
            grad_a[t] = v;
        } else {
            const int64_t u = t - na, k = u / K, j = u % K;
            float v = 0.0f;
            for (int r = 0; r < nrb; ++r) v += ws_b[(k * nrb + r) * K + j];
            grad_b[u] = v;
        }
    }
}

}  // namespace

size_t scale_grads_workspace_bytes(int N, int K, int P) {
    const size_t nct = (static_cast<size_t>(K) + kTileCols - 1) / kTileCols;
    const size_t nrb = (static_cast<size_t>(N) + kTileRows - 1) / kTileRows;
    return static_cast<size_t>(P) * (nct * N + nrb * K) * sizeof(float);
}

cudaError_t launch_scale_grads(const LaunchCtx &ctx, const float *G, int ldg, const uint32_t *packed,
                               const float *a, const float *b, int N, int K, int P, float *grad_a,
                               float *grad_b, void *workspace) {
    if (P != 2 && P != 3) return cudaErrorInvalidValue;
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    const int nct = (K + kTileCols - 1) / kTileCols;
    const int nrb = (N + kTileRows - 1) / kTileRows;
    float *ws_a = static_cast<float *>(workspace);
    float *ws_b = ws_a + static_cast<size_t>(P) * nct * N;

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nct) * static_cast<unsigned>(nrb));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = P == 2 ? cudaLaunchKernelEx(&cfg, scale_grads_tile_kernel<2>, G, ldg, packed, a, b, N, K, Wr, ws_a, ws_b)
                           : cudaLaunchKernelEx(&cfg, scale_grads_tile_kernel<3>, G, ldg, packed, a, b, N, K, Wr, ws_a, ws_b);
    if (e != cudaSuccess) return e;
    const int64_t total = static_cast<int64_t>(P) * (N + K);
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(ctx.num_sms) * 8)));
    cfg.blockDim = dim3(256);
    return cudaLaunchKernelEx(&cfg, scale_grads_sum_kernel, ws_a, ws_b, N, K, P, nct, nrb, grad_a, grad_b);
}

}  // namespace rabit
