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
// Pass 1: a CTA owns a tile of 128 rows x kCols(P) columns; each warp takes 16 rows.  A lane
// reads 4 consecutive columns with one 16-byte load (a warp covers 128 columns per load), and
// the sign words of those columns come straight from the packed row (8 lanes share a word).
// The next two rows' loads (G, sign words, a) are in flight while two rows are summed.  Row sums reduce over
// the lanes and land in a per-column-tile slot; column sums reduce over the warps in shared
// memory and land in a per-row-block slot.  Pass 2 adds the slots in a fixed order, so the
// result does not depend on scheduling.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kTileRows = 128;
constexpr int kThreads = 256;                    // 8 warps x 16 rows
constexpr int kRowsPerWarp = kTileRows / (kThreads / 32);
// Columns per tile (the per-lane b values and column sums take registers).
__host__ __device__ constexpr int tile_cols(int P) { return P == 2 ? 256 : 256; }

template <int kP>
__global__ void __launch_bounds__(kThreads)
scale_grads_tile_kernel(const float *__restrict__ G, int ldg, const uint32_t *__restrict__ packed,
                        const float *__restrict__ a, const float *__restrict__ b, int N, int K, int Wr,
                        float *__restrict__ ws_a, float *__restrict__ ws_b) {
    constexpr int kG = kP == 2 ? 2 : 4;          // words per 32-column group
    constexpr int kCols = tile_cols(kP);
    constexpr int kSteps = kCols / 128;          // 16-byte loads per lane per row
    __shared__ float colsum[kThreads / 32][kP][kCols];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nct = (K + kCols - 1) / kCols;
    const int ct = blockIdx.x % nct, rb = blockIdx.x / nct;
    const int c0 = ct * kCols;                     // first column of the tile
    const int n_begin = rb * kTileRows + warp * kRowsPerWarp;
    // lane's columns: c0 + 128 s + 4 lane + t (t < 4); group (c0/32 + 4 s + lane/8), bits 4(lane%8)+t
    const bool vec = (ldg % 4 == 0) && (reinterpret_cast<uintptr_t>(G) % 16 == 0);

    float bcol[kP][kSteps][4], cacc[kP][kSteps][4];
#pragma unroll
    for (int st = 0; st < kSteps; ++st)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int j = c0 + 128 * st + 4 * lane + t;
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                bcol[k][st][t] = j < K ? __ldg(b + static_cast<int64_t>(k) * K + j) : 0.0f;
                cacc[k][st][t] = 0.0f;
            }
        }
    // Everything one row needs, loaded ahead: G (16 bytes per step), its sign words and a.
    struct Row { float4 g[kSteps]; uint32_t w[kSteps][kP]; float a[kP]; };
    auto load_row = [&](int r, Row &row) {
        const int n = n_begin + r;
        const bool nok = n < N;
        const float *grow = G + static_cast<int64_t>(nok ? n : 0) * ldg;
#pragma unroll
        for (int st = 0; st < kSteps; ++st) {
            const int j = c0 + 128 * st + 4 * lane;
            if (nok && vec && j + 4 <= K) {
                row.g[st] = __ldg(reinterpret_cast<const float4 *>(grow + j));
            } else {
                float v[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) v[t] = nok && j + t < K ? __ldg(grow + j + t) : 0.0f;
                row.g[st] = make_float4(v[0], v[1], v[2], v[3]);
            }
            const int grp = c0 / 32 + 4 * st + (lane >> 3);
#pragma unroll
            for (int k = 0; k < kP; ++k)
                row.w[st][k] = nok && grp < Wr ? __ldg(packed + (static_cast<int64_t>(n) * Wr + grp) * kG + k) : 0u;
        }
#pragma unroll
        for (int k = 0; k < kP; ++k) row.a[k] = nok ? __ldg(a + static_cast<int64_t>(k) * N + n) : 0.0f;
    };
    auto sum_row = [&](int r, const Row &row) {
        const int n = n_begin + r;
        float racc[kP];
#pragma unroll
        for (int k = 0; k < kP; ++k) racc[k] = 0.0f;
        const uint32_t sh = 4 * (lane & 7);
#pragma unroll
        for (int st = 0; st < kSteps; ++st) {
            const float gvals[4] = {row.g[st].x, row.g[st].y, row.g[st].z, row.g[st].w};
#pragma unroll
            for (int k = 0; k < kP; ++k) {
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    // s = +1 for bit 0, -1 for bit 1: flip the sign bit of G
                    const float gs = __uint_as_float(__float_as_uint(gvals[t]) ^ (((row.w[st][k] >> (sh + t)) & 1u) << 31));
                    racc[k] = fmaf(gs, bcol[k][st][t], racc[k]);
                    cacc[k][st][t] = fmaf(gs, row.a[k], cacc[k][st][t]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            float v = racc[k];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0 && n < N) ws_a[(static_cast<int64_t>(k) * nct + ct) * N + n] = v;
        }
    };
    // two rows at a time, the next two rows' loads in flight meanwhile
    Row c0r, c1r, n0r, n1r;
    load_row(0, c0r);
    load_row(1, c1r);
#pragma unroll 1
    for (int r = 0; r < kRowsPerWarp; r += 2) {
        if (n_begin + r >= N) break;               // warp-uniform
        if (r + 2 < kRowsPerWarp) {
            load_row(r + 2, n0r);
            load_row(r + 3, n1r);
        }
        sum_row(r, c0r);
        sum_row(r + 1, c1r);                       // rows past N carry zeros and store nothing
        c0r = n0r;
        c1r = n1r;
    }
    // column sums of the tile: over the 8 warps, in a fixed order
#pragma unroll
    for (int k = 0; k < kP; ++k)
#pragma unroll
        for (int st = 0; st < kSteps; ++st)
#pragma unroll
            for (int t = 0; t < 4; ++t) colsum[warp][k][128 * st + 4 * lane + t] = cacc[k][st][t];
    __syncthreads();
    const int nrb = (N + kTileRows - 1) / kTileRows;
    for (int u = threadIdx.x; u < kP * kCols; u += kThreads) {
        const int k = u / kCols, c = u % kCols;
        const int j = c0 + c;
        if (j >= K) continue;
        float v = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) v += colsum[w][k][c];
        ws_b[(static_cast<int64_t>(k) * nrb + rb) * K + j] = v;
    }
}

// The same pass with G staged by TMA: a producer warp keeps kStages boxes of 32 rows x 256
// columns (32 KiB of fp32) in flight, so the memory parallelism does not depend on registers;
// eight consumer warps take four rows of each box, reading G from shared memory, and load the
// next box's sign words and a while the current box is summed.  CTA = one 256-column tile x
// kBoxesPerCta boxes of rows.  Every wait is bounded: an expired wait sets a fault bit, the
// consumers contribute zeros, and the producer lets its issued copies land before exiting.
constexpr int kBoxRows = 32;
constexpr int kBoxCols = 256;
constexpr int kBoxBytes = kBoxRows * kBoxCols * 4;
constexpr int kStages = 3;
constexpr int kBoxesPerCta = 8;                  // 256 rows
constexpr int kTmaThreads = 288;                 // 8 consumer warps + 1 producer warp
constexpr int kTmaSmem = kStages * kBoxBytes + 128;

template <int kP>
__global__ void __launch_bounds__(kTmaThreads)
scale_grads_tma_kernel(const __grid_constant__ CUtensorMap tmap_g, const uint32_t *__restrict__ packed,
                       const float *__restrict__ a, const float *__restrict__ b, int N, int K, int Wr,
                       float *__restrict__ ws_a, float *__restrict__ ws_b, uint32_t *fault,
                       uint64_t timeout_ns, int debug) {
    constexpr int kG = kP == 2 ? 2 : 4;
    constexpr int kSteps = kBoxCols / 128;
    constexpr int kRowsPerWarp = kBoxRows / 8;
    extern __shared__ __align__(128) uint8_t smem[];
    float *stage = reinterpret_cast<float *>(smem);                       // [kStages][32][256]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kBoxBytes);
    uint64_t *empty = full + kStages;
    __shared__ float colsum[8][kP][kBoxCols];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nct = (K + kBoxCols - 1) / kBoxCols;
    const int ct = blockIdx.x % nct, rb = blockIdx.x / nct;
    const int c0 = ct * kBoxCols;
    const int row0 = rb * kBoxRows * kBoxesPerCta;
    const int boxes = min(kBoxesPerCta, (N - row0 + kBoxRows - 1) / kBoxRows);
    int abort_flag = 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 8);
        }
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_g);
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 8) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < boxes; ++c) {
                const int s = c % kStages;
                if (!mbar_wait_bounded(smem_u32(&empty[s]), ((c / kStages) & 1) ^ 1, &abort_flag, timeout_ns,
                                       fault, FAULT_SCALE_GRADS_WAIT))
                    break;
                if ((debug & 1) && c == 0) continue;   // fault injection: this box never comes
                mbar_arrive_expect_tx(smem_u32(&full[s]), kBoxBytes);
                tma_load_2d(smem_u32(stage + s * kBoxRows * kBoxCols), &tmap_g, smem_u32(&full[s]), c0,
                            row0 + c * kBoxRows);
                issued = c + 1;
            }
            // Let every issued copy land before the CTA can exit (the consumers stop early on an
            // expired wait).  These are the latest phases of their stages, already complete in
            // normal operation.
            int drain_abort = 0;
            for (int c = max(0, issued - kStages); c < issued; ++c)
                if (!((debug & 1) && c == 0))
                    mbar_wait_bounded(smem_u32(&full[c % kStages]), (c / kStages) & 1, &drain_abort, timeout_ns,
                                      fault, FAULT_SCALE_GRADS_WAIT);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // lane's columns: c0 + 128 st + 4 lane + t; group c0/32 + 4 st + lane/8, bits 4(lane%8) + t
    float bcol[kP][kSteps][4], cacc[kP][kSteps][4];
#pragma unroll
    for (int st = 0; st < kSteps; ++st)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int j = c0 + 128 * st + 4 * lane + t;
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                bcol[k][st][t] = j < K ? __ldg(b + static_cast<int64_t>(k) * K + j) : 0.0f;
                cacc[k][st][t] = 0.0f;
            }
        }
    struct Side { uint32_t w[kRowsPerWarp][kSteps][kP]; float a[kRowsPerWarp][kP]; };
    auto load_side = [&](int c, Side &sd) {
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int n = row0 + c * kBoxRows + warp * kRowsPerWarp + i;
            const bool nok = n < N;
#pragma unroll
            for (int st = 0; st < kSteps; ++st) {
                const int grp = c0 / 32 + 4 * st + (lane >> 3);
#pragma unroll
                for (int k = 0; k < kP; ++k)
                    sd.w[i][st][k] = nok && grp < Wr ? __ldg(packed + (static_cast<int64_t>(n) * Wr + grp) * kG + k) : 0u;
            }
#pragma unroll
            for (int k = 0; k < kP; ++k) sd.a[i][k] = nok ? __ldg(a + static_cast<int64_t>(k) * N + n) : 0.0f;
        }
    };
    Side cur, nxt;
    load_side(0, nxt);
    const uint32_t sh = 4 * (lane & 7);
    for (int c = 0; c < boxes; ++c) {
        cur = nxt;
        if (c + 1 < boxes) load_side(c + 1, nxt);
        const int s = c % kStages;
        const bool ok = mbar_wait_bounded(smem_u32(&full[s]), (c / kStages) & 1, &abort_flag, timeout_ns, fault,
                                          FAULT_SCALE_GRADS_WAIT);
        // An expired wait ends this warp's boxes: it stops releasing stages, so the producer's
        // own bounded wait expires and it drains the copies it issued before the CTA exits.
        if (!__all_sync(0xffffffffu, ok)) break;
        const float *box = stage + s * kBoxRows * kBoxCols;
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int r = warp * kRowsPerWarp + i;
            const int n = row0 + c * kBoxRows + r;
            float racc[kP];
#pragma unroll
            for (int k = 0; k < kP; ++k) racc[k] = 0.0f;
#pragma unroll
            for (int st = 0; st < kSteps; ++st) {
                const float4 g4 = *reinterpret_cast<const float4 *>(box + r * kBoxCols + 128 * st + 4 * lane);
                const float gvals[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                for (int k = 0; k < kP; ++k) {
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        // s = +1 for bit 0, -1 for bit 1: flip the sign bit of G
                        const float gs = __uint_as_float(__float_as_uint(gvals[t]) ^
                                                         (((cur.w[i][st][k] >> (sh + t)) & 1u) << 31));
                        racc[k] = fmaf(gs, bcol[k][st][t], racc[k]);
                        cacc[k][st][t] = fmaf(gs, cur.a[i][k], cacc[k][st][t]);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                float v = racc[k];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0 && n < N) ws_a[(static_cast<int64_t>(k) * nct + ct) * N + n] = v;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
    }
    // column sums of the tile: over the 8 consumer warps, in a fixed order
#pragma unroll
    for (int k = 0; k < kP; ++k)
#pragma unroll
        for (int st = 0; st < kSteps; ++st)
#pragma unroll
            for (int t = 0; t < 4; ++t) colsum[warp][k][128 * st + 4 * lane + t] = cacc[k][st][t];
    asm volatile("bar.sync 1, 256;" ::: "memory");   // the 8 consumer warps only
    const int nrb = (N + kBoxRows * kBoxesPerCta - 1) / (kBoxRows * kBoxesPerCta);
    for (int u = threadIdx.x; u < kP * kBoxCols; u += 256) {
        const int k = u / kBoxCols, cc = u % kBoxCols;
        const int j = c0 + cc;
        if (j >= K) continue;
        float v = 0.0f;
        for (int w = 0; w < 8; ++w) v += colsum[w][k][cc];
        ws_b[(static_cast<int64_t>(k) * nrb + rb) * K + j] = v;
    }
}

// Pass 2: grad_a[k][n] = sum over column tiles, grad_b[k][j] = sum over row blocks.  Eight
// partial sums per output keep eight loads in flight per thread; they combine in a fixed
// order, so the result is the same on every run.
__device__ __forceinline__ float strided_sum(const float *__restrict__ p, int count, int64_t stride) {
    float s[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    int i = 0;
    for (; i + 8 <= count; i += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) s[u] += __ldg(p + static_cast<int64_t>(i + u) * stride);
    }
    for (int u = 0; i < count; ++i, ++u) s[u] += __ldg(p + static_cast<int64_t>(i) * stride);
    return ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

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
            grad_a[t] = strided_sum(ws_a + k * nct * N + n, nct, N);
        } else {
            const int64_t u = t - na, k = u / K, j = u % K;
            grad_b[u] = strided_sum(ws_b + k * nrb * K + j, nrb, K);
        }
    }
}

}  // namespace

size_t scale_grads_workspace_bytes(int N, int K, int P) {
    const size_t nct = (static_cast<size_t>(K) + tile_cols(P) - 1) / tile_cols(P);
    const size_t nrb = (static_cast<size_t>(N) + kTileRows - 1) / kTileRows;
    return static_cast<size_t>(P) * (nct * N + nrb * K) * sizeof(float);
}

cudaError_t launch_scale_grads(const LaunchCtx &ctx, const float *G, int ldg, const uint32_t *packed,
                               const float *a, const float *b, int N, int K, int P, float *grad_a,
                               float *grad_b, void *workspace, uint32_t *fault_word, uint64_t timeout_ns,
                               int debug) {
    if (P != 2 && P != 3) return cudaErrorInvalidValue;
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    const int nct = (K + tile_cols(P) - 1) / tile_cols(P);
    float *ws_a = static_cast<float *>(workspace);
    float *ws_b = ws_a + static_cast<size_t>(P) * nct * N;

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nrb = 0;
    cudaError_t e = cudaSuccess;
    // TMA-staged pass when the tensor map can describe G (16-byte aligned base and pitch).
    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    const bool tma = encode && (reinterpret_cast<uintptr_t>(G) % 16 == 0) && ((static_cast<int64_t>(ldg) * 4) % 16 == 0);
    if (tma) {
        CUtensorMap tmap;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldg) * 4};
        cuuint32_t box[2] = {kBoxCols, kBoxRows};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(G), dims, strides,
                            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        static ContextFlags opted[2];
        void (*kern)(CUtensorMap, const uint32_t *, const float *, const float *, int, int, int, float *, float *,
                     uint32_t *, uint64_t, int) = P == 2 ? scale_grads_tma_kernel<2> : scale_grads_tma_kernel<3>;
        e = ensure_smem_optin(ctx, kern, kTmaSmem, opted[P - 2]);
        if (e != cudaSuccess) return e;
        nrb = (N + kBoxRows * kBoxesPerCta - 1) / (kBoxRows * kBoxesPerCta);
        cfg.gridDim = dim3(static_cast<unsigned>(nct) * static_cast<unsigned>(nrb));
        cfg.blockDim = dim3(kTmaThreads);
        cfg.dynamicSmemBytes = kTmaSmem;
        e = cudaLaunchKernelEx(&cfg, kern, tmap, packed, a, b, N, K, Wr, ws_a, ws_b, fault_word, timeout_ns,
                               debug);
    } else {
        nrb = (N + kTileRows - 1) / kTileRows;
        cfg.gridDim = dim3(static_cast<unsigned>(nct) * static_cast<unsigned>(nrb));
        cfg.blockDim = dim3(kThreads);
        e = P == 2 ? cudaLaunchKernelEx(&cfg, scale_grads_tile_kernel<2>, G, ldg, packed, a, b, N, K, Wr, ws_a, ws_b)
                   : cudaLaunchKernelEx(&cfg, scale_grads_tile_kernel<3>, G, ldg, packed, a, b, N, K, Wr, ws_a, ws_b);
    }
    if (e != cudaSuccess) return e;
    const int64_t total = static_cast<int64_t>(P) * (N + K);
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>((total + 255) / 256, static_cast<int64_t>(ctx.num_sms) * 8)));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, scale_grads_sum_kernel, ws_a, ws_b, N, K, P, nct, nrb, grad_a, grad_b);
}

}  // namespace rabit
