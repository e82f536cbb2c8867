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

// The same pass with G staged by TMA, persistent and balanced to the box: the boxes (32 rows x
// 256 columns of G), in column-tile-major order, are dealt as equal contiguous ranges to one
// CTA per SM ("stream-K"), so no CTA has more than one box above the average.  A range spans
// at most two column tiles (the host checks), so a CTA makes at most two runs.  A producer
// warp keeps kStages stages in flight across run boundaries.  A stage holds one box of G
// (32 KiB of fp32), the sign words of the same rows and columns and the rows' a, all brought
// by TMA, so the consumers read shared memory only.  Eight consumer warps take four rows of
// each box; row sums land in the (column tile, row) slot, which exactly one CTA writes; at a
// run's end the warps add their column sums in shared memory, in a fixed order, into the
// CTA's slot for that run (0 or 1), and pass 2 adds the slots of the CTAs that cover a column
// tile in CTA order.  Every wait is bounded: an expired wait sets a fault bit and a flag in
// shared memory, the consumers stop together at the end of the run, and the producer lets
// its issued copies land before exiting.
constexpr int kBoxRows = 32;
constexpr int kBoxCols = 256;
constexpr int kBoxBytes = kBoxRows * kBoxCols * 4;
constexpr int kStages = 5;
constexpr int kTmaThreads = 288;                 // 8 consumer warps + 1 producer warp
constexpr int kMaxGrid = 160;                                 // CTAs of the stream-K pass, at most
constexpr int kWordsBytesMax = kBoxRows * 32 * 4;             // sign words of a box (P = 3: 32 words a row)
constexpr int kABytes = 1024;                                 // a of a box's rows (P x 32 floats), padded
constexpr int kStageBytes = kBoxBytes + kWordsBytesMax + kABytes;
constexpr int kTmaSmem = kStages * kStageBytes + 128;

// First box of CTA c's range, and the CTA whose range holds box u (U boxes over G CTAs).
__host__ __device__ inline int64_t sk_begin(int c, int64_t U, int G) { return U * c / G; }
__host__ __device__ inline int sk_owner(int64_t u, int64_t U, int G) {
    int c = static_cast<int>(u * G / U);
    while (c + 1 < G && sk_begin(c + 1, U, G) <= u) ++c;
    while (c > 0 && sk_begin(c, U, G) > u) --c;
    return c;
}

template <int kP>
__global__ void __launch_bounds__(kTmaThreads, 1)
scale_grads_tma_kernel(const __grid_constant__ CUtensorMap tmap_g, const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_a,
                       const float *__restrict__ b, int N, int K, int Wr,
                       float *__restrict__ ws_a, float *__restrict__ ws_b, uint32_t *fault,
                       uint64_t timeout_ns, int debug) {
    constexpr int kG = kP == 2 ? 2 : 4;
    constexpr int kSteps = kBoxCols / 128;
    constexpr int kRowsPerWarp = kBoxRows / 8;
    constexpr int kRowWords = (kBoxCols / 32) * kG;                 // sign words of a box row
    constexpr uint32_t kTx = kBoxBytes + kBoxRows * kRowWords * 4 + kP * kBoxRows * 4;
    extern __shared__ __align__(128) uint8_t smem[];
    // stage s: G [32][256] fp32, then the sign words [32][kRowWords], then a [kP][32]
    auto stage_g = [&](int st) { return reinterpret_cast<float *>(smem + st * kStageBytes); };
    auto stage_w = [&](int st) { return reinterpret_cast<const uint32_t *>(smem + st * kStageBytes + kBoxBytes); };
    auto stage_a = [&](int st) {
        return reinterpret_cast<const float *>(smem + st * kStageBytes + kBoxBytes + kWordsBytesMax);
    };
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint64_t *empty = full + kStages;
    __shared__ float colsum[8][kP][kBoxCols];
    __shared__ int s_abort;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nct = (K + kBoxCols - 1) / kBoxCols;
    const int bpc = (N + kBoxRows - 1) / kBoxRows;             // boxes per column tile
    const int64_t U = static_cast<int64_t>(nct) * bpc;
    const int64_t u_begin = sk_begin(blockIdx.x, U, gridDim.x), u_end = sk_begin(blockIdx.x + 1, U, gridDim.x);
    int abort_flag = 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 8);
        }
        s_abort = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_g);
        prefetch_tensormap(&tmap_w);
        prefetch_tensormap(&tmap_a);
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 8) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            bool issued[kStages] = {};
            uint32_t last_parity[kStages] = {};
            bool ok = true;
            int q = 0;                                 // boxes of this CTA so far (ring position)
            for (int64_t u = u_begin; ok && u < u_end; ++u, ++q) {
                const int ct = static_cast<int>(u / bpc), box = static_cast<int>(u % bpc);
                {
                    const int s = q % kStages;
                    const uint32_t par = static_cast<uint32_t>(q / kStages) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&empty[s]), par ^ 1u, &abort_flag, timeout_ns, fault,
                                           FAULT_SCALE_GRADS_WAIT)) {
                        ok = false;
                        break;
                    }
                    if ((debug & 1) && q == 0) continue;   // fault injection: this box never comes
                    const uint32_t bar = smem_u32(&full[s]);
                    mbar_arrive_expect_tx(bar, kTx);
                    tma_load_2d(smem_u32(stage_g(s)), &tmap_g, bar, ct * kBoxCols, box * kBoxRows);
                    tma_load_2d(smem_u32(stage_w(s)), &tmap_w, bar, ct * kRowWords, box * kBoxRows);
                    tma_load_2d(smem_u32(stage_a(s)), &tmap_a, bar, box * kBoxRows, 0);
                    issued[s] = true;
                    last_parity[s] = par;
                }
            }
            // Every issued copy lands before the CTA can exit (the consumers stop early on an
            // expired wait).  These are the latest phases of their stages, already complete in
            // normal operation.
            int drain_abort = 0;
            for (int s = 0; s < kStages; ++s)
                if (issued[s])
                    mbar_wait_bounded(smem_u32(&full[s]), last_parity[s], &drain_abort, timeout_ns, fault,
                                      FAULT_SCALE_GRADS_WAIT);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    // lane's columns: c0 + 128 st + 4 lane + t; group c0/32 + 4 st + lane/8, bits 4(lane%8) + t
    const uint32_t sh = 4 * (lane & 7);
    int q = 0;
    int64_t u = u_begin;
    for (int side = 0; u < u_end; ++side) {       // a run: this CTA's boxes of one column tile
        const int ct = static_cast<int>(u / bpc);
        const int64_t run_end = min(u_end, static_cast<int64_t>(ct + 1) * bpc);
        const int c0 = ct * kBoxCols;
        float bcol[kP][kSteps][4], cacc[kP][kSteps][4];
#pragma unroll
        for (int st = 0; st < kSteps; ++st)
#pragma unroll
            for (int tt = 0; tt < 4; ++tt) {
                const int j = c0 + 128 * st + 4 * lane + tt;
#pragma unroll
                for (int k = 0; k < kP; ++k) {
                    bcol[k][st][tt] = j < K ? __ldg(b + static_cast<int64_t>(k) * K + j) : 0.0f;
                    cacc[k][st][tt] = 0.0f;
                }
            }
        for (; u < run_end; ++u, ++q) {
            const int row0 = static_cast<int>(u % bpc) * kBoxRows;
            const int s = q % kStages;
            const bool ok = mbar_wait_bounded(smem_u32(&full[s]), static_cast<uint32_t>(q / kStages) & 1u,
                                              &abort_flag, timeout_ns, fault, FAULT_SCALE_GRADS_WAIT);
            // An expired wait ends this warp's boxes: it stops releasing stages, so the producer's
            // own bounded wait expires and it drains the copies it issued before the CTA exits;
            // the flag stops every consumer warp at the end of this run.
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) s_abort = 1;
                break;
            }
            const uint32_t *words = stage_w(s);
            const float *arow = stage_a(s);
            const float *box = stage_g(s);
#pragma unroll
            for (int i = 0; i < kRowsPerWarp; ++i) {
                const int r = warp * kRowsPerWarp + i;
                const int n = row0 + r;
                float racc[kP], av[kP];
                uint32_t wv[kSteps][kP];
#pragma unroll
                for (int k = 0; k < kP; ++k) {
                    racc[k] = 0.0f;
                    av[k] = arow[k * kBoxRows + r];
#pragma unroll
                    for (int st = 0; st < kSteps; ++st) wv[st][k] = words[r * kRowWords + (4 * st + (lane >> 3)) * kG + k];
                }
#pragma unroll
                for (int st = 0; st < kSteps; ++st) {
                    const float4 g4 = *reinterpret_cast<const float4 *>(box + r * kBoxCols + 128 * st + 4 * lane);
                    const float gvals[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
                    for (int k = 0; k < kP; ++k) {
#pragma unroll
                        for (int tt = 0; tt < 4; ++tt) {
                            // s = +1 for bit 0, -1 for bit 1: flip the sign bit of G
                            const float gs = __uint_as_float(__float_as_uint(gvals[tt]) ^
                                                             (((wv[st][k] >> (sh + tt)) & 1u) << 31));
                            racc[k] = fmaf(gs, bcol[k][st][tt], racc[k]);
                            cacc[k][st][tt] = fmaf(gs, av[k], cacc[k][st][tt]);
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
                for (int tt = 0; tt < 4; ++tt) colsum[warp][k][128 * st + 4 * lane + tt] = cacc[k][st][tt];
        asm volatile("bar.sync 1, 256;" ::: "memory");   // the 8 consumer warps only
        for (int e = threadIdx.x; e < kP * kBoxCols; e += 256) {
            const int k = e / kBoxCols, cc = e % kBoxCols;
            float v = 0.0f;
            for (int w = 0; w < 8; ++w) v += colsum[w][k][cc];
            ws_b[((static_cast<int64_t>(k) * gridDim.x + blockIdx.x) * 2 + side) * kBoxCols + cc] = v;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");   // colsum is rewritten by the next run
        if (s_abort) break;                              // every consumer warp sees the same flag here
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

// sk_grid > 0: ws_b holds the stream-K pass's run slots [P][sk_grid][2][kBoxCols]; otherwise the
// tile pass's row-block slots [P][nrb][K].
__global__ void __launch_bounds__(256)
scale_grads_sum_kernel(const float *__restrict__ ws_a, const float *__restrict__ ws_b, int N, int K,
                       int P, int nct, int nrb, int sk_grid, float *__restrict__ grad_a,
                       float *__restrict__ grad_b) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int64_t na = static_cast<int64_t>(P) * N, nb = static_cast<int64_t>(P) * K;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < na + nb;
         t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (t < na) {
            const int64_t k = t / N, n = t % N;
            grad_a[t] = strided_sum(ws_a + k * nct * N + n, nct, N);
        } else if (sk_grid > 0) {
            // the CTAs whose ranges cover column tile ct, in CTA order; the first one's slot is
            // 1 when its range began in an earlier tile
            const int64_t u = t - na, k = u / K, j = u % K;
            const int ct = static_cast<int>(j / kBoxCols), cc = static_cast<int>(j % kBoxCols);
            const int bpc = (N + kBoxRows - 1) / kBoxRows;
            const int64_t U = static_cast<int64_t>(nct) * bpc, ub = static_cast<int64_t>(ct) * bpc;
            const int cf = sk_owner(ub, U, sk_grid), cl = sk_owner(ub + bpc - 1, U, sk_grid);
            float v = 0.0f;
            for (int c = cf; c <= cl; ++c) {
                const int side = (c == cf && sk_begin(c, U, sk_grid) < ub) ? 1 : 0;
                v += __ldg(ws_b + ((k * sk_grid + c) * 2 + side) * kBoxCols + cc);
            }
            grad_b[u] = v;
        } else {
            const int64_t u = t - na, k = u / K, j = u % K;
            grad_b[u] = strided_sum(ws_b + k * nrb * K + j, nrb, K);
        }
    }
}

}  // namespace

// [P][nct][N] row-sum slots, then the column-sum slots: the tile pass's [P][nrb][K] or the
// stream-K pass's [P][kMaxGrid][2][kBoxCols], whichever is larger.
size_t scale_grads_workspace_bytes(int N, int K, int P) {
    const size_t nct = (static_cast<size_t>(K) + tile_cols(P) - 1) / tile_cols(P);
    const size_t nrb = (static_cast<size_t>(N) + kTileRows - 1) / kTileRows;
    const size_t colslots = std::max(nrb * K, static_cast<size_t>(kMaxGrid) * 2 * kBoxCols);
    return static_cast<size_t>(P) * (nct * N + colslots) * sizeof(float);
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
    // TMA-staged pass when tensor maps can describe G (16-byte aligned base and pitch) and a.
    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    // (a is staged by TMA as well: 16-byte aligned base and rows of N floats, N a multiple of 4)
    // The stream-K deal: a CTA's range of boxes may touch at most two column tiles.
    const int bpc = (N + kBoxRows - 1) / kBoxRows;
    const int64_t boxes = static_cast<int64_t>(nct) * bpc;
    const int sk_grid = static_cast<int>(std::min<int64_t>({boxes, static_cast<int64_t>(ctx.num_sms), kMaxGrid}));
    const bool two_runs = (boxes + sk_grid - 1) / sk_grid - 1 <= bpc;
    const bool tma = encode && (reinterpret_cast<uintptr_t>(G) % 16 == 0) && ((static_cast<int64_t>(ldg) * 4) % 16 == 0) &&
                     (reinterpret_cast<uintptr_t>(a) % 16 == 0) && (N % 4 == 0) && two_runs;
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
        // the sign words of a box: kRowWords words of each of its rows; a of its rows, per path
        const int G = P == 2 ? 2 : 4;
        CUtensorMap tmap_w, tmap_a;
        cuuint64_t wdims[2] = {static_cast<cuuint64_t>(Wr) * G, static_cast<cuuint64_t>(N)};
        cuuint64_t wstrides[1] = {static_cast<cuuint64_t>(Wr) * G * 4};
        cuuint32_t wbox[2] = {static_cast<cuuint32_t>((kBoxCols / 32) * G), kBoxRows};
        r = encode(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), wdims, wstrides, wbox,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        cuuint64_t adims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(P)};
        cuuint64_t astrides[1] = {static_cast<cuuint64_t>(N) * 4};
        cuuint32_t abox[2] = {kBoxRows, static_cast<cuuint32_t>(P)};
        r = encode(&tmap_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(a), adims, astrides, abox,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        static ContextFlags opted[2];
        void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, const float *, int, int, int, float *, float *,
                     uint32_t *, uint64_t, int) = P == 2 ? scale_grads_tma_kernel<2> : scale_grads_tma_kernel<3>;
        e = ensure_smem_optin(ctx, kern, kTmaSmem, opted[P - 2]);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(static_cast<unsigned>(sk_grid));
        cfg.blockDim = dim3(kTmaThreads);
        cfg.dynamicSmemBytes = kTmaSmem;
        e = cudaLaunchKernelEx(&cfg, kern, tmap, tmap_w, tmap_a, b, N, K, Wr, ws_a, ws_b, fault_word, timeout_ns,
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
    return cudaLaunchKernelEx(&cfg, scale_grads_sum_kernel, ws_a, ws_b, N, K, P, nct, nrb, tma ? sk_grid : 0,
                              grad_a, grad_b);
}

}  // namespace rabit
