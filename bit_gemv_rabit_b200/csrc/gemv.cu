// gemv.cu -- decode path of the residual-binary linear layer, batch 1..16.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.1 "Multi-bit Approximation via Stacking" executed per path as described in
// Appendix E.1 "Compute Pipeline" (paths in parallel, signs applied without multiplies,
// warp-shuffle reduction, output scale applied last):
//     y[beta][n] = sum_k a_k[n] * t_k[beta][n],   t_k[beta][n] = sum_j S_k[n][j] z_k[beta][j],
//     z_k[beta][j] = b_k[j] * x[beta][j].
//
// Design for sm_100a (CUDA cores; the integer dot-product pipe is the limit):
//
//  * Signs as masked sums.  t = Z - 2*sum_{bit=1} z with Z = sum_j z.  For each 32-column
//    group z is quantised to 15-bit integers with a power-of-two scale of its own (the group
//    max fixes it, so the error is relative to the local maximum).  One 3-input logic op
//    isolates four sign bits of a word at one position in each byte (values 0 or 2^q), and a
//    dp2a multiplies two of those bytes with two pre-shifted 16-bit z values and accumulates
//    in 32-bit: the integer sum is exact.  Two bit positions per byte (q in {0,1}) with z
//    pre-shifted by 2^(1-q) give every product the same weight 2*z, so each path needs one
//    accumulator, seeded with -Z.  Per 32 weight bits: 16 dp2a, 8 logic ops, 3 shifts.
//  * Lane = 32-column group.  Each lane keeps its group's z pairs in registers (16 per
//    path) and streams rows; a row's contribution is finished in fp32 and the lanes'
//    partial sums of 8 rows are reduced with a butterfly that leaves one row per 4 lanes.
//  * Clusters split K.  The CTAs of a thread-block cluster share a block of rows and each
//    takes a contiguous slice of the 32-column groups, so an SM quantises only its own slice
//    of z; the per-CTA row partials are summed across the cluster through distributed
//    shared memory and each CTA stores a share of y.
//  * Weights stream straight into registers: a warp loads the word pairs of its next 8 rows
//    while it works on the current 8 (one 8-byte load per lane and row, 256 contiguous bytes
//    per warp).  Before the programmatic-launch wait each CTA asks L2 to prefetch its share
//    of the cluster's row block (contiguous in the row-major layout; the previous kernel on
//    the stream may still be running, and an L2 prefetch returns no data to the SM, so it
//    cannot observe a stale value).  Batch rows after the first re-read the words from L1.
//  * RABIT_F32 activations use two 15-bit slices of a 29-bit z (twice the dp2a work).
#include <algorithm>
#include <cstdlib>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kMaxThreads = 512;
constexpr int kGroupRows = 8;            // rows per butterfly reduction and per copy barrier
constexpr int kSmemBudget = 200 * 1024;  // dynamic shared memory a CTA may use

struct GemvArgs {
    const uint2 *packed;   // [N][Wr] groups {path-1 word, path-2 word}
    const float *a;        // [2][N]
    const float *b;        // [2][K]
    const void *x;         // [batch][ldx]
    float *y;              // [batch][ldy]
    int N, K, Wr, batch, ldx, ldy;
    int cluster;           // CTAs per cluster (they split the 32-column groups)
    int rows_per_cluster;  // contiguous rows owned by one cluster
    int block_rows;        // rows a cluster finishes per block (shared memory holds one block)
    int range_max;         // most 32-column groups any CTA owns (<= 32 * nchunks)
    int nchunks;           // warps across a CTA's groups (32 groups each)
    int streams;           // warps along rows
};

struct SmemLayout {
    uint32_t zp, zinit, zscale, arow, red, cred, total;
};

template <int kSlices>
__host__ __device__ inline SmemLayout smem_layout(int rpc, int range_max, int nchunks, int batch) {
    SmemLayout L;
    uint32_t off = 0;
    auto take = [&](uint32_t bytes) { uint32_t o = off; off = (off + bytes + 127u) & ~127u; return o; };
    L.zp = take(static_cast<uint32_t>(kSlices) * 2u * 16u * range_max * 4u);
    L.zinit = take(static_cast<uint32_t>(kSlices) * 2u * range_max * 4u);
    L.zscale = take(2u * range_max * 4u);
    L.arow = take(static_cast<uint32_t>(rpc) * 8u);
    L.red = take(nchunks > 1 ? static_cast<uint32_t>(nchunks) * rpc * 4u : 0u);
    L.cred = take(static_cast<uint32_t>(batch) * rpc * 4u);
    L.total = off;
    return L;
}

__device__ __forceinline__ uint32_t dp2a_lo(uint32_t zpair, uint32_t bytes, uint32_t acc) {
    uint32_t d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(zpair), "r"(bytes), "r"(acc));
    return d;
}
__device__ __forceinline__ uint32_t dp2a_hi(uint32_t zpair, uint32_t bytes, uint32_t acc) {
    uint32_t d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(zpair), "r"(bytes), "r"(acc));
    return d;
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t local_addr, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                 ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes) : "memory");
}

template <bool kF32X>
__device__ __forceinline__ float load_x(const void *x, int64_t idx) {
    if constexpr (kF32X) {
        return __ldg(reinterpret_cast<const float *>(x) + idx);
    } else {
        const unsigned short bits = __ldg(reinterpret_cast<const unsigned short *>(x) + idx);
        return __uint_as_float(static_cast<uint32_t>(bits) << 16);
    }
}

// Sum of v[0..7] over the 32 lanes; afterwards lane l holds the total of v[(l >> 2) & 7].
__device__ __forceinline__ float butterfly8(const float (&v)[8], int lane) {
    const bool b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1, b2 = (lane >> 2) & 1;
    float u[4], t[2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float send = b4 ? v[k] : v[k + 4];
        const float keep = b4 ? v[k + 4] : v[k];
        u[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float send = b3 ? u[k] : u[k + 2];
        const float keep = b3 ? u[k + 2] : u[k];
        t[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const float send = b2 ? t[0] : t[1];
    float s = (b2 ? t[1] : t[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    return s;
}

template <bool kF32X>
__global__ void __launch_bounds__(kMaxThreads, 1)
gemv_kernel(const GemvArgs p) {
    constexpr int kSlices = kF32X ? 2 : 1;
    extern __shared__ __align__(128) uint8_t smem[];
    const SmemLayout L = smem_layout<kSlices>(p.block_rows, p.range_max, p.nchunks, p.batch);
    uint32_t *zp = reinterpret_cast<uint32_t *>(smem + L.zp);        // [slice][path][16][range_max]
    int32_t *zinit = reinterpret_cast<int32_t *>(smem + L.zinit);    // [slice][path][range_max]
    float *zscale = reinterpret_cast<float *>(smem + L.zscale);      // [path][range_max]
    float2 *arow = reinterpret_cast<float2 *>(smem + L.arow);        // [block_rows]
    float *red = reinterpret_cast<float *>(smem + L.red);            // [nchunks][block_rows]
    float *cred = reinterpret_cast<float *>(smem + L.cred);          // [batch][block_rows]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x;
    const int chunk = warp % p.nchunks, stream = warp / p.nchunks;
    const uint32_t rank = cluster_ctarank();
    const int cluster_id = blockIdx.x / p.cluster;
    const int row_begin = cluster_id * p.rows_per_cluster;
    const int row_end = min(p.N, row_begin + p.rows_per_cluster);
    const int cl_rows = max(row_end - row_begin, 0);
    const int RB = p.block_rows;
    // This CTA's slice of 32-column groups, in units of 4 groups (128 columns).
    const int units = p.Wr / 4;
    const int g0 = (static_cast<int>(rank) * units / p.cluster) * 4;
    const int g1 = ((static_cast<int>(rank) + 1) * units / p.cluster) * 4;
    const int range = g1 - g0;

    // Warm L2 with this CTA's share of the cluster's (contiguous) row block while the
    // previous kernel may still be running.
    if (tid == 0 && cl_rows > 0) {
        const uint64_t block_bytes = static_cast<uint64_t>(cl_rows) * p.Wr * 8u;
        const uint64_t lo = (block_bytes * rank / p.cluster) & ~static_cast<uint64_t>(15);
        const uint64_t hi = (block_bytes * (rank + 1) / p.cluster) & ~static_cast<uint64_t>(15);
        const uint8_t *base = reinterpret_cast<const uint8_t *>(p.packed + static_cast<int64_t>(row_begin) * p.Wr);
        for (uint64_t o = lo; o < hi; o += (1u << 20))
            bulk_prefetch_l2(base + o, static_cast<uint32_t>(min(hi - o, static_cast<uint64_t>(1u << 20))));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    const int gl = chunk * 32 + lane;          // this lane's group within the CTA's slice
    const bool lane_on = gl < range;
    const uint2 *wcol = p.packed + g0 + gl;    // this lane's column of word pairs (row 0)

  for (int row0 = row_begin; row0 < row_end; row0 += RB) {
    const int nrows = min(RB, row_end - row0);
    const int ngroups = (nrows + kGroupRows - 1) / kGroupRows;
    for (int r = tid; r < nrows; r += nthreads)
        arow[r] = make_float2(__ldg(p.a + row0 + r), __ldg(p.a + p.N + row0 + r));

    for (int beta = 0; beta < p.batch; ++beta) {
        // ---- z_k = x (.) b_k for this CTA's groups, quantised per 32-column group.
        // 8 consecutive threads per (path, group), 4 columns each.
        const int ztasks = 2 * range * 8;
        for (int t = tid; t < ((ztasks + 31) & ~31); t += nthreads) {
            const bool on = t < ztasks;
            const int q = t & 7;
            const int gloc = (t >> 3) % max(range, 1);
            const int k = ((t >> 3) / max(range, 1)) & 1;
            float z[4];
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = (g0 + gloc) * 32 + 4 * q + i;
                z[i] = 0.0f;
                if (on && j < p.K)
                    z[i] = load_x<kF32X>(p.x, static_cast<int64_t>(beta) * p.ldx + j) * __ldg(p.b + k * p.K + j);
                m = fmaxf(m, fabsf(z[i]));
            }
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            // power-of-two scale 2^e with m * 2^e <= kMaxQ (15-bit, or 29-bit for fp32 x)
            constexpr int kTop = kF32X ? 27 : 13;
            const float kMaxQ = kF32X ? 268435455.0f : 16383.0f;
            int E = static_cast<int>((__float_as_uint(m) >> 23) & 0xFFu) - 127;
            int e = kTop - E;
            if (e > 127) e = 127;
            if (e < -126) e = -126;
            float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
            if (m * sc > kMaxQ) { --e; sc *= 0.5f; }
            int zsum[kSlices];
#pragma unroll
            for (int s = 0; s < kSlices; ++s) zsum[s] = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = 4 * q + i;                 // column within the group
                const int h = col >> 4, u = col & 15, half = u >> 3, pos = u & 7;
                const int sh = pos >> 1, jj = pos & 1;
                const int pair = sh * 4 + jj * 2 + h;
                const int zq = __float2int_rn(z[i] * sc);
                int part[kSlices];
                if constexpr (kF32X) {
                    part[0] = (zq + (1 << 13)) >> 14;       // high 15-bit slice
                    part[1] = zq - (part[0] << 14);         // low slice, in [-2^13, 2^13)
                } else {
                    part[0] = zq;
                }
#pragma unroll
                for (int s = 0; s < kSlices; ++s) {
                    zsum[s] += part[s];
                    if (on) {
                        const int zpre = part[s] * (jj ? 1 : 2);   // weight 2^(1-jj)
                        uint16_t *slot = reinterpret_cast<uint16_t *>(
                            zp + ((s * 2 + k) * 16 + pair) * p.range_max + gloc) + half;
                        *slot = static_cast<uint16_t>(zpre & 0xFFFF);
                    }
                }
            }
#pragma unroll
            for (int s = 0; s < kSlices; ++s) {
                zsum[s] += __shfl_xor_sync(0xffffffffu, zsum[s], 1);
                zsum[s] += __shfl_xor_sync(0xffffffffu, zsum[s], 2);
                zsum[s] += __shfl_xor_sync(0xffffffffu, zsum[s], 4);
            }
            if (on && q == 0) {
#pragma unroll
                for (int s = 0; s < kSlices; ++s) zinit[(s * 2 + k) * p.range_max + gloc] = -zsum[s];
                // t = T * 2^-e and the accumulator ends at -T
                zscale[k * p.range_max + gloc] = -__uint_as_float(static_cast<uint32_t>(127 - e) << 23);
            }
        }
        __syncthreads();

        // ---- this lane's z pairs, accumulator seeds and scales
        uint32_t zr[kSlices][2][16];
        int32_t init[kSlices][2];
        float scl[2];
#pragma unroll
        for (int s = 0; s < kSlices; ++s)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    zr[s][k][i] = lane_on ? zp[((s * 2 + k) * 16 + i) * p.range_max + gl] : 0u;
                init[s][k] = lane_on ? zinit[(s * 2 + k) * p.range_max + gl] : 0;
            }
#pragma unroll
        for (int k = 0; k < 2; ++k) scl[k] = lane_on ? zscale[k * p.range_max + gl] : 0.0f;

        // ---- rows: groups of 8 rows dealt round-robin to the streams; the next group's
        // words are loaded while the current group is computed.
        auto load_group = [&](int g, uint2 (&w)[kGroupRows]) {
#pragma unroll
            for (int i = 0; i < kGroupRows; ++i) {
                const int r = g * kGroupRows + i;
                w[i] = (lane_on && g < ngroups && r < nrows)
                           ? __ldg(wcol + static_cast<int64_t>(row0 + r) * p.Wr)
                           : make_uint2(0u, 0u);
            }
        };
        uint2 cur[kGroupRows], nxt[kGroupRows];
        load_group(stream, cur);
        for (int g = stream; g < ngroups; g += p.streams) {
            load_group(g + p.streams, nxt);
            float part[kGroupRows];
#pragma unroll
            for (int i = 0; i < kGroupRows; ++i) {
                const uint2 wd = cur[i];
                float tk[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const uint32_t word = k ? wd.y : wd.x;
                    int32_t acc[kSlices][2];
#pragma unroll
                    for (int s = 0; s < kSlices; ++s) { acc[s][0] = init[s][k]; acc[s][1] = 0; }
#pragma unroll
                    for (int sh = 0; sh < 4; ++sh) {
                        const uint32_t ws = word >> (2 * sh);
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const uint32_t bits = ws & (0x01010101u << jj);
#pragma unroll
                            for (int s = 0; s < kSlices; ++s) {
                                uint32_t a0 = static_cast<uint32_t>(acc[s][sh & 1]);
                                a0 = dp2a_lo(zr[s][k][sh * 4 + jj * 2 + 0], bits, a0);
                                a0 = dp2a_hi(zr[s][k][sh * 4 + jj * 2 + 1], bits, a0);
                                acc[s][sh & 1] = static_cast<int32_t>(a0);
                            }
                        }
                    }
                    if constexpr (kF32X) {
                        const float hi = static_cast<float>(acc[0][0] + acc[0][1]);
                        const float lo = static_cast<float>(acc[1][0] + acc[1][1]);
                        tk[k] = fmaf(hi, 16384.0f, lo) * scl[k];
                    } else {
                        tk[k] = static_cast<float>(acc[0][0] + acc[0][1]) * scl[k];
                    }
                }
                const int r = min(g * kGroupRows + i, max(nrows - 1, 0));
                const float2 av = arow[r];
                part[i] = fmaf(av.x, tk[0], av.y * tk[1]);
            }
            const float total = butterfly8(part, lane);
            const int ri = g * kGroupRows + ((lane >> 2) & 7);
            if ((lane & 3) == 0 && ri < nrows) {
                if (p.nchunks == 1) cred[beta * RB + ri] = total;
                else red[chunk * RB + ri] = total;
            }
#pragma unroll
            for (int i = 0; i < kGroupRows; ++i) cur[i] = nxt[i];
        }
        __syncthreads();
        if (p.nchunks > 1) {
            for (int r = tid; r < nrows; r += nthreads) {
                float s = 0.0f;
                for (int c = 0; c < p.nchunks; ++c) s += red[c * RB + r];
                cred[beta * RB + r] = s;
            }
            __syncthreads();
        }
    }

    // ---- sum the CTAs' partials through distributed shared memory; each CTA stores a share
    cluster_sync_all();
    const int share = (nrows + p.cluster - 1) / p.cluster;
    const int r_lo = static_cast<int>(rank) * share;
    const int r_hi = min(nrows, r_lo + share);
    const int nr = max(r_hi - r_lo, 0);
    const int items = p.batch * nr;
    for (int it = tid; it < items; it += nthreads) {
        const int beta = it / nr;
        const int r = r_lo + it % nr;
        const uint32_t addr = smem_u32(cred + beta * RB + r);
        float s = 0.0f;
        for (int q = 0; q < p.cluster; ++q) s += ld_dsmem_f32(addr, static_cast<uint32_t>(q));
        p.y[static_cast<int64_t>(beta) * p.ldy + row0 + r] = s;
    }
    cluster_sync_all();  // partners are done reading before cred is reused or freed
  }
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// How many clusters of `cs` CTAs (one CTA per SM, the kernel's largest block) the current
// device holds at once; cached per (device, cluster size, activation type).
int cluster_capacity(int cs, bool x_bf16) {
    static int cache[64][9][2] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 1;
    int &slot = cache[dev][cs][x_bf16 ? 1 : 0];
    if (slot == 0) {
        auto kern = x_bf16 ? gemv_kernel<false> : gemv_kernel<true>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(cs));
        cfg.blockDim = dim3(kMaxThreads);
        cfg.dynamicSmemBytes = kSmemBudget;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = 1;
        }
        slot = n;
    }
    return slot;
}

}  // namespace

cudaError_t launch_gemv(const LaunchCtx &ctx, const uint32_t *packed, const float *a,
                        const float *b, int N, int K, const void *x, bool x_bf16, int batch,
                        int ldx, float *y, int ldy) {
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    const int units = Wr / 4;

    // Cluster size (K split) from a cost model in lane-rows of work per CTA: rows x 32 x
    // chunks for the dot products plus ~10 lane-rows per group for quantising z.  The number
    // of clusters is what the GPU can hold at once (clusters live inside one GPC, so fewer
    // than num_sms / cs may fit), so every cluster runs in the first and only wave.
    auto max_clusters = [&](int cs) -> int {
        if (cs == 1) return ctx.num_sms;
        return cluster_capacity(cs, x_bf16);
    };
    int best_cs = 1;
    double best_cost = 1e300;
    const char *force = std::getenv("RABIT_GEMV_CLUSTER");
    const int forced = force ? std::atoi(force) : 0;
    for (int cs = 1; cs <= 8 && cs <= units; ++cs) {
        if (forced > 0 && cs != forced) continue;
        const int ncl = std::min(max_clusters(cs), ceil_div(N, kGroupRows));
        if (ncl < 1) continue;
        const int rpc = ceil_div(N, ncl);
        const int range = ceil_div(units, cs) * 4;
        const int nch = ceil_div(range, 32);
        const double cost = (static_cast<double>(rpc) * nch * 32.0 + 10.0 * range) * batch;
        if (cost < best_cost * 0.97) {
            best_cost = cost;
            best_cs = cs;
        }
    }
    const int cs = best_cs;
    const int ncl = std::min(max_clusters(cs), ceil_div(N, kGroupRows));
    const int rpc = ceil_div(N, ncl);
    const int range_max = ceil_div(units, cs) * 4;
    const int nchunks = ceil_div(range_max, 32);
    const bool f32x = !x_bf16;
    auto bytes_for = [&](int rows) {
        return f32x ? smem_layout<2>(rows, range_max, nchunks, batch).total
                    : smem_layout<1>(rows, range_max, nchunks, batch).total;
    };
    // Rows per block: the cluster's rows if their partial sums fit, else fewer (multiple of 8).
    int block_rows = ceil_div(rpc, kGroupRows) * kGroupRows;
    while (block_rows > kGroupRows && bytes_for(block_rows) > static_cast<uint32_t>(kSmemBudget))
        block_rows -= kGroupRows;
    const uint32_t smem = bytes_for(block_rows);
    const int streams = std::max(1, std::min(kMaxThreads / 32 / nchunks, ceil_div(block_rows, kGroupRows)));
    const int threads = 32 * nchunks * streams;

    GemvArgs p;
    p.packed = reinterpret_cast<const uint2 *>(packed);
    p.a = a;
    p.b = b;
    p.x = x;
    p.y = y;
    p.N = N;
    p.K = K;
    p.Wr = Wr;
    p.batch = batch;
    p.ldx = ldx;
    p.ldy = ldy;
    p.cluster = cs;
    p.rows_per_cluster = rpc;
    p.block_rows = block_rows;
    p.range_max = range_max;
    p.nchunks = nchunks;
    p.streams = streams;

    auto kern = f32x ? gemv_kernel<true> : gemv_kernel<false>;
    // Opt in to the largest dynamic shared memory once per kernel and device.
    static int opted[2][64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !opted[f32x][dev]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBudget);
        if (e != cudaSuccess) return e;
        opted[f32x][dev] = 1;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ncl * cs));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cs);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace rabit
