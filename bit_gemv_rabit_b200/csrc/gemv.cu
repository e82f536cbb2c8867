// gemv.cu -- decode path of the residual-binary linear layer, batch 1..16.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.1 "Multi-bit Approximation via Stacking" executed per path as described in
// Appendix E.1 "Compute Pipeline" (paths in parallel, signs applied without multiplies,
// warp-shuffle reduction, output scale applied last):
//     y[beta][n] = sum_k a_k[n] * t_k[beta][n],   t_k[beta][n] = sum_j S_k[n][j] z_k[beta][j],
//     z_k[beta][j] = b_k[j] * x[beta][j].
//
// Design for sm_100a (CUDA cores; the integer dot-product pipe sets the compute bound):
//
//  * Signs as masked sums.  t = Z - 2*sum_{bit=1} z with Z = sum_j z.  For each 32-column
//    group z is quantised to 13-bit integers with a power-of-two scale of its own (the group
//    max fixes it, so the error is relative to the local maximum).  One 3-input logic op
//    isolates four sign bits of a word at one position q in each byte (values 0 or 2^q),
//    and a dp2a multiplies two of those bytes with two pre-shifted 16-bit z values and
//    accumulates in 32-bit: the integer sum is exact.  Four bit positions per byte
//    (q = 0..3, then the word shifted by 4) with z pre-shifted by 2^(3-q) give every product
//    the same weight 8*z, so each path needs one accumulator, seeded with -4Z.  Per 32
//    weight bits: 16 dp2a (the fma-heavy pipe, which bounds the kernel), 8 logic ops and
//    one shift.
//  * A CTA owns a contiguous block of whole rows, which is one contiguous range of the
//    row-major packed layout: TMA bulk copies (one per 8 rows, each completing on its own
//    mbarrier) bring it into shared memory, so the weight stream has deep memory-level
//    parallelism and no per-lane address work.  Before the programmatic-launch wait only L2
//    prefetches are issued (of the block, of x, a and b): a prefetch returns no data to the
//    SM, so it cannot observe a value the previous kernel on the stream is still writing.
//  * Lane = 32-column group.  A work item is 8 rows x one chunk of 32 groups; items are
//    dealt round-robin to the warps.  Each lane reads its group's word pair for the 8 rows
//    and its 16 z-pair words per path (four 16-byte shared loads), runs 8 independent
//    accumulation chains, a butterfly sums the 8 rows over the lanes, and the chunk
//    partials meet in shared memory.
//  * RABIT_F32 activations use two 13-bit slices of a 24-bit z (twice the dp2a work).
//  * Batch 2..16: when the CTA's rows and the z tables of 4 (or 2) batch rows fit in shared
//    memory together, one z stage serves those rows (b loaded once) and the rows sweep
//    isolates each word's bit positions once for all of them.  Otherwise the batch rows go
//    one at a time over the staged weights.
#include <algorithm>
#include <type_traits>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kMaxThreads = 768;
// fp32 activations (two slices per z value) and three paths need more registers per thread.
__host__ __device__ constexpr int max_threads(bool f32x, int P) { return (f32x || P == 3) ? 512 : kMaxThreads; }
constexpr int kGroupRows = 8;            // rows per butterfly reduction and per copy barrier
constexpr int kSmemBudget = 200 * 1024;  // dynamic shared memory a CTA may use
// A group's 16 z-pair words per path and slice sit together, 20 words apart from the next
// group's: a lane loads its own with four 16-byte reads, and the 8 lanes of a quarter warp
// land on disjoint banks.
constexpr int kZStride = 20;

struct GemvArgs {
    const uint32_t *packed;  // [N][Wr] groups of G words: the paths' words (+ a zero word for 3)
    const float *a;        // [P][N]
    const float *b;        // [P][K]
    const void *x;         // [batch][ldx]
    float *y;              // [batch][ldy]
    uint32_t *fault;
    uint64_t timeout_ns;
    int N, K, Wr, batch, ldx, ldy;
    int rows_per_cta;      // contiguous rows owned by one CTA
    int pass_rows;         // rows staged in shared memory at a time (multiple of 8)
    int nchunks;           // 32-group chunks of a row
    int vec_x;             // x rows 16-byte aligned: 16-byte loads of 8 columns
    int vec_b;             // every b row 16-byte aligned
};

// Words per 32-column group: two paths as a uint2, three paths as a uint4 (the fourth word is
// padding), as Appendix E.1 groups them.
template <int kP> using GroupWords = typename std::conditional<kP == 2, uint2, uint4>::type;
// Per-row output scales in shared memory: {a_1, a_2} or {a_1, a_2, a_3, 0}.
template <int kP> using RowScales = typename std::conditional<kP == 2, float2, float4>::type;

struct SmemLayout {
    uint32_t w, zp, zinit, zscale, arow, red, bar, total;
};

// Per-group tables have rows Wr + 1 words apart, which keeps their stores conflict-free.
template <int kSlices, int kP>
__host__ __device__ inline SmemLayout smem_layout(int pass_rows, int Wr, int nchunks) {
    SmemLayout L;
    uint32_t off = 0;
    auto take = [&](uint32_t bytes) { uint32_t o = off; off = (off + bytes + 127u) & ~127u; return o; };
    L.w = take(static_cast<uint32_t>(pass_rows) * Wr * static_cast<uint32_t>(sizeof(GroupWords<kP>)));
    L.zp = take(static_cast<uint32_t>(kSlices) * kP * Wr * kZStride * 4u);
    L.zinit = take(static_cast<uint32_t>(kSlices) * kP * (Wr + 1) * 4u);
    L.zscale = take(static_cast<uint32_t>(kP) * (Wr + 1) * 4u);
    L.arow = take(static_cast<uint32_t>(pass_rows) * static_cast<uint32_t>(sizeof(RowScales<kP>)));
    L.red = take(static_cast<uint32_t>(nchunks) * pass_rows * 4u);
    L.bar = take(static_cast<uint32_t>(pass_rows / kGroupRows) * 8u);
    L.total = off;
    return L;
}

__device__ __forceinline__ uint32_t path_word(const uint2 &g, int k) { return k ? g.y : g.x; }
__device__ __forceinline__ uint32_t path_word(const uint4 &g, int k) { return k == 0 ? g.x : (k == 1 ? g.y : g.z); }

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
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                 ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
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

// Columns j0..j0+7 of batch row beta of x; columns at or past K read as 0 (the padding of
// the last group).
template <bool kF32X>
__device__ __forceinline__ void load_x8(const GemvArgs &p, int beta, int j0, bool on, float (&xv)[8]) {
    const int64_t xrow = static_cast<int64_t>(beta) * p.ldx;
    if (on && j0 + 8 <= p.K && p.vec_x) {
        if constexpr (kF32X) {
            const float4 *src = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(p.x) + xrow + j0);
            const float4 u0 = __ldg(src), u1 = __ldg(src + 1);
            xv[0] = u0.x; xv[1] = u0.y; xv[2] = u0.z; xv[3] = u0.w;
            xv[4] = u1.x; xv[5] = u1.y; xv[6] = u1.z; xv[7] = u1.w;
        } else {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(
                reinterpret_cast<const unsigned short *>(p.x) + xrow + j0));
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xv[2 * i] = __uint_as_float(w4[i] << 16);
                xv[2 * i + 1] = __uint_as_float(w4[i] & 0xFFFF0000u);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[i] = on && j0 + i < p.K ? load_x<kF32X>(p.x, xrow + j0 + i) : 0.0f;
    }
}

// Columns j0..j0+7 of every b row, 0 at or past K.
template <int kP>
__device__ __forceinline__ void load_b8(const GemvArgs &p, int j0, bool on, float (&bv)[kP][8]) {
    if (on && j0 + 8 <= p.K && p.vec_b) {
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            const float4 *brow = reinterpret_cast<const float4 *>(p.b + static_cast<int64_t>(k) * p.K + j0);
            const float4 u0 = __ldg(brow), u1 = __ldg(brow + 1);
            bv[k][0] = u0.x; bv[k][1] = u0.y; bv[k][2] = u0.z; bv[k][3] = u0.w;
            bv[k][4] = u1.x; bv[k][5] = u1.y; bv[k][6] = u1.z; bv[k][7] = u1.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int k = 0; k < kP; ++k)
                bv[k][i] = on && j0 + i < p.K ? __ldg(p.b + static_cast<int64_t>(k) * p.K + j0 + i) : 0.0f;
    }
}

// Loads of one z task: 8 columns j0..j0+7 of x (batch row beta) and of every b row.
template <bool kF32X, int kP>
__device__ __forceinline__ void load_ztask(const GemvArgs &p, int beta, int j0, bool on,
                                           float (&xv)[8], float (&bv)[kP][8]) {
    load_x8<kF32X>(p, beta, j0, on, xv);
    load_b8<kP>(p, j0, on, bv);
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

template <bool kF32X, int kP>
__global__ void __launch_bounds__(max_threads(kF32X, kP), 1)
gemv_kernel(const GemvArgs p) {
    constexpr int kSlices = kF32X ? 2 : 1;
    using WG = GroupWords<kP>;
    using AS = RowScales<kP>;
    extern __shared__ __align__(128) uint8_t smem[];
    const SmemLayout L = smem_layout<kSlices, kP>(p.pass_rows, p.Wr, p.nchunks);
    WG *wbuf = reinterpret_cast<WG *>(smem + L.w);                   // [pass_rows][Wr]
    uint32_t *zp = reinterpret_cast<uint32_t *>(smem + L.zp);        // [slice][path][Wr][kZStride]
    int32_t *zinit = reinterpret_cast<int32_t *>(smem + L.zinit);    // [slice][path][zs]
    float *zscale = reinterpret_cast<float *>(smem + L.zscale);      // [path][zs]
    AS *arow = reinterpret_cast<AS *>(smem + L.arow);                // [pass_rows]
    float *red = reinterpret_cast<float *>(smem + L.red);            // [nchunks][pass_rows]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar);     // [pass_rows / 8]
    const int zs = p.Wr + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x;
    const int nwarps = nthreads >> 5;
    const int row_begin = blockIdx.x * p.rows_per_cta;
    const int row_end = min(p.N, row_begin + p.rows_per_cta);
    if (row_begin >= row_end) return;  // whole CTA, before any barrier
    int abort_flag = 0;

    if (tid == 0) {
        for (int g = 0; g < p.pass_rows / kGroupRows; ++g) mbar_init(smem_u32(&bars[g]), 1);
        fence_mbarrier_init();
        // L2 prefetch of this CTA's rows (one contiguous block)
        const uint8_t *base = reinterpret_cast<const uint8_t *>(
            reinterpret_cast<const WG *>(p.packed) + static_cast<int64_t>(row_begin) * p.Wr);
        const uint64_t bytes = static_cast<uint64_t>(row_end - row_begin) * p.Wr * sizeof(WG);
        for (uint64_t o = 0; o < bytes; o += (1u << 20))
            bulk_prefetch_l2(base + o, static_cast<uint32_t>(min(bytes - o, static_cast<uint64_t>(1u << 20))));
    } else if (warp == 1) {
        for (int c = lane * 32; c < p.K; c += 32 * 32)                   // 128-byte lines of b
            for (int k = 0; k < kP; ++k) prefetch_l2(p.b + static_cast<int64_t>(k) * p.K + c);
    } else if (warp == 2) {
        for (int r = lane * 32; r < row_end - row_begin; r += 32 * 32)   // lines of a
            for (int k = 0; k < kP; ++k) prefetch_l2(p.a + static_cast<int64_t>(k) * p.N + row_begin + r);
    } else if (warp == 3) {
        const int per_line = kF32X ? 32 : 64;
        for (int beta = 0; beta < p.batch; ++beta)
            for (int c = lane * per_line; c < p.K; c += 32 * per_line)
                prefetch_l2(reinterpret_cast<const uint8_t *>(p.x) +
                            (static_cast<int64_t>(beta) * p.ldx + c) * (kF32X ? 4 : 2));
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    uint32_t parity = 0;
    for (int pr0 = row_begin; pr0 < row_end; pr0 += p.pass_rows, parity ^= 1u) {
        const int prows = min(p.pass_rows, row_end - pr0);
        const int ngroups = (prows + kGroupRows - 1) / kGroupRows;
        // ---- stage the pass's rows: one bulk copy per 8 rows, each on its own barrier
        if (warp == 0) {
            for (int g = lane; g < ngroups; g += 32) {
                const int rows_g = min(kGroupRows, prows - g * kGroupRows);
                const uint32_t bytes = static_cast<uint32_t>(rows_g) * p.Wr * static_cast<uint32_t>(sizeof(WG));
                const uint32_t bar = smem_u32(&bars[g]);
                mbar_arrive_expect_tx(bar, bytes);
                bulk_g2s(smem_u32(wbuf + static_cast<int64_t>(g) * kGroupRows * p.Wr),
                         reinterpret_cast<const WG *>(p.packed) + static_cast<int64_t>(pr0 + g * kGroupRows) * p.Wr,
                         bytes, bar);
            }
        }
        for (int beta = 0; beta < p.batch; ++beta) {
            // ---- z_k = x (.) b_k over the whole row, quantised per 32-column group and path.
            // 4 consecutive threads per group, 8 columns each; x is read once for both paths.
            // The loads of kZBatch tasks are issued before any of them is used, and a's values
            // for the pass are fetched alongside, so the stage waits on memory about once.
            auto load_scales = [&](int r) -> AS {
                if constexpr (kP == 2)
                    return make_float2(__ldg(p.a + pr0 + r), __ldg(p.a + p.N + pr0 + r));
                else
                    return make_float4(__ldg(p.a + pr0 + r), __ldg(p.a + p.N + pr0 + r),
                                       __ldg(p.a + 2 * static_cast<int64_t>(p.N) + pr0 + r), 0.0f);
            };
            AS apre{};
            if (beta == 0 && tid < prows) apre = load_scales(tid);
            constexpr int kZBatch = 2;
            const int ztasks = 4 * p.Wr;
            const int ztasks_pad = (ztasks + 31) & ~31;
            for (int t0 = tid; t0 < ztasks_pad; t0 += kZBatch * nthreads) {
                float xv[kZBatch][8], zv[kZBatch][kP][8];
#pragma unroll
                for (int u = 0; u < kZBatch; ++u) {
                    const int t = t0 + u * nthreads;
                    load_ztask<kF32X, kP>(p, beta, (t >> 2) * 32 + 8 * (t & 3), t < ztasks, xv[u], zv[u]);
                }
#pragma unroll
                for (int u = 0; u < kZBatch; ++u) {
                    const int t = t0 + u * nthreads;
                    if (t - tid >= ztasks_pad) break;   // warp-uniform: t - tid is the same for all lanes
                    const bool on = t < ztasks;
                    const int q = t & 3;
                    const int gloc = on ? (t >> 2) : 0;
                    const int h = q >> 1, half = q & 1;  // columns 8q..8q+7 of the group
#pragma unroll
                    for (int k = 0; k < kP; ++k) {
                        float m = 0.0f;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            zv[u][k][i] *= xv[u][i];
                            m = fmaxf(m, fabsf(zv[u][k][i]));
                        }
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
                        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
                        // power-of-two scale 2^e with m * 2^e <= kMaxQ (13-bit, or 24-bit for fp32 x)
                        constexpr int kTop = kF32X ? 22 : 11;
                        const float kMaxQ = kF32X ? 8388607.0f : 4095.0f;
                        const int E = static_cast<int>((__float_as_uint(m) >> 23) & 0xFFu) - 127;
                        int e = min(124, max(-126, kTop - E));
                        float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
                        if (m * sc > kMaxQ) { --e; sc *= 0.5f; }
                        int zsum[kSlices];
#pragma unroll
                        for (int s = 0; s < kSlices; ++s) zsum[s] = 0;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            // column 8q+i sits at bit i of byte q: bit position i&3 after a shift
                            // by 4*(i>>2); dp2a.lo takes bytes 0,1 and dp2a.hi bytes 2,3
                            const int qb = i & 3;
                            const int pair = (i >> 2) * 8 + qb * 2 + h;
                            int part[kSlices];
                            if constexpr (kF32X) {
                                const int zq = __float2int_rn(zv[u][k][i] * sc);
                                part[0] = (zq + (1 << 11)) >> 12;       // high 13-bit slice
                                part[1] = zq - (part[0] << 12);         // low slice, in [-2^11, 2^11)
                            } else {
                                // round to nearest even by adding 1.5 * 2^23 (|z * 2^e| < 2^22)
                                part[0] = __float_as_int(fmaf(zv[u][k][i], sc, 12582912.0f)) - 0x4B400000;
                            }
#pragma unroll
                            for (int s = 0; s < kSlices; ++s) {
                                zsum[s] += part[s];
                                if (on) {
                                    const int zpre = part[s] << (3 - qb);      // weight 2^(3-q)
                                    uint16_t *slot = reinterpret_cast<uint16_t *>(
                                        zp + ((s * kP + k) * p.Wr + gloc) * kZStride + pair) + half;
                                    *slot = static_cast<uint16_t>(zpre & 0xFFFF);
                                }
                            }
                        }
#pragma unroll
                        for (int s = 0; s < kSlices; ++s) {
                            zsum[s] += __shfl_xor_sync(0xffffffffu, zsum[s], 1);
                            zsum[s] += __shfl_xor_sync(0xffffffffu, zsum[s], 2);
                        }
                        if (on && q == 0) {
#pragma unroll
                            for (int s = 0; s < kSlices; ++s) zinit[(s * kP + k) * zs + gloc] = -4 * zsum[s];
                            // the accumulator ends at -4T and t = T * 2^-e
                            zscale[k * zs + gloc] = -__uint_as_float(static_cast<uint32_t>(125 - e) << 23);
                        }
                    }
                }
            }
            if (beta == 0) {
                if (tid < prows) arow[tid] = apre;
                for (int r = tid + nthreads; r < p.pass_rows; r += nthreads)   // rows past prows: a = 0
                    arow[r] = r < prows ? load_scales(r) : AS{};
                if (tid >= prows && tid < p.pass_rows) arow[tid] = AS{};
            }
            __syncthreads();

            // ---- rows: work items (8 rows x one 32-group chunk) dealt round-robin to the warps.
            // Rows past prows in the last group read stale words of the pass buffer; their a is
            // 0 and their totals are never stored.
            const int nitems = ngroups * p.nchunks;
            // (g, c) of item warp + j * nwarps, advanced without a division per item
            const int gstep = nwarps / p.nchunks, cstep = nwarps - gstep * p.nchunks;
            int g = warp / p.nchunks, c = warp - (warp / p.nchunks) * p.nchunks;
            for (int item = warp; item < nitems; item += nwarps) {
                const int gl = c * 32 + lane;
                const bool lane_on = gl < p.Wr;
                const int gz = lane_on ? gl : p.Wr - 1;     // lanes past the row read a valid word
                float sk[kP];
                const bool landed = beta != 0 || mbar_wait_bounded(smem_u32(&bars[g]), parity, &abort_flag,
                                                                   p.timeout_ns, p.fault, FAULT_GEMV_WAIT_COPY);
#pragma unroll
                for (int k = 0; k < kP; ++k)   // a copy that never landed contributes nothing
                    sk[k] = landed && lane_on ? zscale[k * zs + gz] : 0.0f;
                WG w[kGroupRows];
                const WG *wrow = wbuf + static_cast<int64_t>(g) * kGroupRows * p.Wr + gz;
#pragma unroll
                for (int i = 0; i < kGroupRows; ++i) w[i] = wrow[static_cast<int64_t>(i) * p.Wr];
                float tk[kP][kGroupRows];
#pragma unroll
                for (int k = 0; k < kP; ++k) {
                    int32_t acc[kSlices][kGroupRows];
                    uint4 zq[kSlices][4];
#pragma unroll
                    for (int s = 0; s < kSlices; ++s) {
                        const uint4 *zrow = reinterpret_cast<const uint4 *>(zp + ((s * kP + k) * p.Wr + gz) * kZStride);
#pragma unroll
                        for (int j = 0; j < 4; ++j) zq[s][j] = zrow[j];
                        const int32_t init = zinit[(s * kP + k) * zs + gz];
#pragma unroll
                        for (int i = 0; i < kGroupRows; ++i) acc[s][i] = init;
                    }
                    // bit position q of every byte (after a shift by 0 or 4) has the value 2^q;
                    // z is pre-shifted by 2^(3-q), so every product weighs 8 z
#pragma unroll
                    for (int s4 = 0; s4 < 2; ++s4) {
#pragma unroll
                        for (int i = 0; i < kGroupRows; ++i) {
                            const uint32_t wv = path_word(w[i], k) >> (4 * s4);
#pragma unroll
                            for (int s = 0; s < kSlices; ++s) {
                                uint32_t a0 = static_cast<uint32_t>(acc[s][i]);
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    const uint32_t bq = wv & (0x01010101u << q);
                                    const uint4 &zz = zq[s][s4 * 2 + (q >> 1)];
                                    a0 = dp2a_lo((q & 1) ? zz.z : zz.x, bq, a0);
                                    a0 = dp2a_hi((q & 1) ? zz.w : zz.y, bq, a0);
                                }
                                acc[s][i] = static_cast<int32_t>(a0);
                            }
                        }
                    }
                    // |acc| < 2^21: the conversions are exact
#pragma unroll
                    for (int i = 0; i < kGroupRows; ++i) {
                        float t = static_cast<float>(acc[0][i]);
                        if constexpr (kF32X) t = fmaf(t, 4096.0f, static_cast<float>(acc[1][i]));
                        tk[k][i] = t * sk[k];
                    }
                }
                float part[kGroupRows];
                if constexpr (kP == 2) {
                    const float4 *a4 = reinterpret_cast<const float4 *>(arow + g * kGroupRows);
#pragma unroll
                    for (int i = 0; i < kGroupRows / 2; ++i) {
                        const float4 av = a4[i];
                        part[2 * i] = fmaf(av.x, tk[0][2 * i], av.y * tk[1][2 * i]);
                        part[2 * i + 1] = fmaf(av.z, tk[0][2 * i + 1], av.w * tk[1][2 * i + 1]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < kGroupRows; ++i) {
                        const float4 av = arow[g * kGroupRows + i];
                        part[i] = fmaf(av.x, tk[0][i], fmaf(av.y, tk[1][i], av.z * tk[2][i]));
                    }
                }
                const float total = butterfly8(part, lane);
                const int ri = g * kGroupRows + ((lane >> 2) & 7);
                if ((lane & 3) == 0 && ri < prows) red[c * p.pass_rows + ri] = total;
                g += gstep;
                c += cstep;
                if (c >= p.nchunks) { c -= p.nchunks; ++g; }
            }
            __syncthreads();
            // ---- y = sum of the chunk partials
            for (int r = tid; r < prows; r += nthreads) {
                float s = 0.0f;
                for (int c = 0; c < p.nchunks; ++c) s += red[c * p.pass_rows + r];
                p.y[static_cast<int64_t>(beta) * p.ldy + pr0 + r] = s;
            }
            __syncthreads();  // red, z tables and (after the last batch row) the pass buffer are reused
        }
    }
}

// ---------------------------------------------------------------- several batch rows at once
// For batch >= 2 the z tables of kNB batch rows live in shared memory together: b is loaded
// once per z task for all of them, and in the rows phase the isolated sign bytes of a word
// serve every batch row's dp2a (the logic ops are shared).

template <int kSlices, int kP>
__host__ __device__ inline SmemLayout smem_layout_multi(int pass_rows, int Wr, int nchunks, int nb) {
    SmemLayout L;
    uint32_t off = 0;
    auto take = [&](uint32_t bytes) { uint32_t o = off; off = (off + bytes + 127u) & ~127u; return o; };
    L.w = take(static_cast<uint32_t>(pass_rows) * Wr * static_cast<uint32_t>(sizeof(GroupWords<kP>)));
    L.zp = take(static_cast<uint32_t>(nb) * kSlices * kP * Wr * kZStride * 4u);
    L.zinit = take(static_cast<uint32_t>(nb) * kSlices * kP * (Wr + 1) * 4u);
    L.zscale = take(static_cast<uint32_t>(nb) * kP * (Wr + 1) * 4u);
    L.arow = take(static_cast<uint32_t>(pass_rows) * static_cast<uint32_t>(sizeof(RowScales<kP>)));
    L.red = take(static_cast<uint32_t>(nb) * nchunks * pass_rows * 4u);
    L.bar = take(static_cast<uint32_t>(pass_rows / kGroupRows) * 8u);
    L.total = off;
    return L;
}

// One z task of one batch row: quantise columns 8q..8q+7 of group gloc for every path (z = x * b,
// zv holds b on entry) and write the row's tables.  Lanes of a group are consecutive.
template <bool kF32X, int kP>
__device__ __forceinline__ void z_task_store(const GemvArgs &p, bool on, int gloc, int q, const float (&xv)[8],
                                             float (&zv)[kP][8], uint32_t *zp, int32_t *zinit, float *zscale) {
    constexpr int kSlices = kF32X ? 2 : 1;
    const int zs = p.Wr + 1;
    const int h = q >> 1, half = q & 1;
#pragma unroll
    for (int k = 0; k < kP; ++k) {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            zv[k][i] *= xv[i];
            m = fmaxf(m, fabsf(zv[k][i]));
        }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        constexpr int kTop = kF32X ? 22 : 11;
        const float kMaxQ = kF32X ? 8388607.0f : 4095.0f;
        const int E = static_cast<int>((__float_as_uint(m) >> 23) & 0xFFu) - 127;
        int e = min(124, max(-126, kTop - E));
        float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
        if (m * sc > kMaxQ) { --e; sc *= 0.5f; }
        int zsum[kSlices];
#pragma unroll
        for (int s = 0; s < kSlices; ++s) zsum[s] = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int qb = i & 3;
            const int pair = (i >> 2) * 8 + qb * 2 + h;
            int part[kSlices];
            if constexpr (kF32X) {
                const int zq = __float2int_rn(zv[k][i] * sc);
                part[0] = (zq + (1 << 11)) >> 12;
                part[1] = zq - (part[0] << 12);
            } else {
                part[0] = __float_as_int(fmaf(zv[k][i], sc, 12582912.0f)) - 0x4B400000;
            }
#pragma unroll
            for (int s = 0; s < kSlices; ++s) {
                zsum[s] += part[s];
                if (on) {
                    uint16_t *slot = reinterpret_cast<uint16_t *>(zp + ((s * kP + k) * p.Wr + gloc) * kZStride + pair) + half;
                    *slot = static_cast<uint16_t>((part[s] << (3 - qb)) & 0xFFFF);
                }
            }
        }
#pragma unroll
        for (int s = 0; s < kSlices; ++s) {
            zsum[s] += __shfl_xor_sync(0xffffffffu, zsum[s], 1);
            zsum[s] += __shfl_xor_sync(0xffffffffu, zsum[s], 2);
        }
        if (on && q == 0) {
#pragma unroll
            for (int s = 0; s < kSlices; ++s) zinit[(s * kP + k) * zs + gloc] = -4 * zsum[s];
            zscale[k * zs + gloc] = -__uint_as_float(static_cast<uint32_t>(125 - e) << 23);
        }
    }
}

constexpr int kMultiThreads = 384;

template <bool kF32X, int kP, int kNB>
__global__ void __launch_bounds__(kMultiThreads, 1)
gemv_multi_kernel(const GemvArgs p) {
    constexpr int kSlices = kF32X ? 2 : 1;
    using WG = GroupWords<kP>;
    using AS = RowScales<kP>;
    extern __shared__ __align__(128) uint8_t smem[];
    const SmemLayout L = smem_layout_multi<kSlices, kP>(p.pass_rows, p.Wr, p.nchunks, kNB);
    WG *wbuf = reinterpret_cast<WG *>(smem + L.w);
    uint32_t *zp0 = reinterpret_cast<uint32_t *>(smem + L.zp);       // [nb][slice][path][Wr][kZStride]
    int32_t *zinit0 = reinterpret_cast<int32_t *>(smem + L.zinit);   // [nb][slice][path][zs]
    float *zscale0 = reinterpret_cast<float *>(smem + L.zscale);     // [nb][path][zs]
    AS *arow = reinterpret_cast<AS *>(smem + L.arow);
    float *red = reinterpret_cast<float *>(smem + L.red);            // [nb][nchunks][pass_rows]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bar);
    const int zs = p.Wr + 1;
    const int zp_stride = kSlices * kP * p.Wr * kZStride;            // words per batch row
    const int zi_stride = kSlices * kP * zs;
    const int zc_stride = kP * zs;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;
    const int row_begin = blockIdx.x * p.rows_per_cta;
    const int row_end = min(p.N, row_begin + p.rows_per_cta);
    if (row_begin >= row_end) return;
    int abort_flag = 0;

    if (tid == 0) {
        for (int g = 0; g < p.pass_rows / kGroupRows; ++g) mbar_init(smem_u32(&bars[g]), 1);
        fence_mbarrier_init();
        const uint8_t *base = reinterpret_cast<const uint8_t *>(
            reinterpret_cast<const WG *>(p.packed) + static_cast<int64_t>(row_begin) * p.Wr);
        const uint64_t bytes = static_cast<uint64_t>(row_end - row_begin) * p.Wr * sizeof(WG);
        for (uint64_t o = 0; o < bytes; o += (1u << 20))
            bulk_prefetch_l2(base + o, static_cast<uint32_t>(min(bytes - o, static_cast<uint64_t>(1u << 20))));
    } else if (warp == 1) {
        for (int c = lane * 32; c < p.K; c += 32 * 32)
            for (int k = 0; k < kP; ++k) prefetch_l2(p.b + static_cast<int64_t>(k) * p.K + c);
    } else if (warp == 2) {
        for (int r = lane * 32; r < row_end - row_begin; r += 32 * 32)
            for (int k = 0; k < kP; ++k) prefetch_l2(p.a + static_cast<int64_t>(k) * p.N + row_begin + r);
    } else if (warp == 3) {
        const int per_line = kF32X ? 32 : 64;
        for (int beta = 0; beta < p.batch; ++beta)
            for (int c = lane * per_line; c < p.K; c += 32 * per_line)
                prefetch_l2(reinterpret_cast<const uint8_t *>(p.x) +
                            (static_cast<int64_t>(beta) * p.ldx + c) * (kF32X ? 4 : 2));
    }
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    uint32_t parity = 0;
    for (int pr0 = row_begin; pr0 < row_end; pr0 += p.pass_rows, parity ^= 1u) {
        const int prows = min(p.pass_rows, row_end - pr0);
        const int ngroups = (prows + kGroupRows - 1) / kGroupRows;
        if (warp == 0) {
            for (int g = lane; g < ngroups; g += 32) {
                const int rows_g = min(kGroupRows, prows - g * kGroupRows);
                const uint32_t bytes = static_cast<uint32_t>(rows_g) * p.Wr * static_cast<uint32_t>(sizeof(WG));
                const uint32_t bar = smem_u32(&bars[g]);
                mbar_arrive_expect_tx(bar, bytes);
                bulk_g2s(smem_u32(wbuf + static_cast<int64_t>(g) * kGroupRows * p.Wr),
                         reinterpret_cast<const WG *>(p.packed) + static_cast<int64_t>(pr0 + g * kGroupRows) * p.Wr,
                         bytes, bar);
            }
        }
        for (int r = tid; r < p.pass_rows; r += nthreads) {
            if (r < prows) {
                if constexpr (kP == 2)
                    arow[r] = make_float2(__ldg(p.a + pr0 + r), __ldg(p.a + p.N + pr0 + r));
                else
                    arow[r] = make_float4(__ldg(p.a + pr0 + r), __ldg(p.a + p.N + pr0 + r),
                                          __ldg(p.a + 2 * static_cast<int64_t>(p.N) + pr0 + r), 0.0f);
            } else {
                arow[r] = AS{};
            }
        }
        bool first_chunk = true;
        for (int beta0 = 0; beta0 < p.batch; beta0 += kNB) {
            const int nbc = min(kNB, p.batch - beta0);
            // ---- z tables of the chunk's batch rows: b loaded once per task
            const int ztasks = 4 * p.Wr;
            const int ztasks_pad = (ztasks + 31) & ~31;
            for (int t = tid; t < ztasks_pad; t += nthreads) {
                const bool on = t < ztasks;
                const int gloc = on ? (t >> 2) : 0, q = t & 3;
                const int j0 = gloc * 32 + 8 * q;
                float bv[kP][8], xv[kNB][8];
                load_b8<kP>(p, j0, on, bv);
#pragma unroll
                for (int bb = 0; bb < kNB; ++bb)
                    if (bb < nbc) load_x8<kF32X>(p, beta0 + bb, j0, on, xv[bb]);
#pragma unroll
                for (int bb = 0; bb < kNB; ++bb) {
                    if (bb >= nbc) break;                    // uniform
                    float zv[kP][8];
#pragma unroll
                    for (int k = 0; k < kP; ++k)
#pragma unroll
                        for (int i = 0; i < 8; ++i) zv[k][i] = bv[k][i];
                    z_task_store<kF32X, kP>(p, on, gloc, q, xv[bb], zv, zp0 + bb * zp_stride,
                                            zinit0 + bb * zi_stride, zscale0 + bb * zc_stride);
                }
            }
            __syncthreads();

            // ---- rows: items (8 rows x 32 groups) round-robin; the sign bytes of each word are
            // isolated once and feed every batch row of the chunk
            const int nitems = ngroups * p.nchunks;
            for (int item = warp; item < nitems; item += nwarps) {
                const int g = item / p.nchunks, c = item - g * p.nchunks;
                const int gl = c * 32 + lane;
                const bool lane_on = gl < p.Wr;
                const int gz = lane_on ? gl : p.Wr - 1;
                const bool landed = !first_chunk || mbar_wait_bounded(smem_u32(&bars[g]), parity, &abort_flag,
                                                                      p.timeout_ns, p.fault, FAULT_GEMV_WAIT_COPY);
                float part[kNB][kGroupRows];
#pragma unroll
                for (int bb = 0; bb < kNB; ++bb)
#pragma unroll
                    for (int i = 0; i < kGroupRows; ++i) part[bb][i] = 0.0f;
                const WG *wrow = wbuf + static_cast<int64_t>(g) * kGroupRows * p.Wr + gz;
#pragma unroll 1
                for (int k = 0; k < kP; ++k) {
                    uint32_t wk[kGroupRows];
#pragma unroll
                    for (int i = 0; i < kGroupRows; ++i)
                        wk[i] = reinterpret_cast<const uint32_t *>(wrow + static_cast<int64_t>(i) * p.Wr)[k];
                    int32_t acc[kNB][kSlices][kGroupRows];
#pragma unroll
                    for (int bb = 0; bb < kNB; ++bb)
#pragma unroll
                        for (int s = 0; s < kSlices; ++s) {
                            const int32_t init = zinit0[bb * zi_stride + (s * kP + k) * zs + gz];
#pragma unroll
                            for (int i = 0; i < kGroupRows; ++i) acc[bb][s][i] = init;
                        }
#pragma unroll
                    for (int s4 = 0; s4 < 2; ++s4) {
#pragma unroll
                        for (int qp = 0; qp < 2; ++qp) {
                            uint4 zz[kNB][kSlices];
#pragma unroll
                            for (int bb = 0; bb < kNB; ++bb)
#pragma unroll
                                for (int s = 0; s < kSlices; ++s)
                                    zz[bb][s] = reinterpret_cast<const uint4 *>(
                                        zp0 + bb * zp_stride + ((s * kP + k) * p.Wr + gz) * kZStride)[s4 * 2 + qp];
#pragma unroll
                            for (int qq = 0; qq < 2; ++qq) {
                                const int q = 2 * qp + qq;
#pragma unroll
                                for (int i = 0; i < kGroupRows; ++i) {
                                    const uint32_t bq = (wk[i] >> (4 * s4)) & (0x01010101u << q);
#pragma unroll
                                    for (int bb = 0; bb < kNB; ++bb)
#pragma unroll
                                        for (int s = 0; s < kSlices; ++s) {
                                            uint32_t a0 = static_cast<uint32_t>(acc[bb][s][i]);
                                            a0 = dp2a_lo(qq ? zz[bb][s].z : zz[bb][s].x, bq, a0);
                                            a0 = dp2a_hi(qq ? zz[bb][s].w : zz[bb][s].y, bq, a0);
                                            acc[bb][s][i] = static_cast<int32_t>(a0);
                                        }
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int bb = 0; bb < kNB; ++bb) {
                        const float sk = landed && lane_on ? zscale0[bb * zc_stride + k * zs + gz] : 0.0f;
#pragma unroll
                        for (int i = 0; i < kGroupRows; ++i) {
                            float t = static_cast<float>(acc[bb][0][i]);
                            if constexpr (kF32X) t = fmaf(t, 4096.0f, static_cast<float>(acc[bb][1][i]));
                            const float ak = reinterpret_cast<const float *>(arow + g * kGroupRows + i)[k];
                            part[bb][i] = fmaf(ak, t * sk, part[bb][i]);
                        }
                    }
                }
#pragma unroll
                for (int bb = 0; bb < kNB; ++bb) {
                    const float total = butterfly8(part[bb], lane);
                    const int ri = g * kGroupRows + ((lane >> 2) & 7);
                    if ((lane & 3) == 0 && ri < prows && bb < nbc)
                        red[(bb * p.nchunks + c) * p.pass_rows + ri] = total;
                }
            }
            __syncthreads();
            for (int u = tid; u < nbc * prows; u += nthreads) {
                const int bb = u / prows, r = u - bb * prows;
                float sum = 0.0f;
                for (int cc = 0; cc < p.nchunks; ++cc) sum += red[(bb * p.nchunks + cc) * p.pass_rows + r];
                p.y[static_cast<int64_t>(beta0 + bb) * p.ldy + pr0 + r] = sum;
            }
            __syncthreads();   // z tables, red and (after the last chunk) the pass buffer are reused
            first_chunk = false;
        }
    }
}

int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace

cudaError_t launch_gemv(const LaunchCtx &ctx, const uint32_t *packed, const float *a,
                        const float *b, int N, int K, int P, const void *x, bool x_bf16, int batch,
                        int ldx, float *y, int ldy, uint32_t *fault_word, uint64_t timeout_ns) {
    if (P != 2 && P != 3) return cudaErrorInvalidValue;
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    const int nchunks = ceil_div(Wr, 32);
    // Rows: as evenly as possible over the SMs, one CTA each.
    const int rows_per_cta = ceil_div(N, std::min(ctx.num_sms, N));
    const int grid = ceil_div(N, rows_per_cta);
    const bool f32x = !x_bf16;
    auto bytes_for = [&](int rows) -> uint32_t {
        if (P == 2) return f32x ? smem_layout<2, 2>(rows, Wr, nchunks).total : smem_layout<1, 2>(rows, Wr, nchunks).total;
        return f32x ? smem_layout<2, 3>(rows, Wr, nchunks).total : smem_layout<1, 3>(rows, Wr, nchunks).total;
    };
    int pass_rows = ceil_div(rows_per_cta, kGroupRows) * kGroupRows;
    while (pass_rows > kGroupRows && bytes_for(pass_rows) > static_cast<uint32_t>(kSmemBudget))
        pass_rows -= kGroupRows;
    if (bytes_for(pass_rows) > static_cast<uint32_t>(kSmemBudget)) return cudaErrorInvalidConfiguration;
    // Warps: as few as give every warp the same number of work items (8 rows x 32 groups)
    // within the thread budget, but enough that the z stage has at most two tasks per thread
    // (up to 16 warps).
    const int items = ceil_div(pass_rows, kGroupRows) * nchunks;
    const int max_warps = max_threads(f32x, P) / 32;
    const int per_warp = ceil_div(items, max_warps);
    const int zwarps = std::min(16, ceil_div(4 * Wr, 64));
    int threads = 32 * std::min(max_warps, std::max(ceil_div(items, per_warp), zwarps));

    GemvArgs p;
    p.packed = packed;
    p.a = a;
    p.b = b;
    p.x = x;
    p.y = y;
    p.fault = fault_word;
    p.timeout_ns = timeout_ns;
    p.N = N;
    p.K = K;
    p.Wr = Wr;
    p.batch = batch;
    p.ldx = ldx;
    p.ldy = ldy;
    p.rows_per_cta = rows_per_cta;
    p.pass_rows = pass_rows;
    p.nchunks = nchunks;
    const size_t xel = x_bf16 ? 2 : 4;
    p.vec_x = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && ((static_cast<size_t>(ldx) * xel) % 16 == 0);
    p.vec_b = (reinterpret_cast<uintptr_t>(b) % 16 == 0) && (K % 4 == 0);

    uint32_t smem = bytes_for(pass_rows);
    void (*kern)(GemvArgs) = P == 2 ? (f32x ? gemv_kernel<true, 2> : gemv_kernel<false, 2>)
                                    : (f32x ? gemv_kernel<true, 3> : gemv_kernel<false, 3>);
    int variant = (P == 3 ? 2 : 0) + (f32x ? 1 : 0);
    // Batch >= 2: the kernel that serves kNB batch rows per z stage and rows sweep, when the
    // CTA's rows and the kNB rows' z tables fit in shared memory together (one pass).
    if (batch >= 2) {
        const int full_rows = ceil_div(rows_per_cta, kGroupRows) * kGroupRows;
        auto multi_bytes = [&](int nb) -> uint32_t {
            if (P == 2) return f32x ? smem_layout_multi<2, 2>(full_rows, Wr, nchunks, nb).total
                                    : smem_layout_multi<1, 2>(full_rows, Wr, nchunks, nb).total;
            return f32x ? smem_layout_multi<2, 3>(full_rows, Wr, nchunks, nb).total
                        : smem_layout_multi<1, 3>(full_rows, Wr, nchunks, nb).total;
        };
        int nb = (!f32x && batch % 4 == 0) ? 4 : 2;
        if (nb == 4 && multi_bytes(4) > static_cast<uint32_t>(kSmemBudget)) nb = 2;
        if (multi_bytes(nb) <= static_cast<uint32_t>(kSmemBudget)) {
            pass_rows = full_rows;
            smem = multi_bytes(nb);
            const int mitems = ceil_div(pass_rows, kGroupRows) * nchunks;
            const int mmax = kMultiThreads / 32;
            const int mper = ceil_div(mitems, mmax);
            const int mz = std::min(mmax, ceil_div(4 * Wr, 64));
            threads = 32 * std::min(mmax, std::max(ceil_div(mitems, mper), mz));
            if (P == 2)
                kern = f32x ? gemv_multi_kernel<true, 2, 2>
                            : (nb == 4 ? gemv_multi_kernel<false, 2, 4> : gemv_multi_kernel<false, 2, 2>);
            else
                kern = f32x ? gemv_multi_kernel<true, 3, 2>
                            : (nb == 4 ? gemv_multi_kernel<false, 3, 4> : gemv_multi_kernel<false, 3, 2>);
            variant = 4 + (P == 3 ? 3 : 0) + (f32x ? 0 : (nb == 4 ? 2 : 1));
        }
    }
    p.pass_rows = pass_rows;
    // Opt in to the largest dynamic shared memory once per kernel and device.
    static ContextFlags opted[10];
    if (cudaError_t e = ensure_smem_optin(ctx, kern, kSmemBudget, opted[variant]); e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace rabit
