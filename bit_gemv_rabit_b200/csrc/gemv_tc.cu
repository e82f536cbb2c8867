// gemv_tc.cu -- decode path of the residual-binary linear layer (batch 1..16) on tcgen05.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.1 "Multi-bit Approximation via Stacking", executed per path as Appendix E.1
// "Compute Pipeline" describes (paths in parallel, signs applied without multiplies,
// output scale applied last):
//     y[beta][n] = sum_k a_k[n] * t_k[beta][n],   t_k[beta][n] = sum_j S_k[n][j] z_k[beta][j],
//     z_k[beta][j] = b_k[j] * x[beta][j].
//
// The signs enter the tensor core as the bits themselves.  With bit = 1 for S = -1,
//     t = Z - 2 * sum_j bit[n][j] * zq[j],   Z = sum_j zq[j],
// where zq = rint(z * 2^e) with one power-of-two scale per (segment, batch row, path).  The
// sum over bits is a u8 x s8 -> s32 product on the tensor cores (tcgen05.mma kind::i8), so it
// is exact; the only rounding is the quantisation of z (16 bits for bf16 x, 24 bits for fp32
// x) and the final conversion to fp32.
//
// Operand A (tensor memory, one lane per weight row): a packed word w of 32 columns gives 8
// registers A_q = w & (0x01010101 << q), q = 0..7, whose byte i holds 2^q * bit(32g + 8i + q)
// (g the group).  One logic op per 4 weight bits, no shifts.  Register q of group g becomes
// tensor-memory column 8g + q, so contraction index 32g + 4q + i <-> column 32g + 8i + q.
// Operand B (shared memory, K-major, 128-byte swizzle): row 4*beta + s holds byte slice s of
// v = zq << (7 - q) at the same contraction index.  Every product is then 2^7 * bit * zq,
// v < 2^31, and the slices recombine exactly: sum_s 2^(8s) acc_s = 128 * sum bit * zq.
// Byte slices are balanced (each in [-128, 127]): v = sum_s 2^(8s) s8(v_s) with
// v_0 = v, v_{s+1} = (v_s + 128) >> 8.
//
// Work split: a unit is 128 rows x 128 columns.  The units of all row tiles, taken row
// tile by row tile, are dealt as equal contiguous ranges to one persistent CTA per SM
// ("stream-K"), so every shape balances to within one unit.  A CTA walks its range in
// segments (a run of chunks of one row tile that share one z scale).  A row tile that one
// CTA covers completely is written straight to y; partial tiles leave their fp32 partial
// sums in the workspace, and the last contributor to arrive (a ticket per tile) adds them
// in contributor order, which is the column order, so results are deterministic.
//
// Roles (192 threads):
//   warp 0      TMA producer: one 128-row x 128-column box of packed words per chunk into an
//               8-stage ring.  Before the programmatic-launch wait it only prefetches its
//               boxes to L2 (no data reaches the SM, so nothing an earlier kernel still writes
//               can be observed).
//   warp 1      tensor memory allocation; one lane issues P x 4 MMAs (M = 128, N = nm,
//               K = 32) per chunk.
//   warps 2..5  thread t owns tensor-memory lane t = row t of the tile: per segment the z
//               stage (scales, slices, the B tables), per chunk the expansion into A, per
//               segment the epilogue (tcgen05.ld, exact recombination, scales, a_k), per row
//               tile the output or the partial and the ticket.
// Every wait on another agent is bounded; an expired wait records a fault bit and the CTA
// drains what it has in flight and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "rabit.h"
#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kRows = 128;          // rows per tile: MMA M, tensor-memory lanes
constexpr int kChunkCols = 128;     // columns per unit
constexpr int kThreads = 192;
constexpr int kExpandThreads = 128;
constexpr int kAStages = 2;         // A stages in tensor memory
constexpr int kBBudget = 64 * 1024; // shared memory for one segment's B tables
constexpr int kMaxSegChunks = 16;
constexpr int kMaxBatch = 16;
constexpr int kPrefetchChunks = 32; // boxes a CTA prefetches to L2 before the launch wait

template <int kP> struct Geometry {
    static constexpr int kGroupWords = kP == 2 ? 2 : 4;             // words per 32-column group
    static constexpr int kChunkWords = 4 * kGroupWords;             // words per row per chunk
    static constexpr int kStageBytes = kRows * kChunkWords * 4;     // 4 KiB (P=2), 8 KiB (P=3)
    static constexpr int kWStages = kP == 2 ? 8 : 6;
};

struct TcArgs {
    const float *a;        // [P][N]
    const float *b;        // [P][K]
    const void *x;         // [batch][ldx]
    float *y;              // [batch][ldy]
    float *partial;        // workspace: [grid][2][batch][128] (fixed-size region at offset 0)
    int *tickets;          // workspace: [tiles], after the partial sums
    uint32_t *fault;
    uint64_t timeout_ns;
    long long units;       // tiles * chunks
    int N, K, batch, ldx, ldy;
    int tiles, chunks;     // row tiles, 128-column chunks per row
    int nm;                // MMA N: B rows per path, 16 .. 64
    int seg_chunks;        // chunks per segment at most
    int debug;             // bit 1: the producer withholds the first copy (fault-injection test)
};

struct Ctl {
    uint64_t w_full[8];
    uint64_t w_empty[8];
    uint64_t a_full[kAStages];
    uint64_t a_empty[kAStages];
    uint64_t acc_full;
    uint64_t drain;
    uint64_t group;                    // barrier of the 4 expansion warps (bounded, unlike bar.sync)
    uint32_t tmem_base;
    int abort;
    int last;                          // fix-up: this CTA arrived last for the tile
    // per segment, double-buffered by segment parity
    uint32_t zmax[2][kMaxBatch][3];    // max |x b_k| (float bits) per (batch row, path)
    long long zsum[2][kMaxBatch][3];   // sum of zq per (batch row, path)
};

// Scale exponent e of a segment: |zq| = |rint(z 2^e)| <= 2^(top+1) for every z of the segment.
__device__ __forceinline__ int scale_exponent(uint32_t zmax_bits, int top) {
    const float mx = __uint_as_float(zmax_bits);
    if (!(mx > 0.0f)) return 0;
    const int E = static_cast<int>((zmax_bits >> 23) & 0xFFu) - 127;
    return min(126, max(-126, top - E));   // 2^-e stays a normal float
}

// Barrier of the 4 expansion warps on an mbarrier of count 4, with a bounded wait: a warp that
// left after an expired wait makes the others time out too instead of hanging (bar.sync has no
// bound).  `phase` is the caller's running parity.  Returns false once the CTA is aborting.
__device__ __forceinline__ bool group_sync(Ctl *ctl, uint32_t &phase, int lane, const TcArgs &p) {
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ctl->group));
    const bool ok = mbar_wait_bounded(smem_u32(&ctl->group), phase, &ctl->abort, p.timeout_ns, p.fault,
                                      FAULT_GEMV_WAIT_MMA);
    phase ^= 1u;
    return __all_sync(0xffffffffu, ok);
}

__host__ __device__ inline int nm_for(int batch) {
    const int rows = 4 * batch;
    return rows <= 16 ? 16 : ((rows + 15) / 16) * 16;
}

// Units of CTA i: [U*i/G, U*(i+1)/G).
__device__ __forceinline__ long long range_begin(long long U, int G, int i) { return U * i / G; }
// The CTA whose range holds unit u.
__device__ __forceinline__ int unit_owner(long long U, int G, long long u) {
    return static_cast<int>(((u + 1) * G - 1) / U);
}

// Byte offset of (row r, contraction byte k) in a K-major operand of 128-byte rows stored in
// 128-byte-swizzled atoms of 8 rows (the layout the descriptor's SWIZZLE_128B names).
__device__ __forceinline__ uint32_t sw128_offset(int r, int k) {
    return static_cast<uint32_t>((r >> 3) * 1024 + (r & 7) * 128 + ((((k >> 4) ^ (r & 7)) & 7) << 4) + (k & 15));
}

template <bool kF32X>
__device__ __forceinline__ float load_x(const TcArgs &p, int beta, int j) {
    if (j >= p.K) return 0.0f;
    const int64_t idx = static_cast<int64_t>(beta) * p.ldx + j;
    if constexpr (kF32X) {
        return __ldg(reinterpret_cast<const float *>(p.x) + idx);
    } else {
        return __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short *>(p.x) + idx)) << 16);
    }
}
__device__ __forceinline__ float load_b(const TcArgs &p, int k, int j) {
    return j < p.K ? __ldg(p.b + static_cast<int64_t>(k) * p.K + j) : 0.0f;
}

// The segment's z stage, run by the 128 expansion threads (te = 0..127): per (batch row,
// path) the scale and the sum of zq, and the B tables of chunks [0, nch) of the segment
// starting at column j0 of the row.  Statistics go to buffer `buf` (zeroed beforehand); the
// other buffer is zeroed here for the next segment.  Returns false if the CTA is aborting.
template <bool kF32X, int kP>
__device__ bool z_stage(const TcArgs &p, Ctl *ctl, uint8_t *bsm, int j0, int nch, int te, int buf,
                        uint32_t &gphase) {
    constexpr int kSlices = kF32X ? 4 : 3;
    constexpr int kTop = kF32X ? 22 : 14;       // |zq| <= 2^(kTop+1): 16 or 24 bits with sign
    const int lane = te & 31;
    // ---- pass 1: max |x b_k| over the segment's columns
    const int ncols = nch * kChunkCols;
    for (int beta = 0; beta < p.batch; ++beta) {
        float m[kP];
#pragma unroll
        for (int k = 0; k < kP; ++k) m[k] = 0.0f;
        for (int c = te; c < ncols; c += kExpandThreads) {
            const float xv = load_x<kF32X>(p, beta, j0 + c);
#pragma unroll
            for (int k = 0; k < kP; ++k) m[k] = fmaxf(m[k], fabsf(xv * load_b(p, k, j0 + c)));
        }
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            const uint32_t r = __reduce_max_sync(0xffffffffu, __float_as_uint(m[k]));
            if (lane == 0) atomicMax(&ctl->zmax[buf][beta][k], r);
        }
    }
    if (!group_sync(ctl, gphase, lane, p)) return false;
    for (int i = te; i < kMaxBatch * 3; i += kExpandThreads) {
        (&ctl->zmax[buf ^ 1][0][0])[i] = 0u;
        (&ctl->zsum[buf ^ 1][0][0])[i] = 0;
    }
    // ---- pass 2: tuples (chunk r, group g, bit position q) -> one 32-bit B word per slice
    const int ntuples = nch * 32;               // a multiple of 32: whole warps take part
    for (int tu = te; tu < ntuples; tu += kExpandThreads) {
        const int r = tu >> 5, g = (tu >> 3) & 3, q = tu & 7;
        const int jb = j0 + r * kChunkCols + 32 * g + q;       // column of byte i is jb + 8i
        const int kb = 32 * g + 4 * q;                          // contraction byte of byte 0
        const int shift = 1 << (7 - q);
        float bv[kP][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int k = 0; k < kP; ++k) bv[k][i] = load_b(p, k, jb + 8 * i);
        for (int beta = 0; beta < p.batch; ++beta) {
            float xv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = load_x<kF32X>(p, beta, jb + 8 * i);
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                const int e = scale_exponent(ctl->zmax[buf][beta][k], kTop);
                const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
                uint32_t word[kSlices];
#pragma unroll
                for (int s = 0; s < kSlices; ++s) word[s] = 0u;
                int zs = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int zq = __float2int_rn(xv[i] * bv[k][i] * sc);
                    zs += zq;
                    int v = zq * shift;
#pragma unroll
                    for (int s = 0; s < kSlices; ++s) {
                        word[s] |= (static_cast<uint32_t>(v) & 0xFFu) << (8 * i);
                        v = (v + 128) >> 8;
                    }
                }
                const int zw = __reduce_add_sync(0xffffffffu, zs);
                if (lane == 0)
                    atomicAdd(reinterpret_cast<unsigned long long *>(&ctl->zsum[buf][beta][k]),
                              static_cast<unsigned long long>(static_cast<long long>(zw)));
                uint8_t *blk = bsm + static_cast<size_t>(r * kP + k) * p.nm * 128;
#pragma unroll
                for (int s = 0; s < kSlices; ++s)
                    *reinterpret_cast<uint32_t *>(blk + sw128_offset(4 * beta + s, kb)) = word[s];
            }
        }
    }
    fence_proxy_async_shared();                 // B tables -> tensor core (async proxy)
    return group_sync(ctl, gphase, lane, p);    // zsum complete for the epilogue
}

template <bool kF32X, int kP>
__global__ void __launch_bounds__(kThreads, 1)
gemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const TcArgs p) {
    using Geo = Geometry<kP>;
    constexpr int kWStages = Geo::kWStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *wring = smem;                                          // kWStages x stage
    uint8_t *bsm = smem + kWStages * Geo::kStageBytes;              // B tables (kBBudget)
    Ctl *ctl = reinterpret_cast<Ctl *>(bsm + kBBudget);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const long long U = p.units;
    const long long u0 = range_begin(U, G, cta), u1 = range_begin(U, G, cta + 1);
    volatile int *abort_flag = &ctl->abort;
    // TMEM columns: accumulators of path k at [k*nm, (k+1)*nm); A stage s, path k at
    // a_col0 + (s*kP + k)*32.
    const uint32_t a_col0 = static_cast<uint32_t>(kP * p.nm);
    const uint32_t tmem_cols = (a_col0 + kAStages * kP * 32) <= 256 ? 256u : 512u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWStages; ++s) {
            mbar_init(smem_u32(&ctl->w_full[s]), 1);
            mbar_init(smem_u32(&ctl->w_empty[s]), 4);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(smem_u32(&ctl->a_full[s]), 4);
            mbar_init(smem_u32(&ctl->a_empty[s]), 1);
        }
        mbar_init(smem_u32(&ctl->acc_full), 1);
        mbar_init(smem_u32(&ctl->drain), 1);
        mbar_init(smem_u32(&ctl->group), 4);
        ctl->abort = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tmap_w);
        // L2 prefetch of the first boxes of this CTA's range (weights only)
        int n = 0;
        for (long long u = u0; u < u1 && n < kPrefetchChunks; ++u, ++n)
            tma_prefetch_2d(&tmap_w, static_cast<int>(u % p.chunks) * Geo::kChunkWords,
                            static_cast<int>(u / p.chunks) * kRows);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl->tmem_base), tmem_cols);
        tmem_relinquish();
    }
    // B rows this call does not use stay zero for the whole kernel.
    for (int i = threadIdx.x; i < kBBudget / 16; i += kThreads)
        reinterpret_cast<uint4 *>(bsm)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < 2 * kMaxBatch * 3; i += kThreads) {
        (&ctl->zmax[0][0][0])[i] = 0u;
        (&ctl->zsum[0][0][0])[i] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    // The next kernel on the stream may start its own prologue (and its L2 prefetches) now;
    // its reads of our outputs wait for this grid's completion in its griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool issued[8] = {};
            uint32_t last_parity[8] = {};
            bool ok = true;
            uint32_t it = 0;
            for (long long u = u0; u < u1; ++u, ++it) {
                const uint32_t s = it % kWStages, ph = (it / kWStages) & 1u;
                if (!mbar_wait_bounded(smem_u32(&ctl->w_empty[s]), ph ^ 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMV_WAIT_COPY)) {
                    ok = false;
                    break;
                }
                if ((p.debug & 2) && it == 0) continue;   // fault injection: this copy never comes
                const uint32_t bar = smem_u32(&ctl->w_full[s]);
                mbar_arrive_expect_tx(bar, Geo::kStageBytes);
                tma_load_2d(smem_u32(wring + s * Geo::kStageBytes), &tmap_w, bar,
                            static_cast<int>(u % p.chunks) * Geo::kChunkWords,
                            static_cast<int>(u / p.chunks) * kRows);
                issued[s] = true;
                last_parity[s] = ph;
            }
            // Every issued copy lands before the CTA can exit, also when the consumers stopped
            // early on an expired wait.  These are the latest phases of their stages, already
            // complete in normal operation.
            (void)ok;
            int drain_abort = 0;
            for (int s = 0; s < kWStages; ++s)
                if (issued[s])
                    mbar_wait_bounded(smem_u32(&ctl->w_full[s]), last_parity[s], &drain_abort, p.timeout_ns,
                                      p.fault, FAULT_GEMM_DRAIN);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_u8s8_s32(kRows, p.nm);
            const uint32_t b_base = smem_u32(bsm);
            bool ok = true, any = false;
            uint32_t it = 0;
            for (long long u = u0; ok && u < u1;) {
                const long long tile_end = std::min<long long>(u1, (u / p.chunks + 1) * p.chunks);
                for (long long su = u; ok && su < tile_end; su += p.seg_chunks) {
                    const int nch = static_cast<int>(std::min<long long>(tile_end - su, p.seg_chunks));
                    for (int r = 0; r < nch; ++r, ++it) {
                        const uint32_t s = it % kAStages, ph = (it / kAStages) & 1u;
                        if (!mbar_wait_bounded(smem_u32(&ctl->a_full[s]), ph, abort_flag, p.timeout_ns,
                                               p.fault, FAULT_GEMV_WAIT_MMA)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < kP; ++k) {
                            const uint32_t bblk = b_base + static_cast<uint32_t>((r * kP + k) * p.nm * 128);
                            const uint32_t acol = a_col0 + static_cast<uint32_t>((s * kP + k) * 32);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                tc_mma_i8_ts(tmem + static_cast<uint32_t>(k * p.nm), tmem + acol + 8 * kk,
                                             smem_desc_kmajor_sw128(bblk + 32 * kk), idesc,
                                             (r | kk) != 0 ? 1u : 0u);
                        }
                        any = true;
                        tc_commit(smem_u32(&ctl->a_empty[s]));     // frees A stage s when done
                    }
                    if (ok) tc_commit(smem_u32(&ctl->acc_full));
                }
                u = tile_end;
            }
            if (!ok && any) {
                tc_commit(smem_u32(&ctl->drain));
                int drain_abort = 0;
                mbar_wait_bounded(smem_u32(&ctl->drain), 0, &drain_abort, p.timeout_ns, p.fault,
                                  FAULT_GEMM_DRAIN);
            }
        }
    } else {
        // ------------------------------------------------------------ z stage, expansion, epilogue
        const int te = threadIdx.x - 64;             // 0..127 = tensor-memory lane = tile row
        const int q4 = warp & 3;                     // lane quarter this warp may access
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const int row = q4 * 32 + lane;
        bool ok = true;
        uint32_t it = 0, seg = 0, gphase = 0;
        for (long long u = u0; u < u1;) {
            const int t = static_cast<int>(u / p.chunks);
            const long long tile_begin = static_cast<long long>(t) * p.chunks;
            const long long tile_end = std::min<long long>(u1, tile_begin + p.chunks);
            const int n = t * kRows + row;
            float ypart[kMaxBatch];
#pragma unroll
            for (int i = 0; i < kMaxBatch; ++i) ypart[i] = 0.0f;
            float arow[kP];
#pragma unroll
            for (int k = 0; k < kP; ++k) arow[k] = n < p.N ? __ldg(p.a + static_cast<int64_t>(k) * p.N + n) : 0.0f;

            for (long long su = u; su < tile_end; su += p.seg_chunks, ++seg) {
                const int nch = static_cast<int>(std::min<long long>(tile_end - su, p.seg_chunks));
                const int j0 = static_cast<int>(su - tile_begin) * kChunkCols;
                const int buf = static_cast<int>(seg & 1u);
                if (!z_stage<kF32X, kP>(p, ctl, bsm, j0, nch, te, buf, gphase)) { ok = false; break; }
                for (int r = 0; r < nch && ok; ++r, ++it) {
                    const uint32_t ws = it % kWStages, wph = (it / kWStages) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&ctl->w_full[ws]), wph, abort_flag, p.timeout_ns,
                                           p.fault, FAULT_GEMV_WAIT_COPY))
                        ok = false;
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    const uint4 *src = reinterpret_cast<const uint4 *>(wring + ws * Geo::kStageBytes +
                                                                        row * Geo::kChunkWords * 4);
                    uint32_t words[kP][4];
                    if constexpr (kP == 2) {
                        const uint4 g0 = src[0], g1 = src[1];
                        words[0][0] = g0.x; words[1][0] = g0.y; words[0][1] = g0.z; words[1][1] = g0.w;
                        words[0][2] = g1.x; words[1][2] = g1.y; words[0][3] = g1.z; words[1][3] = g1.w;
                    } else {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const uint4 v = src[g];
                            words[0][g] = v.x; words[1][g] = v.y; words[2][g] = v.z;
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&ctl->w_empty[ws]));
                    const uint32_t as = it % kAStages, aph = (it / kAStages) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&ctl->a_empty[as]), aph ^ 1u, abort_flag, p.timeout_ns,
                                           p.fault, FAULT_GEMV_WAIT_COPY))
                        ok = false;
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < kP; ++k) {
                        uint32_t v[32];
#pragma unroll
                        for (int g = 0; g < 4; ++g)
#pragma unroll
                            for (int q = 0; q < 8; ++q) v[8 * g + q] = words[k][g] & (0x01010101u << q);
                        tmem_st_32x32b_x32(tmem + lane_addr + a_col0 + static_cast<uint32_t>((as * kP + k) * 32), v);
                    }
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&ctl->a_full[as]));
                }
                if (!ok) break;
                // ---- epilogue of the segment
                if (!mbar_wait_bounded(smem_u32(&ctl->acc_full), seg & 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMV_WAIT_MMA))
                    ok = false;
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < kP; ++k) {
#pragma unroll
                    for (int c = 0; c < kMaxBatch / 4; ++c) {
                        if (16 * c >= 4 * p.batch) break;
                        uint32_t acc[16];
                        tmem_ld_32x32b_x16(tmem + lane_addr + static_cast<uint32_t>(k * p.nm + 16 * c), acc);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int beta = 4 * c + i;
                            if (beta < p.batch) {
                                long long comb = static_cast<long long>(static_cast<int>(acc[4 * i])) +
                                                 (static_cast<long long>(static_cast<int>(acc[4 * i + 1])) << 8) +
                                                 (static_cast<long long>(static_cast<int>(acc[4 * i + 2])) << 16) +
                                                 (static_cast<long long>(static_cast<int>(acc[4 * i + 3])) << 24);
                                const long long tk = ctl->zsum[buf][beta][k] - 2 * (comb >> 7);
                                const int e = scale_exponent(ctl->zmax[buf][beta][k], kF32X ? 22 : 14);
                                const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
                                ypart[beta] += arow[k] * (static_cast<float>(tk) * inv);
                            }
                        }
                    }
                }
                tc_fence_before();
            }
            if (!ok) break;
            // ---- row tile done: write y, or the partial and the ticket
            const int first = unit_owner(U, G, tile_begin);
            const int lastc = unit_owner(U, G, tile_begin + p.chunks - 1);
            if (first == lastc) {
                if (n < p.N) {
#pragma unroll
                    for (int beta = 0; beta < kMaxBatch; ++beta)
                        if (beta < p.batch) p.y[static_cast<int64_t>(beta) * p.ldy + n] = ypart[beta];
                }
            } else {
                const int side = (t == static_cast<int>(u0 / p.chunks)) ? 0 : 1;
                float *slot = p.partial + (static_cast<int64_t>(cta) * 2 + side) * p.batch * kRows;
#pragma unroll
                for (int beta = 0; beta < kMaxBatch; ++beta)
                    if (beta < p.batch) slot[beta * kRows + row] = ypart[beta];
                __threadfence();
                if (!group_sync(ctl, gphase, lane, p)) { ok = false; break; }
                if (te == 0) {
                    const int old = atomicAdd(&p.tickets[t], 1);
                    ctl->last = (old == lastc - first) ? 1 : 0;
                }
                if (!group_sync(ctl, gphase, lane, p)) { ok = false; break; }
                if (ctl->last) {
                    __threadfence();
                    for (int beta = 0; beta < p.batch; ++beta) {
                        float sum = 0.0f;
                        for (int i = first; i <= lastc; ++i) {
                            const int ti = static_cast<int>(range_begin(U, G, i) / p.chunks);
                            const int si = (t == ti) ? 0 : 1;
                            sum += __ldcg(p.partial + ((static_cast<int64_t>(i) * 2 + si) * p.batch + beta) * kRows + row);
                        }
                        if (n < p.N) p.y[static_cast<int64_t>(beta) * p.ldy + n] = sum;
                    }
                    if (te == 0) p.tickets[t] = 0;
                }
            }
            u = tile_end;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols);
    }
}

}  // namespace

// Workspace: the partial sums first, in a region of fixed size (the largest grid and batch),
// then one counter per row tile.  Counters a call does not use are never written, so a
// workspace zero-filled once serves every later call, whatever its shape.
constexpr size_t kPartialBytes = static_cast<size_t>(kGemvMaxGrid) * 2 * kMaxBatch * kRows * sizeof(float);

size_t gemv_workspace_bytes(int N, int K, int P, int batch) {
    (void)K;
    (void)P;
    (void)batch;
    const size_t tiles = (static_cast<size_t>(N) + kRows - 1) / kRows;
    return kPartialBytes + ((tiles * sizeof(int) + 15) / 16) * 16;
}

cudaError_t launch_gemv_tc(const LaunchCtx &ctx, const uint32_t *packed, const float *a, const float *b,
                           int N, int K, int P, const void *x, bool x_bf16, int batch, int ldx, float *y,
                           int ldy, void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug) {
    if (P != 2 && P != 3) return cudaErrorInvalidValue;
    const int Kp = static_cast<int>(padded_cols(K));
    const int G = P == 2 ? 2 : 4;
    const int words_per_row = Kp / 32 * G;

    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tmap;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(words_per_row), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(words_per_row) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(4 * G), static_cast<cuuint32_t>(kRows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(packed), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    TcArgs args;
    args.a = a;
    args.b = b;
    args.x = x;
    args.y = y;
    args.fault = fault_word;
    args.timeout_ns = timeout_ns;
    args.N = N;
    args.K = K;
    args.batch = batch;
    args.ldx = ldx;
    args.ldy = ldy;
    args.tiles = (N + kRows - 1) / kRows;
    args.chunks = Kp / kChunkCols;
    args.units = static_cast<long long>(args.tiles) * args.chunks;
    args.nm = nm_for(batch);
    args.seg_chunks = std::min(kMaxSegChunks, kBBudget / (P * args.nm * 128));
    args.debug = debug;
    const int grid = static_cast<int>(std::min<long long>(args.units, std::min(ctx.num_sms, kGemvMaxGrid)));
    args.partial = static_cast<float *>(workspace);
    args.tickets = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + kPartialBytes);

    const int stage_bytes = P == 2 ? Geometry<2>::kStageBytes * Geometry<2>::kWStages
                                   : Geometry<3>::kStageBytes * Geometry<3>::kWStages;
    const int smem = stage_bytes + kBBudget + static_cast<int>(sizeof(Ctl)) + 1024;
    void (*kern)(CUtensorMap, TcArgs);
    if (P == 2) kern = x_bf16 ? gemv_tc_kernel<false, 2> : gemv_tc_kernel<true, 2>;
    else kern = x_bf16 ? gemv_tc_kernel<false, 3> : gemv_tc_kernel<true, 3>;
    static ContextFlags opted[4];
    if (cudaError_t e = ensure_smem_optin(ctx, kern, smem, opted[(P - 2) * 2 + (x_bf16 ? 0 : 1)]); e != cudaSuccess)
        return e;

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, args);
}

}  // namespace rabit
