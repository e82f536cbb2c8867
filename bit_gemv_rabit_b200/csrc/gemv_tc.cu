// gemv_tc.cu -- decode path of the residual-binary linear layer (batch 1..16) on tcgen05.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.1 "Multi-bit Approximation via Stacking", executed per path as Appendix E.1
// "Compute Pipeline" describes (paths in parallel, signs applied without multiplies,
// output scale applied last):
//     y[beta][n] = sum_k a_k[n] * t_k[beta][n],   t_k[beta][n] = sum_j S_k[n][j] z_k[beta][j],
//     z_k[beta][j] = b_k[j] * x[beta][j].
//
// Arithmetic.  z is quantised per segment (a run of at most 8 chunks of 128 columns of one
// row tile) and batch row and path: zq = rint(z * 2^e), |zq| < 2^15 for bf16 x (2^23 for fp32
// x), one power-of-two scale.  The sign sum t = sum_j S_j zq_j is then computed exactly on the
// tensor cores with packed 4-bit operands (tcgen05.mma kind::mxf4, every block scale 1.0):
//   - A (tensor memory, lane = weight row): each sign as the e2m1 value +1 or -1.  From a
//     packed word w, register r = 0..3 is ((w << (3 - r)) & 0x88888888) | 0x22222222: its
//     nibble i is the sign of column 4i + r of the word (bit 3 of an e2m1 nibble is its sign).
//     Register r of group g is tensor-memory column 4g + r, so contraction index
//     32g + 8r + i holds column 32g + 4i + r.
//   - B (shared memory, K-major, 128-byte swizzle): v = zq + 2^15 (2^23) is written in base 4,
//     v = sum_s 4^s u_s with u_s in {0,1,2,3}, and row 8 beta + s (12 beta + s) holds u_s as
//     the e2m1 code u_s itself, i.e. the value u_s / 2.  One more row holds 1.0 everywhere.
//   Each accumulator D_s = sum_j S_j u_s,j / 2 and D_one = sum_j S_j are small integers or
//   halves, exact in fp32, and t = sum_s 4^s (2 D_s) - 2^15 D_one (2^23 for fp32) exactly.
// The only rounding is the quantisation of z and the final conversion of t to fp32.
//
// Work split: a unit is 128 rows x 128 columns.  The units of all row tiles, taken row
// tile by row tile, are dealt as equal contiguous ranges to one persistent CTA per SM
// ("stream-K"), so every shape balances to within one unit.  A row tile that one CTA covers
// completely is written straight to y; partial tiles leave fp32 partial sums in the
// workspace, and the last contributor to arrive (a counter per tile) adds them in
// contributor order, which is the column order, so results are deterministic.
//
// Roles (224 threads):
//   warp 0      TMA producer: one 128-row x 128-column box of packed words per chunk into an
//               8-stage ring.  Before the programmatic-launch wait it only prefetches its
//               boxes to L2 (no data reaches the SM, so nothing an earlier kernel still writes
//               can be observed).
//   warp 1      tensor-memory allocation; one lane issues P x 2 MMAs (M = 128, N = nm, K = 64)
//               per chunk.
//   warps 2..5  thread t owns tensor-memory lane t = row t of the tile: per segment the z
//               stage (scales, digits, the B tables), per chunk the expansion of the signs into
//               A, per segment the epilogue; per row tile the output or the partial.
//   warp 6      stager: x, b and a of each segment into a double-buffered shared-memory stage
//               with cp.async, so the z stage reads shared memory only.
// Every wait on another agent is bounded; an expired wait records a fault bit, and the CTA
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
constexpr int kThreads = 224;
constexpr int kExpandThreads = 128;
constexpr int kMaxBatch = 16;
constexpr int kMaxSegChunks = 8;
constexpr int kBCap = 32 * 1024;    // shared memory the B tables of a segment may take
constexpr int kSfCols = 32;         // tensor-memory columns holding the (constant) scale factors
constexpr int kPrefetchChunks = 32; // boxes a CTA prefetches to L2 before the launch wait
constexpr int kMaxWStages = 8;

template <int kP> struct Geometry {
    static constexpr int kGroupWords = kP == 2 ? 2 : 4;             // words per 32-column group
    static constexpr int kChunkWords = 4 * kGroupWords;             // words per row per chunk
    static constexpr int kStageBytes = kRows * kChunkWords * 4;     // 4 KiB (P=2), 8 KiB (P=3)
    static constexpr int kWStages = kP == 2 ? 8 : 4;
};

// Digits per batch row: 8 base-4 digits for 16-bit v (bf16 x), 12 for 24-bit v (fp32 x).
template <bool kF32X> struct Digits {
    static constexpr int kD = kF32X ? 12 : 8;
    static constexpr int kOffsetLog2 = kF32X ? 23 : 15;           // v = zq + 2^offset
    static constexpr int kTop = kF32X ? 22 : 14;                  // first guess of the scale exponent
    static constexpr float kZqLimit = kF32X ? 8388607.0f : 32767.0f;
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
    int nm;                // MMA N: digit rows of all batch rows + the ones row, rounded to 8
    int acc_stride;        // tensor-memory columns per path's accumulator (nm rounded to 16)
    int ones_row;
    int seg_chunks;        // chunks per segment at most (even)
    int a_stages;          // A stages in tensor memory (2 or 4)
    uint32_t tmem_cols;
    // shared-memory layout (bytes from the 1024-aligned base)
    int off_b, off_stage, stage_bytes, stage_off_x, stage_off_b, stage_off_a, xrow, brow;
    int x_vec, b_vec;      // rows of x / b start 16-byte aligned (cp.async of 16 bytes)
    int x_pair;            // x rows start 4-byte aligned (cp.async of 4 bytes)
    int debug;             // bit 1: the producer withholds its first copy (fault-injection test)
};

struct Ctl {
    uint64_t w_full[kMaxWStages];
    uint64_t w_empty[kMaxWStages];
    uint64_t a_full[4];
    uint64_t a_empty[4];
    uint64_t acc_full;
    uint64_t x_full[2];
    uint64_t x_empty[2];
    uint64_t drain;
    uint64_t group;                    // barrier of the 4 expansion warps (bounded, unlike bar.sync)
    uint32_t tmem_base;
    int abort;
    int last;                          // fix-up: this CTA arrived last for the tile
    uint32_t zmax[2][kMaxBatch][3];    // max |x b_k| (float bits) per (batch row, path), by segment parity
};

__host__ __device__ inline int digits_for(bool f32x) { return f32x ? 12 : 8; }
__host__ __device__ inline int nm_for(int batch, bool f32x) { return ((digits_for(f32x) * batch + 1 + 7) / 8) * 8; }
// Padded position of column c in a staged row: 4 words after every 32 columns, so the z
// stage's strided reads (columns 32g + 4i + r of a chunk) hit 32 different banks.
__host__ __device__ inline int pad_f32(int c) { return c + 4 * (c >> 5); }
__host__ __device__ inline int pad_bf16(int c) { return c + 8 * (c >> 5); }

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

// Scale exponent of a segment: zq = rint(z 2^e) stays within +-limit for every z of the segment.
__device__ __forceinline__ int seg_exponent(uint32_t zmax_bits, int top, float limit) {
    const float mx = __uint_as_float(zmax_bits);
    if (!(mx > 0.0f)) return 0;
    const int E = static_cast<int>((zmax_bits >> 23) & 0xFFu) - 127;
    int e = min(126, max(-126, top - E));                 // 2^-e stays a normal float
    if (mx * __uint_as_float(static_cast<uint32_t>(e + 127) << 23) > limit) --e;
    return e;
}

// Instruction descriptor, kind::mxf4: packed e2m1 A and B (K-major), fp32 accumulator, e8m0
// block scales, K = 64.  Fields as in the kind::f16 descriptor; A and B format 1 = e2m1,
// bit 23 = scale format e8m0, scale-factor ids 0.
__host__ __device__ constexpr uint32_t idesc_mxf4_f32(int M, int N) {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
           (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void tc_mma_mxf4_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                               uint32_t sfa, uint32_t sfb, uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], [%1], %2, %3, [%5], [%6], p;\n\t}"
                 ::"r"(d), "r"(a), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb) : "memory");
}
__device__ __forceinline__ void tmem_st_x16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                   "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]) : "memory");
}
__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_ld_x1(uint32_t taddr, uint32_t &v) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// The 8 base-4 digits of a 16-bit value, digit s moved to bits 4s..4s+1.
__device__ __forceinline__ uint32_t spread16(uint32_t v) {
    v = prmt(v, 0u, 0x4140u);                       // byte 0 -> byte 0, byte 1 -> byte 2
    v = (v | (v << 4)) & 0x0F0F0F0Fu;
    v = (v | (v << 2)) & 0x33333333u;
    return v;
}

// Transpose of an 8 x 8 matrix of nibbles: afterwards nibble i of e[j] is what nibble j of
// e[i] was.  Three rounds swap the register-index bit with the nibble-index bit 2, 1, 0.
__device__ __forceinline__ void transpose8x8_nibbles(uint32_t (&e)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t a = e[i], b = e[i + 4];
        e[i] = prmt(a, b, 0x5410u);
        e[i + 4] = prmt(a, b, 0x7632u);
    }
#pragma unroll
    for (int h = 0; h < 8; h += 4)
#pragma unroll
        for (int i = h; i < h + 2; ++i) {
            const uint32_t a = e[i], b = e[i + 2];
            e[i] = prmt(a, b, 0x6240u);
            e[i + 2] = prmt(a, b, 0x7351u);
        }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const uint32_t a = e[i], b = e[i + 1];
        e[i] = (a & 0x0F0F0F0Fu) | ((b << 4) & 0xF0F0F0F0u);
        e[i + 1] = ((a >> 4) & 0x0F0F0F0Fu) | (b & 0xF0F0F0F0u);
    }
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

// Staged x value of batch row beta at segment column c (0 beyond K: the stager zero-fills).
template <bool kF32X>
__device__ __forceinline__ float staged_x(const uint8_t *xs, const TcArgs &p, int beta, int c) {
    if constexpr (kF32X) {
        return reinterpret_cast<const float *>(xs)[beta * p.xrow + pad_f32(c)];
    } else {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const unsigned short *>(xs)[beta * p.xrow + pad_bf16(c)]) << 16);
    }
}

// The segment's z stage, run by the 128 expansion threads (te = 0..127): the per (batch row,
// path) scale and the B tables of chunks [0, nch) of the segment, from the staged x and b.
// Writes zmax[buf] (zeroed beforehand) and zeroes zmax[buf ^ 1] for the next segment.
template <bool kF32X, int kP>
__device__ bool z_stage(const TcArgs &p, Ctl *ctl, uint8_t *bsm, const uint8_t *stage, int nch, int te, int buf,
                        uint32_t &gphase) {
    using Dg = Digits<kF32X>;
    constexpr int kD = Dg::kD;
    const int lane = te & 31;
    const uint8_t *xs = stage + p.stage_off_x;
    const float *bs = reinterpret_cast<const float *>(stage + p.stage_off_b);
    // ---- pass 1: max |x b_k| over the segment's columns
    const int ncols = nch * kChunkCols;
    for (int beta = 0; beta < p.batch; ++beta) {
        float m[kP];
#pragma unroll
        for (int k = 0; k < kP; ++k) m[k] = 0.0f;
        for (int c = te; c < ncols; c += kExpandThreads) {
            const float xv = staged_x<kF32X>(xs, p, beta, c);
#pragma unroll
            for (int k = 0; k < kP; ++k) m[k] = fmaxf(m[k], fabsf(xv * bs[k * p.brow + pad_f32(c)]));
        }
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            const uint32_t r = __reduce_max_sync(0xffffffffu, __float_as_uint(m[k]));
            if (lane == 0) atomicMax(&ctl->zmax[buf][beta][k], r);
        }
    }
    if (!group_sync(ctl, gphase, lane, p)) return false;
    for (int i = te; i < kMaxBatch * 3; i += kExpandThreads) (&ctl->zmax[buf ^ 1][0][0])[i] = 0u;
    // ---- pass 2: tuples (chunk r, group g, register q): 8 columns 32g + 4i + q of the chunk
    // give one 32-bit B word per digit row.
    const int ntuples = nch * 16;
    for (int tu = te; tu < ntuples; tu += kExpandThreads) {
        const int r = tu >> 4, g = (tu >> 2) & 3, q = tu & 3;
        const int cb = r * kChunkCols + 32 * g + q;             // segment column of nibble i is cb + 4i
        const int kbyte = 64 * (r & 1) + 16 * g + 4 * q;        // byte of the word in the pair row
        uint8_t *pair = bsm + static_cast<size_t>((r >> 1) * kP) * p.nm * 128;
        for (int beta = 0; beta < p.batch; ++beta) {
            float xv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) xv[i] = staged_x<kF32X>(xs, p, beta, cb + 4 * i);
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                const int e = seg_exponent(ctl->zmax[buf][beta][k], Dg::kTop, Dg::kZqLimit);
                const float sc = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
                uint32_t lo[8], hi[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float z = xv[i] * bs[k * p.brow + pad_f32(cb + 4 * i)];
                    const uint32_t v = static_cast<uint32_t>(__float2int_rn(z * sc) + (1 << Dg::kOffsetLog2));
                    lo[i] = spread16(v & 0xFFFFu);
                    if constexpr (kF32X) hi[i] = spread16(v >> 16);
                }
                transpose8x8_nibbles(lo);
                uint8_t *blk = pair + static_cast<size_t>(k) * p.nm * 128;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    *reinterpret_cast<uint32_t *>(blk + sw128_offset(kD * beta + s, kbyte)) = lo[s];
                if constexpr (kF32X) {
                    transpose8x8_nibbles(hi);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        *reinterpret_cast<uint32_t *>(blk + sw128_offset(kD * beta + 8 + s, kbyte)) = hi[s];
                }
            }
        }
    }
    fence_proxy_async_shared();                 // B tables -> tensor core (async proxy)
    return group_sync(ctl, gphase, lane, p);
}

template <bool kF32X, int kP>
__global__ void __launch_bounds__(kThreads, 1)
gemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_w, const TcArgs p) {
    using Geo = Geometry<kP>;
    using Dg = Digits<kF32X>;
    constexpr int kWStages = Geo::kWStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *wring = smem;                                          // kWStages x stage
    uint8_t *bsm = smem + p.off_b;                                  // B tables of one segment
    uint8_t *stages = smem + p.off_stage;                           // 2 x staged x, b, a
    Ctl *ctl = reinterpret_cast<Ctl *>(stages + 2 * p.stage_bytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const long long U = p.units;
    const long long u0 = range_begin(U, G, cta), u1 = range_begin(U, G, cta + 1);
    volatile int *abort_flag = &ctl->abort;
    // Tensor memory: scale factors (all 1.0) at [0, 32); the accumulator of path k at
    // acc_col0 + k*acc_stride; A stage s, path k at a_col0 + (s*kP + k)*16.
    const uint32_t sf_col = 0;
    const uint32_t acc_col0 = kSfCols;
    const uint32_t a_col0 = acc_col0 + static_cast<uint32_t>(kP * p.acc_stride);
    const int nb = (p.off_stage - p.off_b) / 16;   // 16-byte words of the B region

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWStages; ++s) {
            mbar_init(smem_u32(&ctl->w_full[s]), 1);
            mbar_init(smem_u32(&ctl->w_empty[s]), 4);
        }
        for (int s = 0; s < p.a_stages; ++s) {
            mbar_init(smem_u32(&ctl->a_full[s]), 4);
            mbar_init(smem_u32(&ctl->a_empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&ctl->x_full[s]), 64);     // 32 lanes x (async arrive + arrive)
            mbar_init(smem_u32(&ctl->x_empty[s]), 4);
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
        tmem_alloc(smem_u32(&ctl->tmem_base), p.tmem_cols);
        tmem_relinquish();
    }
    // B tables: zero, then the ones row (e2m1 1.0 = nibble 2) of every (pair, path) block;
    // digit rows are rewritten per segment, the others stay as set here.
    for (int i = threadIdx.x; i < nb; i += kThreads) reinterpret_cast<uint4 *>(bsm)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < 2 * kMaxBatch * 3; i += kThreads) (&ctl->zmax[0][0][0])[i] = 0u;
    __syncthreads();
    {
        const int blocks = nb * 16 / (p.nm * 128);
        for (int i = threadIdx.x; i < blocks * 32; i += kThreads) {
            const int blk = i / 32, kw = i % 32;
            *reinterpret_cast<uint32_t *>(bsm + static_cast<size_t>(blk) * p.nm * 128 + sw128_offset(p.ones_row, 4 * kw)) =
                0x22222222u;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    if (warp >= 2 && warp < 6) {
        // scale factors: 32 columns of 0x7F bytes (e8m0 1.0) on every lane
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0x7F7F7F7Fu;
        tmem_st_32x32b_x32(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + sf_col, v);
        tc_wait_st();
    }
    fence_proxy_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // The next kernel on the stream may start its own prologue (and its L2 prefetches) now;
    // its reads of our outputs wait for this grid's completion in its griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool issued[kMaxWStages] = {};
            uint32_t last_parity[kMaxWStages] = {};
            uint32_t it = 0;
            for (long long u = u0; u < u1; ++u, ++it) {
                const uint32_t s = it % kWStages, ph = (it / kWStages) & 1u;
                if (!mbar_wait_bounded(smem_u32(&ctl->w_empty[s]), ph ^ 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMV_WAIT_COPY))
                    break;
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
            int drain_abort = 0;
            for (int s = 0; s < kWStages; ++s)
                if (issued[s])
                    mbar_wait_bounded(smem_u32(&ctl->w_full[s]), last_parity[s], &drain_abort, p.timeout_ns,
                                      p.fault, FAULT_GEMM_DRAIN);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_mxf4_f32(kRows, p.nm);
            const uint32_t b_base = smem_u32(bsm);
            bool ok = true, any = false;
            uint32_t it = 0;
            for (long long u = u0; ok && u < u1;) {
                const long long tile_end = std::min<long long>(u1, (u / p.chunks + 1) * p.chunks);
                for (long long su = u; ok && su < tile_end; su += p.seg_chunks) {
                    const int nch = static_cast<int>(std::min<long long>(tile_end - su, p.seg_chunks));
                    for (int r = 0; r < nch; ++r, ++it) {
                        const uint32_t s = it % p.a_stages, ph = (it / p.a_stages) & 1u;
                        if (!mbar_wait_bounded(smem_u32(&ctl->a_full[s]), ph, abort_flag, p.timeout_ns,
                                               p.fault, FAULT_GEMV_WAIT_MMA)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < kP; ++k) {
                            const uint32_t bblk = b_base + static_cast<uint32_t>(((r >> 1) * kP + k) * p.nm * 128 + 64 * (r & 1));
                            const uint32_t acol = a_col0 + static_cast<uint32_t>((s * kP + k) * 16);
#pragma unroll
                            for (int kk = 0; kk < 2; ++kk)
                                tc_mma_mxf4_ts(tmem + acc_col0 + static_cast<uint32_t>(k * p.acc_stride), tmem + acol + 8 * kk,
                                               smem_desc_kmajor_sw128(bblk + 32 * kk), idesc, tmem + sf_col,
                                               tmem + sf_col + 16, (r | kk) != 0 ? 1u : 0u);
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
    } else if (warp == 6) {
        // ------------------------------------------------------------ stager: x, b, a per segment
        uint32_t seg = 0;
        bool ok = true;
        constexpr int kXSize = kF32X ? 4 : 2;
        constexpr int kPer16 = 16 / kXSize;
        for (long long u = u0; ok && u < u1;) {
            const int t = static_cast<int>(u / p.chunks);
            const long long tile_begin = static_cast<long long>(t) * p.chunks;
            const long long tile_end = std::min<long long>(u1, tile_begin + p.chunks);
            for (long long su = u; su < tile_end; su += p.seg_chunks, ++seg) {
                const int nch = static_cast<int>(std::min<long long>(tile_end - su, p.seg_chunks));
                const int j0 = static_cast<int>(su - tile_begin) * kChunkCols;
                const int ncols = nch * kChunkCols;
                const int buf = static_cast<int>(seg & 1u);
                if (!mbar_wait_bounded(smem_u32(&ctl->x_empty[buf]), ((seg >> 1) & 1u) ^ 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMV_WAIT_COPY)) {
                    ok = false;
                    break;
                }
                uint8_t *st = stages + buf * p.stage_bytes;
                const uint32_t xs = smem_u32(st + p.stage_off_x), bsd = smem_u32(st + p.stage_off_b),
                               as = smem_u32(st + p.stage_off_a);
                // b rows: 4 floats per 16-byte piece
                for (int k = 0; k < kP; ++k) {
                    const float *brow = p.b + static_cast<int64_t>(k) * p.K;
                    for (int c = 4 * lane; c < ncols; c += 128) {
                        const int j = j0 + c;
                        const uint32_t dst = bsd + static_cast<uint32_t>((k * p.brow + pad_f32(c)) * 4);
                        if (p.b_vec && j + 4 <= p.K) {
                            cp_async16(dst, brow + j, 16u);
                        } else {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                cp_async4(dst + 4 * i, j + i < p.K ? brow + j + i : p.b, j + i < p.K ? 4u : 0u);
                        }
                    }
                }
                // x rows: kPer16 elements per 16-byte piece
                for (int beta = 0; beta < p.batch; ++beta) {
                    const uint8_t *xrow = reinterpret_cast<const uint8_t *>(p.x) + static_cast<int64_t>(beta) * p.ldx * kXSize;
                    for (int c = kPer16 * lane; c < ncols; c += 32 * kPer16) {
                        const int j = j0 + c;
                        const int cpad = kF32X ? pad_f32(c) : pad_bf16(c);
                        const uint32_t dst = xs + static_cast<uint32_t>((beta * p.xrow + cpad) * kXSize);
                        if (p.x_vec && j + kPer16 <= p.K) {
                            cp_async16(dst, xrow + static_cast<int64_t>(j) * kXSize, 16u);
                        } else if (p.x_pair) {
                            // 4-byte pieces: one fp32, or a bf16 pair whose second half may lie past K
#pragma unroll
                            for (int i = 0; i < kPer16; i += 4 / kXSize) {
                                const bool in = j + i < p.K;
                                const uint32_t bytes = in ? static_cast<uint32_t>(min(4, (p.K - j - i) * kXSize)) : 0u;
                                cp_async4(dst + i * kXSize, in ? xrow + static_cast<int64_t>(j + i) * kXSize : p.x, bytes);
                            }
                        } else {
                            // rows not 4-byte aligned (bf16 only): plain loads and stores
                            unsigned short *d = reinterpret_cast<unsigned short *>(st + p.stage_off_x) + beta * p.xrow + cpad;
#pragma unroll
                            for (int i = 0; i < kPer16; ++i)
                                d[i] = j + i < p.K ? __ldg(reinterpret_cast<const unsigned short *>(xrow) + j + i)
                                                   : static_cast<unsigned short>(0);
                        }
                    }
                }
                // a of the tile's rows
                for (int k = 0; k < kP; ++k)
                    for (int r = lane; r < kRows; r += 32) {
                        const int n = t * kRows + r;
                        cp_async4(as + static_cast<uint32_t>((k * kRows + r) * 4),
                                  n < p.N ? p.a + static_cast<int64_t>(k) * p.N + n : p.a, n < p.N ? 4u : 0u);
                    }
                cp_async_arrive_noinc(smem_u32(&ctl->x_full[buf]));   // when this lane's copies land
                mbar_arrive(smem_u32(&ctl->x_full[buf]));            // its plain stores (release)
            }
            u = tile_end;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
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

            for (long long su = u; su < tile_end; su += p.seg_chunks, ++seg) {
                const int nch = static_cast<int>(std::min<long long>(tile_end - su, p.seg_chunks));
                const int buf = static_cast<int>(seg & 1u);
                const uint8_t *stage = stages + buf * p.stage_bytes;
                if (!mbar_wait_bounded(smem_u32(&ctl->x_full[buf]), (seg >> 1) & 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMV_WAIT_COPY))
                    ok = false;
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                if (!z_stage<kF32X, kP>(p, ctl, bsm, stage, nch, te, buf, gphase)) { ok = false; break; }
                // Chunks go two at a time: both are read and stored to tensor memory before one
                // wait for the stores, so the store round trip is paid once per pair.
                for (int r0 = 0; r0 < nch && ok; r0 += 2) {
                    const int cnt = min(2, nch - r0);
                    uint32_t words[2][kP][4];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h >= cnt) break;
                        const uint32_t itc = it + h;
                        const uint32_t ws = itc % kWStages, wph = (itc / kWStages) & 1u;
                        if (!mbar_wait_bounded(smem_u32(&ctl->w_full[ws]), wph, abort_flag, p.timeout_ns,
                                               p.fault, FAULT_GEMV_WAIT_COPY))
                            ok = false;
                        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                        const uint4 *src = reinterpret_cast<const uint4 *>(wring + ws * Geo::kStageBytes +
                                                                            row * Geo::kChunkWords * 4);
                        if constexpr (kP == 2) {
                            const uint4 g0 = src[0], g1 = src[1];
                            words[h][0][0] = g0.x; words[h][1][0] = g0.y; words[h][0][1] = g0.z; words[h][1][1] = g0.w;
                            words[h][0][2] = g1.x; words[h][1][2] = g1.y; words[h][0][3] = g1.z; words[h][1][3] = g1.w;
                        } else {
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                const uint4 v = src[g];
                                words[h][0][g] = v.x; words[h][1][g] = v.y; words[h][2][g] = v.z;
                            }
                        }
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&ctl->w_empty[ws]));
                    }
                    if (!ok) break;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h >= cnt) break;
                        const uint32_t itc = it + h;
                        const uint32_t as = itc % p.a_stages, aph = (itc / p.a_stages) & 1u;
                        if (!mbar_wait_bounded(smem_u32(&ctl->a_empty[as]), aph ^ 1u, abort_flag, p.timeout_ns,
                                               p.fault, FAULT_GEMV_WAIT_COPY))
                            ok = false;
                        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < kP; ++k) {
                            uint32_t v[16];
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
                                const uint32_t w = words[h][k][g];
                                v[4 * g + 0] = ((w << 3) & 0x88888888u) | 0x22222222u;
                                v[4 * g + 1] = ((w << 2) & 0x88888888u) | 0x22222222u;
                                v[4 * g + 2] = ((w << 1) & 0x88888888u) | 0x22222222u;
                                v[4 * g + 3] = (w & 0x88888888u) | 0x22222222u;
                            }
                            tmem_st_x16(tmem + lane_addr + a_col0 + static_cast<uint32_t>((as * kP + k) * 16), v);
                        }
                    }
                    if (!ok) break;
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        for (int h = 0; h < cnt; ++h) mbar_arrive(smem_u32(&ctl->a_full[(it + h) % p.a_stages]));
                    it += cnt;
                }
                if (!ok) break;
                // ---- epilogue of the segment
                if (!mbar_wait_bounded(smem_u32(&ctl->acc_full), seg & 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMV_WAIT_MMA))
                    ok = false;
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                const float *arow = reinterpret_cast<const float *>(stage + p.stage_off_a);
#pragma unroll
                for (int k = 0; k < kP; ++k) {
                    const uint32_t dcol = tmem + lane_addr + acc_col0 + static_cast<uint32_t>(k * p.acc_stride);
                    uint32_t one_bits;
                    tmem_ld_x1(dcol + static_cast<uint32_t>(p.ones_row), one_bits);
                    tc_wait_ld();
                    const long long ones = static_cast<long long>(__float2int_rn(__uint_as_float(one_bits)));
                    const float ak = arow[k * kRows + row];
#pragma unroll
                    for (int beta = 0; beta < kMaxBatch; ++beta) {
                        if (beta >= p.batch) break;
                        uint32_t d[Dg::kD];
                        if constexpr (kF32X) {
                            uint32_t d0[4], d1[4], d2[4];
                            tmem_ld_x4(dcol + 12 * beta, d0);
                            tmem_ld_x4(dcol + 12 * beta + 4, d1);
                            tmem_ld_x4(dcol + 12 * beta + 8, d2);
                            tc_wait_ld();
#pragma unroll
                            for (int i = 0; i < 4; ++i) { d[i] = d0[i]; d[4 + i] = d1[i]; d[8 + i] = d2[i]; }
                        } else {
                            uint32_t d8[8];
                            tmem_ld_x8(dcol + 8 * beta, d8);
                            tc_wait_ld();
#pragma unroll
                            for (int i = 0; i < 8; ++i) d[i] = d8[i];
                        }
                        long long tsum = 0;
#pragma unroll
                        for (int s = Dg::kD - 1; s >= 0; --s)
                            tsum = 4 * tsum + static_cast<long long>(__float2int_rn(2.0f * __uint_as_float(d[s])));
                        const long long tk = tsum - (ones << Dg::kOffsetLog2);
                        const int e = seg_exponent(ctl->zmax[buf][beta][k], Dg::kTop, Dg::kZqLimit);
                        const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
                        ypart[beta] += ak * (static_cast<float>(tk) * inv);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ctl->x_empty[buf]));   // stage buffer free
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
                    // The partials of contributors first..lastc, added in that (column) order.
                    // Loads go out eight at a time so their latencies overlap.
                    for (int beta = 0; beta < p.batch; ++beta) {
                        float sum = 0.0f;
                        for (int i0 = first; i0 <= lastc; i0 += 8) {
                            float v[8];
#pragma unroll
                            for (int d = 0; d < 8; ++d) {
                                const int i = i0 + d;
                                v[d] = 0.0f;
                                if (i <= lastc) {
                                    const int ti = static_cast<int>(range_begin(U, G, i) / p.chunks);
                                    const int si = (t == ti) ? 0 : 1;
                                    v[d] = __ldcg(p.partial + ((static_cast<int64_t>(i) * 2 + si) * p.batch + beta) * kRows + row);
                                }
                            }
#pragma unroll
                            for (int d = 0; d < 8; ++d)
                                if (i0 + d <= lastc) sum += v[d];
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
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

// Workspace: the partial sums first, in a region of fixed size (the largest grid and batch),
// then one counter per row tile.  Counters a call does not use are never written, so a
// workspace zero-filled once serves every later call, whatever its shape.
constexpr size_t kPartialBytes = static_cast<size_t>(kGemvMaxGrid) * 2 * kMaxBatch * kRows * sizeof(float);

}  // namespace

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
    const bool f32x = !x_bf16;
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

    TcArgs args{};
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
    args.nm = nm_for(batch, f32x);
    args.ones_row = digits_for(f32x) * batch;
    const int pair_bytes = P * args.nm * 128;                     // B of two chunks, all paths
    const int seg_pairs = std::max(1, std::min(kMaxSegChunks / 2, kBCap / pair_bytes));
    args.seg_chunks = 2 * seg_pairs;
    // tensor memory: scale factors, accumulators, A stages (4 when they fit in 256 columns)
    args.acc_stride = (args.nm + 15) / 16 * 16;
    const int fixed_cols = kSfCols + P * args.acc_stride;
    args.a_stages = (fixed_cols + 4 * P * 16 <= 256) ? 4 : ((fixed_cols + 2 * P * 16 <= 256) ? 2 : 4);
    args.tmem_cols = (fixed_cols + args.a_stages * P * 16 <= 256) ? 256u : 512u;
    args.debug = debug;
    const int grid = static_cast<int>(std::min<long long>(args.units, std::min(ctx.num_sms, kGemvMaxGrid)));
    args.partial = static_cast<float *>(workspace);
    args.tickets = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + kPartialBytes);

    // shared memory
    const int seg_cols = args.seg_chunks * kChunkCols;
    const int xsize = f32x ? 4 : 2;
    args.xrow = f32x ? pad_f32(seg_cols) : pad_bf16(seg_cols);   // padded elements per staged row
    args.brow = pad_f32(seg_cols);
    auto up16 = [](int v) { return (v + 15) / 16 * 16; };
    args.stage_off_x = 0;
    args.stage_off_b = up16(batch * args.xrow * xsize);
    args.stage_off_a = args.stage_off_b + up16(P * args.brow * 4);
    args.stage_bytes = up16(args.stage_off_a + P * kRows * 4);
    const int wring = (P == 2 ? Geometry<2>::kStageBytes * Geometry<2>::kWStages
                              : Geometry<3>::kStageBytes * Geometry<3>::kWStages);
    args.off_b = wring;
    args.off_stage = args.off_b + seg_pairs * pair_bytes;
    const int smem = args.off_stage + 2 * args.stage_bytes + static_cast<int>(sizeof(Ctl)) + 1024;
    args.x_vec = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && ((static_cast<int64_t>(ldx) * xsize) % 16 == 0);
    args.b_vec = (reinterpret_cast<uintptr_t>(b) % 16 == 0) && ((static_cast<int64_t>(K) * 4) % 16 == 0);
    args.x_pair = (reinterpret_cast<uintptr_t>(x) % 4 == 0) && ((static_cast<int64_t>(ldx) * xsize) % 4 == 0);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;

    void (*kern)(CUtensorMap, TcArgs);
    if (P == 2) kern = x_bf16 ? gemv_tc_kernel<false, 2> : gemv_tc_kernel<true, 2>;
    else kern = x_bf16 ? gemv_tc_kernel<false, 3> : gemv_tc_kernel<true, 3>;
    static ContextFlags opted[4];
    // the opt-in is set once per kernel and context, to the largest size any call asks for
    if (cudaError_t e = ensure_smem_optin(ctx, kern, 227 * 1024, opted[(P - 2) * 2 + (x_bf16 ? 0 : 1)]);
        e != cudaSuccess)
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
