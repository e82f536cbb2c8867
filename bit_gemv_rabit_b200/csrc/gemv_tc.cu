// gemv_tc.cu -- decode path of the residual-binary linear layer (batch 1..16) on tcgen05.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.1 "Multi-bit Approximation via Stacking", executed per path as Appendix E.1
// "Compute Pipeline" describes (paths in parallel, signs applied without multiplies,
// output scale applied last):
//     y[beta][n] = sum_k a_k[n] * t_k[beta][n],   t_k[beta][n] = sum_j S_k[n][j] z_k[beta][j],
//     z_k[beta][j] = b_k[j] * x[beta][j].
// One launch serves one layer or a group of independent layers (same path count, activation
// type and batch; e.g. the projections of a decoder that read the same input).
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
// Work split: a unit is 128 rows x 128 columns of one layer.  The units of all layers and row
// tiles, in order, are dealt as equal contiguous ranges to one persistent CTA per SM
// ("stream-K"), so every shape balances to within one unit.  A row tile that one CTA covers
// completely is written straight to y; partial tiles leave fp32 partial sums in the
// workspace, and the last contributor to arrive (a counter per tile) adds them in
// contributor order, which is the column order, so results are deterministic.
//
// Roles (16 warps; each group of four covers the four tensor-memory lane quarters):
//   warp 0       TMA producer: one 128-row x 128-column box of packed words per chunk into an
//                8-stage ring.  Before the programmatic-launch wait it only prefetches boxes to
//                L2 (no data reaches the SM, so nothing an earlier kernel still writes is seen).
//   warps 1, 3   MMA issuers (warp 1 also allocates tensor memory): one lane each issues the
//                MMAs of half the paths (M = 128, N = nm, K = 64, two per chunk and path) into the
//                segment's accumulator; two accumulators alternate when tensor memory allows,
//                so one segment's epilogue overlaps the next one's MMAs.  A single issuing
//                thread is slower than the tensor core at N <= 64, hence two.
//   warp 2       stager: x, b and a of each segment into a double-buffered shared-memory stage
//                with cp.async.
//   warps 4..7   z group: per segment the scales and the B tables (double-buffered), then the
//                previous segment's epilogue; per row tile the output or the partial.
//   warps 8..15  expansion: the sign words of each chunk into A stages in tensor memory;
//                warps 8..11 take even chunks and 12..15 odd ones, so two warps per SM
//                sub-partition hide each other's tensor-memory store latency.
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
constexpr int kThreads = 512;
constexpr int kZThread0 = 128;      // first thread of the z group (warp 4)
constexpr int kGroupThreads = 128;
constexpr int kMaxBatch = 16;
constexpr int kMaxSegChunks = 8;
constexpr int kBCap = 32 * 1024;    // shared memory one segment's B tables may take
constexpr int kSfCols = 32;         // tensor-memory columns holding the (constant) scale factors
constexpr int kAStages = 4;         // chunk i uses A stage i % 4 (even chunks 0, 2; odd 1, 3)
constexpr int kPrefetchChunks = 32; // boxes a CTA prefetches to L2 before the launch wait
constexpr int kWStages = 8;

template <int kP> struct Geometry {
    static constexpr int kGroupWords = kP == 2 ? 2 : 4;             // words per 32-column group
    static constexpr int kChunkWords = 4 * kGroupWords;             // words per row per chunk
    static constexpr int kStageBytes = kRows * kChunkWords * 4;     // 4 KiB (P=2), 8 KiB (P=3)
};

// Digits per batch row: 8 base-4 digits for 16-bit v (bf16 x), 12 for 24-bit v (fp32 x).
template <bool kF32X> struct Digits {
    static constexpr int kD = kF32X ? 12 : 8;
    static constexpr int kOffsetLog2 = kF32X ? 23 : 15;           // v = zq + 2^offset
    static constexpr int kTop = kF32X ? 22 : 14;                  // first guess of the scale exponent
    static constexpr float kZqLimit = kF32X ? 8388607.0f : 32767.0f;
};

struct Prob {
    const float *a;        // [P][N]
    const float *b;        // [P][K]
    const void *x;         // [batch][ldx]
    float *y;              // [batch][ldy]
    long long unit0;       // index of the layer's first unit in the launch
    int N, K, ldx, ldy;
    int tiles, chunks;     // row tiles, 128-column chunks per row
    int tile0;             // index of the layer's first row tile in the launch (counters)
    int x_vec, b_vec;      // rows of x / b start 16-byte aligned (cp.async of 16 bytes)
    int x_pair;            // x rows start 4-byte aligned (cp.async of 4 bytes)
};

struct GArgs {
    CUtensorMap tmap[kGemvMaxGroup];   // packed signs of each layer
    Prob prob[kGemvMaxGroup];
    float *partial;        // workspace: [grid][2][batch][128] (fixed-size region at offset 0)
    int *tickets;          // workspace: one counter per row tile, after the partial sums
    uint32_t *fault;
    uint64_t timeout_ns;
    long long units;
    int nprob, batch;
    int nm;                // MMA N: digit rows of all batch rows + the ones row, rounded to 8
    int acc_stride;        // tensor-memory columns per path's accumulator (nm rounded to 16)
    int n_acc;             // accumulators that alternate between segments (1 or 2)
    int ones_row;
    int seg_chunks;        // chunks per segment at most (even)
    uint32_t tmem_cols;
    // shared-memory layout (bytes from the 1024-aligned base)
    int off_b, b_buf_bytes, off_stage, stage_bytes, stage_off_x, stage_off_b, stage_off_a, xrow, brow;
    int debug;             // bit 1: the producer withholds its first copy (fault-injection test)
};

struct Ctl {
    uint64_t w_full[kWStages];
    uint64_t w_empty[kWStages];
    uint64_t a_full[kAStages];
    uint64_t a_empty[kAStages];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t x_full[2];
    uint64_t x_empty[2];
    uint64_t drain[2];                 // one per MMA issuer
    uint64_t group;                    // barrier of the z group (bounded, unlike bar.sync)
    uint32_t tmem_base;
    int abort;
    int last;                          // fix-up: this CTA arrived last for the tile
    uint32_t zmax[2][kMaxBatch][3];    // max |x b_k| (float bits) per (batch row, path), by segment parity
    int e[2][kMaxBatch][3];            // scale exponent per (batch row, path), by segment parity
};

// One segment of a CTA's range: chunks [c0, c0 + nch) of row tile `tile` of layer `prob`.
struct Seg {
    int prob, tile, c0, nch;
    long long tile_begin;              // launch-wide index of the tile's first unit
    bool last_of_tile;                 // the CTA's last segment in this tile
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
__device__ __forceinline__ int prob_of_unit(const GArgs &p, long long u) {
    int i = 0;
    while (i + 1 < p.nprob && p.prob[i + 1].unit0 <= u) ++i;
    return i;
}
// Launch-wide index of the row tile that holds unit u.
__device__ __forceinline__ int tile_of_unit(const GArgs &p, long long u) {
    const Prob &q = p.prob[prob_of_unit(p, u)];
    return q.tile0 + static_cast<int>((u - q.unit0) / q.chunks);
}

// The next segment of the range [u, u1): every role walks the same sequence.
__device__ __forceinline__ bool next_seg(const GArgs &p, long long &u, long long u1, Seg &s) {
    if (u >= u1) return false;
    const int i = prob_of_unit(p, u);
    const Prob &q = p.prob[i];
    const int t = static_cast<int>((u - q.unit0) / q.chunks);
    const long long tb = q.unit0 + static_cast<long long>(t) * q.chunks;
    const long long tend = std::min<long long>(u1, tb + q.chunks);
    const int nch = static_cast<int>(std::min<long long>(tend - u, p.seg_chunks));
    s.prob = i;
    s.tile = t;
    s.c0 = static_cast<int>(u - tb);
    s.nch = nch;
    s.tile_begin = tb;
    s.last_of_tile = (u + nch == tend);
    u += nch;
    return true;
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

// Barrier of the z group's four warps on an mbarrier of count 4, with a bounded wait: a warp
// that left after an expired wait makes the others time out too instead of hanging (bar.sync
// has no bound).  `phase` is the caller's running parity.  False once the CTA is aborting.
__device__ __forceinline__ bool group_sync(Ctl *ctl, uint32_t &phase, int lane, const GArgs &p) {
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&ctl->group));
    const bool ok = mbar_wait_bounded(smem_u32(&ctl->group), phase, &ctl->abort, p.timeout_ns, p.fault,
                                      FAULT_GEMV_WAIT_MMA);
    phase ^= 1u;
    return __all_sync(0xffffffffu, ok);
}

// A bounded wait taken by a whole warp: true when every lane saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const GArgs &p, Ctl *ctl, uint32_t bit) {
    const bool ok = mbar_wait_bounded(bar, parity, &ctl->abort, p.timeout_ns, p.fault, bit);
    return __all_sync(0xffffffffu, ok);
}

// Staged x value of batch row beta at segment column c (0 beyond K: the stager zero-fills).
template <bool kF32X>
__device__ __forceinline__ float staged_x(const uint8_t *xs, const GArgs &p, int beta, int c) {
    if constexpr (kF32X) {
        return reinterpret_cast<const float *>(xs)[beta * p.xrow + pad_f32(c)];
    } else {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const unsigned short *>(xs)[beta * p.xrow + pad_bf16(c)]) << 16);
    }
}

// The segment's z stage, run by the z group (zt = 0..127): the per (batch row, path) scale
// exponents (into e[buf]) and the B tables of chunks [0, nch) of the segment (into bsm), from
// the staged x and b.  zmax[buf] is zero on entry; zmax[buf ^ 1] is zeroed for the next segment.
template <bool kF32X, int kP>
__device__ bool z_stage(const GArgs &p, Ctl *ctl, uint8_t *bsm, const uint8_t *stage, int nch, int zt, int buf,
                        uint32_t &gphase) {
    using Dg = Digits<kF32X>;
    constexpr int kD = Dg::kD;
    const int lane = zt & 31;
    const uint8_t *xs = stage + p.stage_off_x;
    const float *bs = reinterpret_cast<const float *>(stage + p.stage_off_b);
    // ---- pass 1: max |x b_k| over the segment's columns
    const int ncols = nch * kChunkCols;
    for (int beta = 0; beta < p.batch; ++beta) {
        float m[kP];
#pragma unroll
        for (int k = 0; k < kP; ++k) m[k] = 0.0f;
        for (int c = zt; c < ncols; c += kGroupThreads) {
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
    for (int i = zt; i < kMaxBatch * 3; i += kGroupThreads) (&ctl->zmax[buf ^ 1][0][0])[i] = 0u;
    if (zt < p.batch * kP) {
        const int beta = zt / kP, k = zt % kP;
        ctl->e[buf][beta][k] = seg_exponent(ctl->zmax[buf][beta][k], Dg::kTop, Dg::kZqLimit);
    }
    // ---- pass 2: tuples (chunk r, group g, register q): 8 columns 32g + 4i + q of the chunk
    // give one 32-bit B word per digit row.
    const int ntuples = nch * 16;
    for (int tu = zt; tu < ntuples; tu += kGroupThreads) {
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
                uint32_t lo[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float z = xv[i] * bs[k * p.brow + pad_f32(cb + 4 * i)];
                    uint32_t v;
                    if constexpr (kF32X) {
                        v = static_cast<uint32_t>(__float2int_rn(z * sc) + (1 << Dg::kOffsetLog2));
                    } else {
                        // |z sc| < 2^15: adding 1.5 * 2^23 rounds it to an integer (to nearest
                        // even, as rint) held in the low mantissa bits; adding 2^15 there too
                        // gives v = zq + 2^15 in the low 16 bits.
                        v = __float_as_uint(fmaf(z, sc, 12582912.0f + 32768.0f)) & 0xFFFFu;
                    }
                    lo[i] = spread16(v & 0xFFFFu);
                }
                transpose8x8_nibbles(lo);
                uint8_t *blk = pair + static_cast<size_t>(k) * p.nm * 128;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    *reinterpret_cast<uint32_t *>(blk + sw128_offset(kD * beta + s, kbyte)) = lo[s];
                if constexpr (kF32X) {
                    uint32_t hi[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float z = xv[i] * bs[k * p.brow + pad_f32(cb + 4 * i)];
                        const uint32_t v = static_cast<uint32_t>(__float2int_rn(z * sc) + (1 << Dg::kOffsetLog2));
                        hi[i] = spread16(v >> 16);
                    }
                    transpose8x8_nibbles(hi);
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        *reinterpret_cast<uint32_t *>(blk + sw128_offset(kD * beta + 8 + s, kbyte)) = hi[s];
                }
            }
        }
    }
    fence_proxy_async_shared();                 // B tables -> tensor core (async proxy)
    return group_sync(ctl, gphase, lane, p);    // e[buf] and the tables are complete
}

template <bool kF32X, int kP>
__global__ void __launch_bounds__(kThreads, 1)
gemv_tc_kernel(const __grid_constant__ GArgs p) {
    using Geo = Geometry<kP>;
    using Dg = Digits<kF32X>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *wring = smem;                                          // kWStages x weight box
    uint8_t *bsm = smem + p.off_b;                                  // 2 x B tables
    uint8_t *stages = smem + p.off_stage;                           // 2 x staged x, b, a
    Ctl *ctl = reinterpret_cast<Ctl *>(stages + 2 * p.stage_bytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const long long U = p.units;
    const long long u0 = range_begin(U, G, cta), u1 = range_begin(U, G, cta + 1);
    volatile int *abort_flag = &ctl->abort;
    // Tensor memory: scale factors (all 1.0) at [0, 32); accumulator j of path k at
    // 32 + (j*kP + k)*acc_stride; A stage s, path k at a_col0 + (s*kP + k)*16.
    const uint32_t acc_col0 = kSfCols;
    const uint32_t a_col0 = acc_col0 + static_cast<uint32_t>(p.n_acc * kP * p.acc_stride);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kWStages; ++s) {
            mbar_init(smem_u32(&ctl->w_full[s]), 1);
            mbar_init(smem_u32(&ctl->w_empty[s]), 4);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(smem_u32(&ctl->a_full[s]), 4);
            mbar_init(smem_u32(&ctl->a_empty[s]), 2);     // one commit per MMA issuer
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&ctl->b_full[s]), 4);
            mbar_init(smem_u32(&ctl->b_empty[s]), 2);
            mbar_init(smem_u32(&ctl->acc_full[s]), 2);
            mbar_init(smem_u32(&ctl->acc_empty[s]), 4);
            mbar_init(smem_u32(&ctl->x_full[s]), 64);     // 32 lanes x (async arrive + arrive)
            mbar_init(smem_u32(&ctl->x_empty[s]), 4);
        }
        mbar_init(smem_u32(&ctl->drain[0]), 1);
        mbar_init(smem_u32(&ctl->drain[1]), 1);
        mbar_init(smem_u32(&ctl->group), 4);
        ctl->abort = 0;
        fence_mbarrier_init();
        // L2 prefetch of the first boxes of this CTA's range (weights only)
        long long u = u0;
        Seg s;
        int n = 0;
        while (n < kPrefetchChunks && next_seg(p, u, u1, s)) {
            prefetch_tensormap(&p.tmap[s.prob]);
            for (int r = 0; r < s.nch && n < kPrefetchChunks; ++r, ++n)
                tma_prefetch_2d(&p.tmap[s.prob], (s.c0 + r) * Geo::kChunkWords, s.tile * kRows);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl->tmem_base), p.tmem_cols);
        tmem_relinquish();
    }
    // B tables (both buffers): zero, then the ones row (e2m1 1.0 = nibble 2) of every
    // (pair, path) block; digit rows are rewritten per segment, the others stay as set here.
    const int nb16 = (p.off_stage - p.off_b) / 16;
    for (int i = threadIdx.x; i < nb16; i += kThreads) reinterpret_cast<uint4 *>(bsm)[i] = make_uint4(0u, 0u, 0u, 0u);
    for (int i = threadIdx.x; i < 2 * kMaxBatch * 3; i += kThreads) (&ctl->zmax[0][0][0])[i] = 0u;
    __syncthreads();
    {
        const int blocks = nb16 * 16 / (p.nm * 128);
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
    if (warp >= 4 && warp < 8) {
        // scale factors: 32 columns of 0x7F bytes (e8m0 1.0) on every lane
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0x7F7F7F7Fu;
        tmem_st_32x32b_x32(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16), v);
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
            bool issued[kWStages] = {};
            uint32_t last_parity[kWStages] = {};
            uint32_t it = 0;
            bool ok = true;
            long long u = u0;
            Seg s;
            while (ok && next_seg(p, u, u1, s)) {
                for (int r = 0; r < s.nch; ++r, ++it) {
                    const uint32_t st = it % kWStages, ph = (it / kWStages) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&ctl->w_empty[st]), ph ^ 1u, abort_flag, p.timeout_ns,
                                           p.fault, FAULT_GEMV_WAIT_COPY)) {
                        ok = false;
                        break;
                    }
                    if ((p.debug & 2) && it == 0) continue;   // fault injection: this copy never comes
                    const uint32_t bar = smem_u32(&ctl->w_full[st]);
                    mbar_arrive_expect_tx(bar, Geo::kStageBytes);
                    tma_load_2d(smem_u32(wring + st * Geo::kStageBytes), &p.tmap[s.prob], bar,
                                (s.c0 + r) * Geo::kChunkWords, s.tile * kRows);
                    issued[st] = true;
                    last_parity[st] = ph;
                }
            }
            // Every issued copy lands before the CTA can exit, also when the consumers stopped
            // early on an expired wait.  These are the latest phases of their stages, already
            // complete in normal operation.
            int drain_abort = 0;
            for (int st = 0; st < kWStages; ++st)
                if (issued[st])
                    mbar_wait_bounded(smem_u32(&ctl->w_full[st]), last_parity[st], &drain_abort, p.timeout_ns,
                                      p.fault, FAULT_GEMM_DRAIN);
        }
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------------------ MMA issuers
        if (lane == 0) {
            const int issuer = warp == 1 ? 0 : 1;     // paths k with k % 2 == issuer
            const uint32_t idesc = idesc_mxf4_f32(kRows, p.nm);
            // Descriptors and addresses are built once; per MMA only their start fields move
            // (the descriptor's start address is addr >> 4 in its low bits, so a byte offset
            // o adds o >> 4).
            const uint64_t bdesc0 = smem_desc_kmajor_sw128(smem_u32(bsm));
            const uint32_t block16 = static_cast<uint32_t>(p.nm * 128) >> 4;       // one (pair, path) block
            const uint32_t buf16 = static_cast<uint32_t>(p.b_buf_bytes) >> 4;
            bool ok = true, any = false;
            uint32_t it = 0, seg = 0;
            long long u = u0;
            Seg s;
            while (ok && next_seg(p, u, u1, s)) {
                const uint32_t bb = seg & 1u, ab = seg % static_cast<uint32_t>(p.n_acc);
                if (!mbar_wait_bounded(smem_u32(&ctl->b_full[bb]), (seg >> 1) & 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMV_WAIT_MMA) ||
                    !mbar_wait_bounded(smem_u32(&ctl->acc_empty[ab]), ((seg / p.n_acc) & 1u) ^ 1u, abort_flag,
                                       p.timeout_ns, p.fault, FAULT_GEMV_WAIT_MMA)) {
                    ok = false;
                    break;
                }
                const uint64_t bseg = bdesc0 + bb * buf16;
                const uint32_t dacc = tmem + acc_col0 + ab * static_cast<uint32_t>(kP * p.acc_stride);
                for (int r = 0; r < s.nch; ++r, ++it) {
                    const uint32_t st = it % kAStages, ph = (it / kAStages) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&ctl->a_full[st]), ph, abort_flag, p.timeout_ns, p.fault,
                                           FAULT_GEMV_WAIT_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bchunk = bseg + static_cast<uint32_t>((r >> 1) * kP) * block16 + (r & 1) * 4u;
                    const uint32_t achunk = tmem + a_col0 + st * kP * 16;
#pragma unroll
                    for (int k = issuer; k < kP; k += 2) {
                        const uint64_t bk = bchunk + static_cast<uint32_t>(k) * block16;
                        const uint32_t dk = dacc + static_cast<uint32_t>(k * p.acc_stride);
                        tc_mma_mxf4_ts(dk, achunk + k * 16, bk, idesc, tmem, tmem + 16, r != 0 ? 1u : 0u);
                        tc_mma_mxf4_ts(dk, achunk + k * 16 + 8, bk + 2, idesc, tmem, tmem + 16, 1u);
                    }
                    any = true;
                    tc_commit(smem_u32(&ctl->a_empty[st]));     // frees A stage st when done
                }
                if (!ok) break;
                tc_commit(smem_u32(&ctl->b_empty[bb]));         // B tables free when these MMAs are done
                tc_commit(smem_u32(&ctl->acc_full[ab]));
                ++seg;
            }
            if (!ok && any) {
                tc_commit(smem_u32(&ctl->drain[issuer]));
                int drain_abort = 0;
                mbar_wait_bounded(smem_u32(&ctl->drain[issuer]), 0, &drain_abort, p.timeout_ns, p.fault,
                                  FAULT_GEMM_DRAIN);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ stager: x, b, a per segment
        uint32_t seg = 0;
        constexpr int kXSize = kF32X ? 4 : 2;
        constexpr int kPer16 = 16 / kXSize;
        long long u = u0;
        Seg s;
        while (next_seg(p, u, u1, s)) {
            const Prob &q = p.prob[s.prob];
            const int j0 = s.c0 * kChunkCols;
            const int ncols = s.nch * kChunkCols;
            const int buf = static_cast<int>(seg & 1u);
            if (!warp_wait(smem_u32(&ctl->x_empty[buf]), ((seg >> 1) & 1u) ^ 1u, p, ctl, FAULT_GEMV_WAIT_COPY)) break;
            uint8_t *st = stages + buf * p.stage_bytes;
            const uint32_t xs = smem_u32(st + p.stage_off_x), bsd = smem_u32(st + p.stage_off_b),
                           as = smem_u32(st + p.stage_off_a);
            // b rows: 4 floats per 16-byte piece
            for (int k = 0; k < kP; ++k) {
                const float *brow = q.b + static_cast<int64_t>(k) * q.K;
                for (int c = 4 * lane; c < ncols; c += 128) {
                    const int j = j0 + c;
                    const uint32_t dst = bsd + static_cast<uint32_t>((k * p.brow + pad_f32(c)) * 4);
                    if (q.b_vec && j + 4 <= q.K) {
                        cp_async16(dst, brow + j, 16u);
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            cp_async4(dst + 4 * i, j + i < q.K ? brow + j + i : q.b, j + i < q.K ? 4u : 0u);
                    }
                }
            }
            // x rows: kPer16 elements per 16-byte piece
            for (int beta = 0; beta < p.batch; ++beta) {
                const uint8_t *xrow = reinterpret_cast<const uint8_t *>(q.x) + static_cast<int64_t>(beta) * q.ldx * kXSize;
                for (int c = kPer16 * lane; c < ncols; c += 32 * kPer16) {
                    const int j = j0 + c;
                    const int cpad = kF32X ? pad_f32(c) : pad_bf16(c);
                    const uint32_t dst = xs + static_cast<uint32_t>((beta * p.xrow + cpad) * kXSize);
                    if (q.x_vec && j + kPer16 <= q.K) {
                        cp_async16(dst, xrow + static_cast<int64_t>(j) * kXSize, 16u);
                    } else if (q.x_pair) {
                        // 4-byte pieces: one fp32, or a bf16 pair whose second half may lie past K
#pragma unroll
                        for (int i = 0; i < kPer16; i += 4 / kXSize) {
                            const bool in = j + i < q.K;
                            const uint32_t bytes = in ? static_cast<uint32_t>(min(4, (q.K - j - i) * kXSize)) : 0u;
                            cp_async4(dst + i * kXSize, in ? xrow + static_cast<int64_t>(j + i) * kXSize : q.x, bytes);
                        }
                    } else {
                        // rows not 4-byte aligned (bf16 only): plain loads and stores
                        unsigned short *d = reinterpret_cast<unsigned short *>(st + p.stage_off_x) + beta * p.xrow + cpad;
#pragma unroll
                        for (int i = 0; i < kPer16; ++i)
                            d[i] = j + i < q.K ? __ldg(reinterpret_cast<const unsigned short *>(xrow) + j + i)
                                               : static_cast<unsigned short>(0);
                    }
                }
            }
            // a of the tile's rows
            for (int k = 0; k < kP; ++k)
                for (int r = lane; r < kRows; r += 32) {
                    const int n = s.tile * kRows + r;
                    cp_async4(as + static_cast<uint32_t>((k * kRows + r) * 4),
                              n < q.N ? q.a + static_cast<int64_t>(k) * q.N + n : q.a, n < q.N ? 4u : 0u);
                }
            cp_async_arrive_noinc(smem_u32(&ctl->x_full[buf]));   // when this lane's copies land
            mbar_arrive(smem_u32(&ctl->x_full[buf]));            // its plain stores (release)
            ++seg;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp >= 8) {
        // ------------------------------------------------------------ expansion of the sign words
        const int half = (warp - 8) >> 2;            // 0: even chunks, 1: odd chunks
        const int q4 = warp & 3;                     // lane quarter this warp may access
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const int row = q4 * 32 + lane;
        uint32_t it = 0;
        for (long long u = u0; u < u1; ++u, ++it) {
            if (static_cast<int>(it & 1u) != half) continue;
            const uint32_t ws = it % kWStages, wph = (it / kWStages) & 1u;
            if (!warp_wait(smem_u32(&ctl->w_full[ws]), wph, p, ctl, FAULT_GEMV_WAIT_COPY)) break;
            const uint4 *src = reinterpret_cast<const uint4 *>(wring + ws * Geo::kStageBytes + row * Geo::kChunkWords * 4);
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
            if (!warp_wait(smem_u32(&ctl->a_empty[as]), aph ^ 1u, p, ctl, FAULT_GEMV_WAIT_COPY)) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                uint32_t v[16];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t w = words[k][g];
                    v[4 * g + 0] = ((w << 3) & 0x88888888u) | 0x22222222u;
                    v[4 * g + 1] = ((w << 2) & 0x88888888u) | 0x22222222u;
                    v[4 * g + 2] = ((w << 1) & 0x88888888u) | 0x22222222u;
                    v[4 * g + 3] = (w & 0x88888888u) | 0x22222222u;
                }
                tmem_st_x16(tmem + lane_addr + a_col0 + (as * kP + k) * 16, v);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->a_full[as]));
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ z group: z stage, epilogue, output
        const int zt = threadIdx.x - kZThread0;      // 0..127 = tensor-memory lane = tile row
        const int q4 = warp & 3;
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const int row = q4 * 32 + lane;
        bool ok = true;
        uint32_t seg = 0, gphase = 0;
        float ypart[kMaxBatch];
#pragma unroll
        for (int i = 0; i < kMaxBatch; ++i) ypart[i] = 0.0f;
        const int first_tile = tile_of_unit(p, u0);

        // Epilogue of segment sg (already z-staged; its MMAs were issued): t -> ypart, and the
        // row tile's output after its last segment.
        auto epilogue = [&](const Seg &s, uint32_t sg) -> bool {
            const uint32_t ab = sg % static_cast<uint32_t>(p.n_acc), buf = sg & 1u;
            if (!warp_wait(smem_u32(&ctl->acc_full[ab]), (sg / p.n_acc) & 1u, p, ctl, FAULT_GEMV_WAIT_MMA)) return false;
            tc_fence_after();
            const uint8_t *stage = stages + buf * p.stage_bytes;
            const float *arow = reinterpret_cast<const float *>(stage + p.stage_off_a);
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                const uint32_t dcol = tmem + lane_addr + acc_col0 + (ab * kP + k) * static_cast<uint32_t>(p.acc_stride);
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
                    for (int sd = Dg::kD - 1; sd >= 0; --sd)
                        tsum = 4 * tsum + static_cast<long long>(__float2int_rn(2.0f * __uint_as_float(d[sd])));
                    const long long tk = tsum - (ones << Dg::kOffsetLog2);
                    const float inv = __uint_as_float(static_cast<uint32_t>(127 - ctl->e[buf][beta][k]) << 23);
                    ypart[beta] += ak * (static_cast<float>(tk) * inv);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(&ctl->acc_empty[ab]));   // accumulator free for a later segment
                mbar_arrive(smem_u32(&ctl->x_empty[buf]));    // stage buffer free
            }
            if (!s.last_of_tile) return true;
            // ---- row tile done: write y, or the partial and the counter
            const Prob &q = p.prob[s.prob];
            const int n = s.tile * kRows + row;
            const int gtile = q.tile0 + s.tile;
            const int first = unit_owner(U, G, s.tile_begin);
            const int lastc = unit_owner(U, G, s.tile_begin + q.chunks - 1);
            if (first == lastc) {
                if (n < q.N) {
#pragma unroll
                    for (int beta = 0; beta < kMaxBatch; ++beta)
                        if (beta < p.batch) q.y[static_cast<int64_t>(beta) * q.ldy + n] = ypart[beta];
                }
            } else {
                const int side = (gtile == first_tile) ? 0 : 1;
                float *slot = p.partial + (static_cast<int64_t>(cta) * 2 + side) * p.batch * kRows;
#pragma unroll
                for (int beta = 0; beta < kMaxBatch; ++beta)
                    if (beta < p.batch) slot[beta * kRows + row] = ypart[beta];
                __threadfence();
                if (!group_sync(ctl, gphase, lane, p)) return false;
                if (zt == 0) {
                    const int old = atomicAdd(&p.tickets[gtile], 1);
                    ctl->last = (old == lastc - first) ? 1 : 0;
                }
                if (!group_sync(ctl, gphase, lane, p)) return false;
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
                                    const int si = (gtile == tile_of_unit(p, range_begin(U, G, i))) ? 0 : 1;
                                    v[d] = __ldcg(p.partial + ((static_cast<int64_t>(i) * 2 + si) * p.batch + beta) * kRows + row);
                                }
                            }
#pragma unroll
                            for (int d = 0; d < 8; ++d)
                                if (i0 + d <= lastc) sum += v[d];
                        }
                        if (n < q.N) q.y[static_cast<int64_t>(beta) * q.ldy + n] = sum;
                    }
                    if (zt == 0) p.tickets[gtile] = 0;
                }
            }
#pragma unroll
            for (int i = 0; i < kMaxBatch; ++i) ypart[i] = 0.0f;
            return true;
        };

        long long u = u0;
        Seg s, prev{};
        bool pending = false;
        while (next_seg(p, u, u1, s)) {
            const uint32_t buf = seg & 1u;
            if (!warp_wait(smem_u32(&ctl->x_full[buf]), (seg >> 1) & 1u, p, ctl, FAULT_GEMV_WAIT_COPY) ||
                !warp_wait(smem_u32(&ctl->b_empty[buf]), ((seg >> 1) & 1u) ^ 1u, p, ctl, FAULT_GEMV_WAIT_MMA)) {
                ok = false;
                break;
            }
            const uint8_t *stage = stages + buf * p.stage_bytes;
            if (!z_stage<kF32X, kP>(p, ctl, bsm + buf * p.b_buf_bytes, stage, s.nch, zt, static_cast<int>(buf), gphase)) {
                ok = false;
                break;
            }
            if (lane == 0) mbar_arrive(smem_u32(&ctl->b_full[buf]));
            if (pending && !epilogue(prev, seg - 1)) { ok = false; break; }
            prev = s;
            pending = true;
            ++seg;
        }
        if (ok && pending) epilogue(prev, seg - 1);
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

struct Layout {
    int nm, acc_stride, n_acc, seg_chunks, b_buf_bytes, xrow, brow, stage_off_x, stage_off_b, stage_off_a,
        stage_bytes, off_b, off_stage, smem;
    uint32_t tmem_cols;
};

// Shared- and tensor-memory layout of a launch; false when `batch` rows do not fit at once.
bool plan_layout(int P, bool f32x, int batch, Layout &L) {
    L.nm = nm_for(batch, f32x);
    L.acc_stride = (L.nm + 15) / 16 * 16;
    const int a_cols = kAStages * P * 16;
    if (kSfCols + 2 * P * L.acc_stride + a_cols <= 512) L.n_acc = 2;
    else if (kSfCols + P * L.acc_stride + a_cols <= 512) L.n_acc = 1;
    else return false;
    const int need = kSfCols + L.n_acc * P * L.acc_stride + a_cols;
    L.tmem_cols = need <= 256 ? 256u : 512u;
    const int pair_bytes = P * L.nm * 128;                        // B of two chunks, all paths
    const int seg_pairs = std::max(1, std::min(kMaxSegChunks / 2, kBCap / pair_bytes));
    L.seg_chunks = 2 * seg_pairs;
    L.b_buf_bytes = seg_pairs * pair_bytes;
    const int seg_cols = L.seg_chunks * kChunkCols;
    const int xsize = f32x ? 4 : 2;
    L.xrow = f32x ? pad_f32(seg_cols) : pad_bf16(seg_cols);       // padded elements per staged row
    L.brow = pad_f32(seg_cols);
    auto up16 = [](int v) { return (v + 15) / 16 * 16; };
    L.stage_off_x = 0;
    L.stage_off_b = up16(batch * L.xrow * xsize);
    L.stage_off_a = L.stage_off_b + up16(P * L.brow * 4);
    L.stage_bytes = up16(L.stage_off_a + P * kRows * 4);
    L.off_b = (P == 2 ? Geometry<2>::kStageBytes : Geometry<3>::kStageBytes) * kWStages;
    L.off_stage = L.off_b + 2 * L.b_buf_bytes;
    L.smem = L.off_stage + 2 * L.stage_bytes + static_cast<int>(sizeof(Ctl)) + 1024;
    return L.smem <= 227 * 1024;
}

}  // namespace

size_t gemv_workspace_bytes(int N, int K, int P, int batch) {
    (void)K;
    (void)P;
    (void)batch;
    const size_t tiles = (static_cast<size_t>(N) + kRows - 1) / kRows;
    return kPartialBytes + ((tiles * sizeof(int) + 15) / 16) * 16;
}

size_t gemv_group_workspace_bytes(const GemvLayer *layers, int count) {
    size_t tiles = 0;
    for (int i = 0; i < count; ++i) tiles += (static_cast<size_t>(layers[i].N) + kRows - 1) / kRows;
    return kPartialBytes + ((tiles * sizeof(int) + 15) / 16) * 16;
}

cudaError_t launch_gemv_group(const LaunchCtx &ctx, const GemvLayer *layers, int count, int P, bool x_bf16,
                              int batch, void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug) {
    if ((P != 2 && P != 3) || count < 1 || count > kGemvMaxGroup) return cudaErrorInvalidValue;
    const bool f32x = !x_bf16;
    const int xsize = f32x ? 4 : 2;
    // The largest batch slice whose accumulators fit in tensor memory (and its tables in shared
    // memory); a bigger batch runs as several launches over slices of the batch rows.
    int slice = batch;
    Layout L{};
    while (slice > 1 && !plan_layout(P, f32x, slice, L)) --slice;
    if (!plan_layout(P, f32x, slice, L)) return cudaErrorInvalidValue;

    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    if (!encode) return cudaErrorNotSupported;
    void (*kern)(GArgs);
    if (P == 2) kern = x_bf16 ? gemv_tc_kernel<false, 2> : gemv_tc_kernel<true, 2>;
    else kern = x_bf16 ? gemv_tc_kernel<false, 3> : gemv_tc_kernel<true, 3>;
    static ContextFlags opted[4];
    // the opt-in is set once per kernel and context, to the largest size any call asks for
    if (cudaError_t e = ensure_smem_optin(ctx, kern, 227 * 1024, opted[(P - 2) * 2 + (x_bf16 ? 0 : 1)]);
        e != cudaSuccess)
        return e;

    GArgs args{};
    const int G = P == 2 ? 2 : 4;
    long long units = 0;
    int tiles = 0;
    for (int i = 0; i < count; ++i) {
        const GemvLayer &l = layers[i];
        const int Kp = static_cast<int>(padded_cols(l.K));
        const int words_per_row = Kp / 32 * G;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(words_per_row), static_cast<cuuint64_t>(l.N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(words_per_row) * 4};
        cuuint32_t box[2] = {static_cast<cuuint32_t>(4 * G), static_cast<cuuint32_t>(kRows)};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&args.tmap[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(l.packed), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        Prob &q = args.prob[i];
        q.a = l.a;
        q.b = l.b;
        q.N = l.N;
        q.K = l.K;
        q.ldx = l.ldx;
        q.ldy = l.ldy;
        q.tiles = (l.N + kRows - 1) / kRows;
        q.chunks = Kp / kChunkCols;
        q.unit0 = units;
        q.tile0 = tiles;
        q.b_vec = (reinterpret_cast<uintptr_t>(l.b) % 16 == 0) && ((static_cast<int64_t>(l.K) * 4) % 16 == 0);
        units += static_cast<long long>(q.tiles) * q.chunks;
        tiles += q.tiles;
    }
    args.partial = static_cast<float *>(workspace);
    args.tickets = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + kPartialBytes);
    args.fault = fault_word;
    args.timeout_ns = timeout_ns;
    args.units = units;
    args.nprob = count;
    args.nm = L.nm;
    args.acc_stride = L.acc_stride;
    args.n_acc = L.n_acc;
    args.seg_chunks = L.seg_chunks;
    args.tmem_cols = L.tmem_cols;
    args.off_b = L.off_b;
    args.b_buf_bytes = L.b_buf_bytes;
    args.off_stage = L.off_stage;
    args.stage_bytes = L.stage_bytes;
    args.stage_off_x = L.stage_off_x;
    args.stage_off_b = L.stage_off_b;
    args.stage_off_a = L.stage_off_a;
    args.xrow = L.xrow;
    args.brow = L.brow;
    args.debug = debug;
    const int grid = static_cast<int>(std::min<long long>(units, std::min(ctx.num_sms, kGemvMaxGrid)));

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(L.smem);
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Batch slices share the layout of the first (largest) slice: a narrower last slice only
    // uses fewer rows of the tables and accumulators.
    for (int b0 = 0; b0 < batch; b0 += slice) {
        args.batch = std::min(slice, batch - b0);
        args.ones_row = digits_for(f32x) * args.batch;
        for (int i = 0; i < count; ++i) {
            const GemvLayer &l = layers[i];
            Prob &q = args.prob[i];
            q.x = static_cast<const uint8_t *>(l.x) + static_cast<int64_t>(b0) * l.ldx * xsize;
            q.y = l.y + static_cast<int64_t>(b0) * l.ldy;
            q.x_vec = (reinterpret_cast<uintptr_t>(q.x) % 16 == 0) && ((static_cast<int64_t>(l.ldx) * xsize) % 16 == 0);
            q.x_pair = (reinterpret_cast<uintptr_t>(q.x) % 4 == 0) && ((static_cast<int64_t>(l.ldx) * xsize) % 4 == 0);
        }
        if (cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args); e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_gemv_tc(const LaunchCtx &ctx, const uint32_t *packed, const float *a, const float *b,
                           int N, int K, int P, const void *x, bool x_bf16, int batch, int ldx, float *y,
                           int ldy, void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug) {
    GemvLayer l{packed, a, b, N, K, x, ldx, y, ldy};
    return launch_gemv_group(ctx, &l, 1, P, x_bf16, batch, workspace, fault_word, timeout_ns, debug);
}

}  // namespace rabit
