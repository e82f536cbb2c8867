// gemv_tc.cu -- decode path of the residual-binary linear layer (batch 1..16) on tcgen05.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.1 "Multi-bit Approximation via Stacking", executed per path as Appendix E.1
// "Compute Pipeline" describes (paths in parallel, signs applied without multiplies,
// output scale applied last):
//     y[beta][n] = sum_k a_k[n] * t_k[beta][n],   t_k[beta][n] = sum_j S_k[n][j] z_k[beta][j],
//     z_k[beta][j] = b_k[j] * x[beta][j].
// One call serves one layer or a group of independent layers (same path count, activation
// type and batch; e.g. the projections of a decoder that read the same input).
//
// Arithmetic.  z (an fp32 product) is quantised once per (layer, path, batch row), over the
// whole row: zq = rint(z * 2^e) with one power-of-two scale such that |zq| <= 2^15 - 1 (bf16
// x) or 2^23 - 1 (fp32 x).  The sign sum t = sum_j S_j zq_j is then computed exactly on the
// tensor cores with packed 4-bit operands (tcgen05.mma kind::mxf4, every block scale 1.0):
//   - A (tensor memory, lane = weight row): each sign as the e2m1 value +1 or -1.  From a
//     packed word w, register r = 0..3 is ((w << (3 - r)) & 0x88888888) | 0x22222222: its
//     nibble i is the sign of column 4i + r of the word (bit 3 of an e2m1 nibble is its sign).
//     Register r of 32-column group g is tensor-memory column 4g + r, so contraction index
//     32g + 8r + i holds column 32g + 4i + r.
//   - B (shared memory, K-major, 128-byte swizzle): zq in balanced base 4 with D digits
//     (D = 8 for bf16 x, 12 for fp32 x): zq = sum_s 4^s d_s, d_s in {-2, -1, 0, 1} for
//     s < D - 1 and the top digit in {-2, ..., 2}; row D*beta + s holds d_s as an e2m1 value
//     (all five values are exact in e2m1).
//   Each accumulator D_s = sum_j S_j d_s,j is an integer below 2^24 in magnitude, exact in
//   fp32, and t = sum_s 4^s D_s is formed exactly in 64-bit integers.  The only roundings are
//   z itself, its quantisation and the conversion of t to fp32.
//
// Three kernels per call, chained by programmatic dependent launch:
//   gemv_blockmax_kernel, gemv_prep_kernel  one CTA per (layer, batch row, 1024 columns): the
//                     maximum |z| of the block per path, then the row's scale from the block
//                     maxima and the B operand of the block for every path, written to the
//                     workspace as the exact shared-memory image the tensor core reads (the main
//                     kernel moves it with bulk copies of about 32 KiB).  The first also clears
//                     the fix-up counters.
//   gemv_tc_kernel    the signs.  A unit is one 128-byte-wide TMA box of packed words: 128 or
//                     256 rows (one or two halves; a row tile has the same height) x 512
//                     columns (2 paths) or 256 (3 paths), 16 or 32 KiB -- the copy engine
//                     streams boxes of 32 KiB at the copy rate of plain loads, while smaller
//                     copies are bound by a per-copy cost.  The units of all layers and row
//                     tiles, in order, are dealt as equal contiguous ranges to one persistent
//                     CTA per SM ("stream-K"), so every shape balances to within one unit.  A CTA accumulates its run of units inside one row tile
//                     in tensor memory and reads the accumulators once per run.  A row tile
//                     that one CTA covers completely is written straight to y; partial tiles
//                     leave fp32 partial sums in the workspace, and the last contributor to
//                     arrive (a counter per tile) adds them in contributor order, which is the
//                     column order, so results are deterministic.
// Roles of gemv_tc_kernel (25 warps; each group of four covers the four tensor-memory lane
// quarters):
//   warp 0        producer: per unit one TMA box of packed sign words into a ring of stages,
//                 and per run of units about 32 KiB of B images at a time (one bulk copy) into
//                 a second ring.  The boxes of the first pass over the ring are requested
//                 before the programmatic-launch wait (the kernel this one waits for, the prep
//                 kernel, does not write the signs); the B images after it.
//   warps 1, 22..24  MMA issuers (warp 1 also owns the tensor memory): one lane each issues
//                 the MMAs of one half and path (M = 128, N = rows of B, K = 64; four per
//                 256-column pair) into the run's accumulators.  One issuing thread sustains
//                 about one MMA per 50 clocks, far below the tensor core, hence four.
//   warps 2..5    epilogue: per run, t from the accumulators, scaled by 2^-e and a, then the
//                 output or the partial and the fix-up.
//   warps 6..21   expansion: the sign words of a unit from shared memory into A stages in
//                 tensor memory, one stage per (half, 256-column pair); four groups of four
//                 warps, group g filling stage g, so four stages are expanded at once.
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

constexpr int kRows = 128;              // rows per half unit: MMA M, tensor-memory lanes
constexpr int kPairCols = 256;          // columns per pair (one B image, four MMA K steps)
constexpr int kUnitGroups = kPairCols / 32;   // 32-column groups per pair
constexpr int kMaxBatch = 16;
constexpr int kSfCols = 32;             // tensor-memory columns holding the (constant) scale factors
constexpr int kMaxWStages = 8;
constexpr int kMaxAStages = 4;
constexpr int kMaxBBufs = 2;
constexpr int kPrefetchUnits = 0;       // boxes a CTA prefetches to L2 before the wait (they would
                                        // delay the prep kernel's reads, which gate the MMAs)
constexpr int kEarlyBoxes = 2;          // boxes requested before the programmatic-launch wait
constexpr int kThreads = 25 * 32;
constexpr int kWarpExpand0 = 6;         // expansion warps 6..21: four groups of four
constexpr int kWarpIssuer1 = 22;        // MMA issuers 1..3 are warps 22..24
constexpr int kPrepThreads = 128;      // small enough to share an SM with a main-kernel CTA
constexpr int kPrepCols = 8 * kPrepThreads;   // columns per prep CTA

template <int kP> struct Geometry {
    static constexpr int kGroupWords = kP == 2 ? 2 : 4;             // words per 32-column group
    static constexpr int kBoxPairs = 32 / (kUnitGroups * kGroupWords);   // pairs in 128 bytes of a row
};

template <bool kF32X> struct Digits {
    static constexpr int kD = kF32X ? 12 : 8;
    static constexpr int kLowBits = 2 * (kD - 1);                  // bits of the D-1 low digits
    static constexpr int kOffset = kF32X ? 2796202 : 10922;        // 2 (4^(D-1) - 1) / 3
    static constexpr int kTop = kF32X ? 22 : 14;                   // first guess of the scale exponent
    static constexpr float kZqLimit = kF32X ? 8388607.0f : 32767.0f;
};

// ---------------------------------------------------------------- prep kernel
struct PrepLayer {
    const void *x;          // [batch][ldx]
    const float *b;         // [P][K]
    long long img_off;      // byte offset of the layer's B images inside one batch slice's images
    int K, ldx, pairs;      // pairs: 256-column units per row
    int blocks;             // CTAs per batch row
    int vec;                // x rows and b rows start 16-byte aligned
};

struct PrepArgs {
    PrepLayer layer[kGemvMaxGroup];
    uint8_t *img;           // [slices][layers][pairs][P][nm rows x 128 bytes]
    float *inv;             // [layer][P][batch]: 2^-e
    float *bmax;            // [layer][P][batch][maxblk]: max |z| of each block of columns
    int *tickets;           // fix-up counters of the main kernel, cleared here
    long long slice_bytes;
    int ntickets, nprob, batch, slice, nm, maxblk;
};

// The (layer, batch row, column block) of a prep CTA.
__device__ __forceinline__ void prep_coords(const PrepArgs &p, int &l, int &beta, int &blk) {
    int bid = blockIdx.x;
    l = 0;
    while (l + 1 < p.nprob && bid >= p.layer[l].blocks * p.batch) {
        bid -= p.layer[l].blocks * p.batch;
        ++l;
    }
    beta = bid / p.layer[l].blocks;
    blk = bid - beta * p.layer[l].blocks;
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

// e2m1 codes, in every nibble that `m` selects (0x1 per nibble), of the digits d = u - 2 for
// base-4 digits u in bits 0..1 of the nibbles of w: u = 0, 1, 2, 3 -> d = -2 (0xC), -1 (0xA),
// 0 (0x0), 1 (0x2).  Bit 3 = (u < 2), bit 2 = (u == 0), bit 1 = (u odd).
__device__ __forceinline__ uint32_t low_digit_codes(uint32_t w, uint32_t m) {
    const uint32_t b0 = w & m, b1 = (w >> 1) & m;
    const uint32_t n1 = b1 ^ m, n0 = b0 ^ m;
    return (n1 << 3) | ((n1 & n0) << 2) | (b0 << 1);
}

// e2m1 code of a digit d in {-2, ..., 2}: sign in bit 3, |d| = 1 -> 0x2, |d| = 2 -> 0x4.
__device__ __forceinline__ uint32_t top_digit_code(int d) {
    return (d < 0 ? 8u : 0u) | static_cast<uint32_t>(2 * abs(d));
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
    for (int i = 0; i < 8; i += 4) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t a = e[i + j], b = e[i + j + 2];
            e[i + j] = prmt(a, b, 0x6240u);
            e[i + j + 2] = prmt(a, b, 0x7351u);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
        const uint32_t a = e[i], b = e[i + 1];
        e[i] = (a & 0x0F0F0F0Fu) | ((b << 4) & 0xF0F0F0F0u);
        e[i + 1] = ((a >> 4) & 0x0F0F0F0Fu) | (b & 0xF0F0F0F0u);
    }
}

// Scale exponent of a row: zq = rint(z 2^e) stays within +-limit for every z of the row.
__device__ __forceinline__ int row_exponent(float mx, int top, float limit) {
    if (!(mx > 0.0f)) return 0;
    const int E = static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu) - 127;
    int e = min(126, max(-126, top - E));                 // 2^-e stays a normal float
    if (mx * __uint_as_float(static_cast<uint32_t>(e + 127) << 23) > limit) --e;
    return e;
}

// Byte offset, inside one (unit, path) B image of 128-byte rows in 128-byte-swizzled atoms of
// 8 rows, of the 4-byte word r of 16-byte group gg of row `row`.
__device__ __forceinline__ uint32_t b_image_offset(int row, int gg, int r) {
    return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + (((gg ^ (row & 7)) & 7) << 4) + 4 * r);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

template <bool kF32X>
__device__ __forceinline__ float load_x(const void *xrow, int j) {
    if constexpr (kF32X) return static_cast<const float *>(xrow)[j];
    else return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t *>(xrow)[j]) << 16);
}

// First prep kernel: the max |z| of each path over the block's 1024 columns (8 per thread),
// one value per (layer, path, batch row, block).  It also clears the fix-up counters.
template <bool kF32X, int kP>
__global__ void __launch_bounds__(kPrepThreads)
gemv_blockmax_kernel(const __grid_constant__ PrepArgs p) {
    __shared__ float red[kP][kPrepThreads / 32];
    // x and b may come from the previous kernel on the stream; the next kernel of this call
    // reads what we write only after its own wait.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (blockIdx.x == 0)
        for (int i = tid; i < p.ntickets; i += kPrepThreads) p.tickets[i] = 0;
    int l, beta, blk;
    prep_coords(p, l, beta, blk);
    const PrepLayer &q = p.layer[l];
    const int K = q.K;
    const float *b = q.b;
    const void *xrow = static_cast<const uint8_t *>(q.x) +
                       static_cast<int64_t>(beta) * q.ldx * (kF32X ? 4 : 2);
    float mx[kP];
#pragma unroll
    for (int k = 0; k < kP; ++k) mx[k] = 0.0f;
    const int c0 = blk * kPrepCols + 8 * tid;
    if (q.vec && c0 + 8 <= K) {
        float xv[8];
        if constexpr (kF32X) {
            const float4 v0 = reinterpret_cast<const float4 *>(xrow)[c0 / 4];
            const float4 v1 = reinterpret_cast<const float4 *>(xrow)[c0 / 4 + 1];
            xv[0] = v0.x; xv[1] = v0.y; xv[2] = v0.z; xv[3] = v0.w;
            xv[4] = v1.x; xv[5] = v1.y; xv[6] = v1.z; xv[7] = v1.w;
        } else {
            const uint4 v = reinterpret_cast<const uint4 *>(xrow)[c0 / 8];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                xv[2 * h] = __uint_as_float(w[h] << 16);
                xv[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
            }
        }
#pragma unroll
        for (int k = 0; k < kP; ++k) {
            const float4 b0 = reinterpret_cast<const float4 *>(b + static_cast<int64_t>(k) * K)[c0 / 4];
            const float4 b1 = reinterpret_cast<const float4 *>(b + static_cast<int64_t>(k) * K)[c0 / 4 + 1];
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int h = 0; h < 8; ++h) mx[k] = fmaxf(mx[k], fabsf(__fmul_rn(bv[h], xv[h])));
        }
    } else {
        for (int c = c0; c < min(c0 + 8, K); ++c) {
            const float xv = load_x<kF32X>(xrow, c);
#pragma unroll
            for (int k = 0; k < kP; ++k) mx[k] = fmaxf(mx[k], fabsf(__fmul_rn(b[static_cast<int64_t>(k) * K + c], xv)));
        }
    }
#pragma unroll
    for (int k = 0; k < kP; ++k) {
        mx[k] = warp_max(mx[k]);
        if (lane == 0) red[k][warp] = mx[k];
    }
    __syncthreads();
    if (tid < kP) {
        float m = red[tid][0];
#pragma unroll
        for (int w = 1; w < kPrepThreads / 32; ++w) m = fmaxf(m, red[tid][w]);
        p.bmax[((static_cast<int64_t>(l) * kP + tid) * p.batch + beta) * p.maxblk + blk] = m;
    }
}

// Second prep kernel: the row's scale from the block maxima, then the B images of the block.
template <bool kF32X, int kP>
__global__ void __launch_bounds__(kPrepThreads)
gemv_prep_kernel(const __grid_constant__ PrepArgs p) {
    using Dg = Digits<kF32X>;
    constexpr int kD = Dg::kD;
    // The block maxima come from the previous kernel.  The main kernel of this call may start
    // once every CTA is past this point: it reads nothing of ours before its own wait.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int tid = threadIdx.x;
    int l, beta, blk;
    prep_coords(p, l, beta, blk);
    const PrepLayer &q = p.layer[l];
    const int K = q.K;
    const float *b = q.b;
    const void *xrow = static_cast<const uint8_t *>(q.x) +
                       static_cast<int64_t>(beta) * q.ldx * (kF32X ? 4 : 2);
    float sc[kP];
#pragma unroll
    for (int k = 0; k < kP; ++k) {
        const float *bm = p.bmax + ((static_cast<int64_t>(l) * kP + k) * p.batch + beta) * p.maxblk;
        float m = 0.0f;
        for (int i = 0; i < q.blocks; ++i) m = fmaxf(m, bm[i]);
        const int e = row_exponent(m, Dg::kTop, Dg::kZqLimit);
        sc[k] = __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
        if (blk == 0 && tid == k)
            p.inv[(static_cast<int64_t>(l) * kP + k) * p.batch + beta] =
                __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
    }

    // ---- B images: thread (g, r) writes word r of group g of every digit row, for the
    // columns 32g + 4i + r, i = 0..7 (nibble i of the word)
    const int g = blk * (kPrepCols / 32) + (tid >> 2);
    const int r = tid & 3;
    if (g >= q.pairs * kUnitGroups) return;
    const int sl = beta / p.slice, bl = beta - sl * p.slice;
    const int nb = min(p.slice, p.batch - sl * p.slice);
    const int gg = g & (kUnitGroups - 1);
    uint8_t *base = p.img + sl * p.slice_bytes + q.img_off + static_cast<int64_t>(g >> 3) * kP * p.nm * 128;
    float xv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int c = 32 * g + 4 * i + r;
        xv[i] = c < K ? load_x<kF32X>(xrow, c) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < kP; ++k) {
        uint32_t w0[8], w1[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = 32 * g + 4 * i + r;
            const float z = c < K ? __fmul_rn(b[static_cast<int64_t>(k) * K + c], xv[i]) : 0.0f;
            const int v = __float2int_rn(__fmul_rn(z, sc[k])) + Dg::kOffset;
            const int top = v >> Dg::kLowBits;                         // arithmetic: -2..2
            const uint32_t low = static_cast<uint32_t>(v) & ((1u << Dg::kLowBits) - 1u);
            if constexpr (kF32X) {
                w0[i] = low_digit_codes(spread16(low & 0xFFFFu), 0x11111111u);
                w1[i] = low_digit_codes(spread16(low >> 16), 0x00000111u) | (top_digit_code(top) << 12);
            } else {
                w0[i] = low_digit_codes(spread16(low), 0x01111111u) | (top_digit_code(top) << 28);
                w1[i] = 0u;
            }
        }
        transpose8x8_nibbles(w0);
        if constexpr (kF32X) transpose8x8_nibbles(w1);
        uint8_t *pb = base + static_cast<int64_t>(k) * p.nm * 128;
#pragma unroll
        for (int s = 0; s < kD; ++s)
            *reinterpret_cast<uint32_t *>(pb + b_image_offset(kD * bl + s, gg, r)) = s < 8 ? w0[s] : w1[s - 8];
        if (bl == nb - 1)   // rows past the slice's digits (MMA N is a multiple of 8)
            for (int row = kD * nb; row < p.nm; ++row)
                *reinterpret_cast<uint32_t *>(pb + b_image_offset(row, gg, r)) = 0u;
    }
}

// ---------------------------------------------------------------- main kernel
struct Prob {
    const float *a;        // [P][N]
    const float *inv;      // 2^-e of the slice's first batch row: [P][inv_stride]
    const uint8_t *img;    // the layer's B images for this slice: [pairs][P][nm x 128 bytes]
    float *y;              // [batch][ldy], from the slice's first batch row
    long long unit0;       // index of the layer's first unit in the launch
    int N, ldy;
    int tiles;             // row tiles of 128 * mh rows
    int pairs;             // 256-column pairs per row
    int tunits;            // units per row tile
    int tile0;             // index of the layer's first row tile in the launch (counters)
};

struct GArgs {
    CUtensorMap tmap[kGemvMaxGroup];   // packed signs of each layer
    Prob prob[kGemvMaxGroup];
    float *partial;        // workspace: [grid][2][batch][128 * mh] (fixed-size region at offset 0)
    int *tickets;          // workspace: one counter per row tile
    uint32_t *fault;
    uint64_t timeout_ns;
    long long units;
    int nprob;
    int nb;                // batch rows of this launch (a slice of the call's batch)
    int nm;                // MMA N: digit rows of the slice, rounded up to 8
    int acc_stride;        // tensor-memory columns per accumulator (nm rounded to 16)
    int n_acc;             // accumulator sets that alternate between runs (1 or 2)
    int mh;                // 128-row halves per unit and tile (1 or 2)
    int n_a, n_w, n_b;     // A stages (tensor memory), sign-box stages, B-chunk buffers
    int cpu;               // units per B chunk
    int inv_stride;        // the call's batch
    uint32_t tmem_cols;
    int w_bytes;           // one sign box: 128 * mh rows x 128 bytes
    int chunk_bytes;       // one B-chunk buffer
    int debug;             // bit 1: the producer withholds its first box (fault-injection test)
};

struct Ctl {
    uint64_t w_full[kMaxWStages];
    uint64_t w_empty[kMaxWStages];
    uint64_t b_full[kMaxBBufs];
    uint64_t b_empty[kMaxBBufs];
    uint64_t a_full[kMaxAStages];
    uint64_t a_empty[kMaxAStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain[4];                 // one per MMA issuer
    uint64_t group;                    // barrier of the epilogue warps (bounded, unlike bar.sync)
    uint32_t tmem_base;
    int abort;
    int last;                          // fix-up: this CTA arrived last for the tile
    float inv[kGemvMaxGroup][3][kMaxBatch];   // 2^-e of every layer, path and batch row
};

// One run of a CTA's range: units [u0, u0 + n) of row tile `tile` of layer `prob` (unit v of
// a tile covers pairs [v * kUpp, v * kUpp + kUpp) of the row).
struct Run {
    int prob, tile, u0, n;
    long long tile_begin;              // launch-wide index of the tile's first unit
};

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
    return q.tile0 + static_cast<int>((u - q.unit0) / q.tunits);
}

// The next run of the range [u, u1): every role walks the same sequence.
__device__ __forceinline__ bool next_run(const GArgs &p, long long &u, long long u1, Run &r) {
    if (u >= u1) return false;
    const int i = prob_of_unit(p, u);
    const Prob &q = p.prob[i];
    const int t = static_cast<int>((u - q.unit0) / q.tunits);
    const long long tb = q.unit0 + static_cast<long long>(t) * q.tunits;
    const long long te = std::min<long long>(u1, tb + q.tunits);
    r.prob = i;
    r.tile = t;
    r.u0 = static_cast<int>(u - tb);
    r.n = static_cast<int>(te - u);
    r.tile_begin = tb;
    u = te;
    return true;
}

// Instruction descriptor, kind::mxf4: packed e2m1 A and B (K-major), fp32 accumulator, e8m0
// block scales, K = 64.  A and B format 1 = e2m1, bit 23 = scale format e8m0, N >> 3 at 17,
// M >> 4 at 24, scale-factor ids 0.
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
__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_ld_x4(uint32_t taddr, uint32_t (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(taddr) : "memory");
}
// Bulk copy (no tensor map, no multicast) global -> this CTA's shared memory, completion via
// mbarrier tx-count.  Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar) : "memory");
}

// Barrier of the four epilogue warps on an mbarrier of count 4, with a bounded wait: a warp
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

// The same for a warp that waits long and often (the epilogue): it sleeps between polls, so
// the issue slots go to the warps that stream.
__device__ __forceinline__ bool warp_wait_idle(uint32_t bar, uint32_t parity, const GArgs &p, Ctl *ctl,
                                               uint32_t bit) {
    bool ok = true;
    if (!mbar_try_wait(bar, parity)) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bar, parity)) {
            __nanosleep(256);
            if (ctl->abort) { ok = false; break; }
            if (global_timer_ns() - t0 > p.timeout_ns) {
                atomicOr(p.fault, bit);
                ctl->abort = 1;
                ok = false;
                break;
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// A stage j of the tensor-memory ring holds the signs of (unit i, half h, pair q) with
// j = (i * mh + h) * kUpp + q, in stage j % n_a, which expansion group j % n_a fills.
template <int kUpp>
__device__ __forceinline__ uint32_t a_seq(int i, int h, int q, int mh) {
    return static_cast<uint32_t>((i * mh + h) * kUpp + q);
}

template <bool kF32X, int kP>
__global__ void __launch_bounds__(kThreads, 1)
gemv_tc_kernel(const __grid_constant__ GArgs p) {
    using Dg = Digits<kF32X>;
    constexpr int kUpp = Geometry<kP>::kBoxPairs;      // pairs per unit (one 128-byte box row)
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *wring = smem;                                          // n_w sign boxes
    uint8_t *bring = smem + p.n_w * p.w_bytes;                      // n_b B chunks
    Ctl *ctl = reinterpret_cast<Ctl *>(bring + p.n_b * p.chunk_bytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const long long U = p.units;
    const long long u0 = range_begin(U, G, cta), u1 = range_begin(U, G, cta + 1);
    const int mh = p.mh;
    const int tile_rows = kRows * mh;
    // MMA issuers: two per half, one for path 0 (and path 2 when there are three), one for path 1
    const int n_issuers = 2 * mh;
    const uint32_t pair_bytes = static_cast<uint32_t>(kP * p.nm * 128);
    volatile int *abort_flag = &ctl->abort;
    // Tensor memory: scale factors (all 1.0) at [0, 32); accumulator of set s, half h, path k
    // at 32 + ((s*mh + h)*kP + k)*acc_stride; A stage j, path k at a_col0 + (j*kP + k)*32.
    const uint32_t acc_col0 = kSfCols;
    const uint32_t a_col0 = acc_col0 + static_cast<uint32_t>(p.n_acc * mh * kP * p.acc_stride);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.n_w; ++s) {
            mbar_init(smem_u32(&ctl->w_full[s]), 1);
            // the expansion warps that read it: four per group with a triple in the unit
            mbar_init(smem_u32(&ctl->w_empty[s]), 4 * std::min(p.n_a, mh * kUpp));
        }
        for (int s = 0; s < p.n_b; ++s) {
            mbar_init(smem_u32(&ctl->b_full[s]), 1);
            mbar_init(smem_u32(&ctl->b_empty[s]), n_issuers);
        }
        for (int s = 0; s < p.n_a; ++s) {
            mbar_init(smem_u32(&ctl->a_full[s]), 4);
            mbar_init(smem_u32(&ctl->a_empty[s]), 2);       // the two issuers of its half
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_u32(&ctl->acc_full[s]), n_issuers);
            mbar_init(smem_u32(&ctl->acc_empty[s]), 4);
        }
        for (int s = 0; s < 4; ++s) mbar_init(smem_u32(&ctl->drain[s]), 1);
        mbar_init(smem_u32(&ctl->group), 4);
        ctl->abort = 0;
        ctl->last = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl->tmem_base), p.tmem_cols);
        tmem_relinquish();
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
        tmem_st_32x32b_x32(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16), v);
        tc_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The next kernel on the stream may start its prologue now; whatever it reads of ours
    // waits for this grid's completion in its own griddepcontrol.wait.
    asm volatile("griddepcontrol.launch_dependents;");

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int S = p.n_w;
            bool issued[kMaxWStages] = {};
            uint32_t last_parity[kMaxWStages] = {};
            bool bissued[kMaxBBufs] = {};
            uint32_t blast_parity[kMaxBBufs] = {};
            for (int l = 0; l < p.nprob; ++l) prefetch_tensormap(&p.tmap[l]);
            // The first sign boxes go out before the programmatic-launch wait (the prep kernel
            // does not write the signs), the rest of the ring only after the first B chunk: the
            // copy engine serves requests in order, and the MMAs need both.
            const int early = S < kEarlyBoxes ? S : kEarlyBoxes;
            {
                long long u = u0;
                Run r;
                int i = 0;
                while (i < early + kPrefetchUnits && next_run(p, u, u1, r)) {
                    for (int v = 0; v < r.n && i < early + kPrefetchUnits; ++v, ++i) {
                        const int cx = (r.u0 + v) * 32, cy = r.tile * tile_rows;
                        if (i < early) {
                            const uint32_t bar = smem_u32(&ctl->w_full[i]);
                            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(p.w_bytes));
                            if ((p.debug & 2) && i == 0) continue;   // fault injection: never arrives
                            tma_load_2d(smem_u32(wring + i * p.w_bytes), &p.tmap[r.prob], bar, cx, cy);
                            issued[i] = true;
                        } else {
                            tma_prefetch_2d(&p.tmap[r.prob], cx, cy);
                        }
                    }
                }
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            bool ok = true;
            int i = 0, st = 0, bb = 0;
            uint32_t par = 0, bpar = 0;
            long long u = u0;
            Run r;
            while (ok && next_run(p, u, u1, r)) {
                const Prob &q = p.prob[r.prob];
                for (int v = 0; v < r.n; ++v, ++i) {
                    if (v % p.cpu == 0) {
                        // B chunk: the images of the pairs of units v .. v + cpu - 1 of the run
                        const int pr0 = (r.u0 + v) * kUpp;
                        const int pr1 = std::min(q.pairs, (r.u0 + std::min(v + p.cpu, r.n)) * kUpp);
                        if (!mbar_wait_bounded(smem_u32(&ctl->b_empty[bb]), bpar ^ 1u, abort_flag, p.timeout_ns,
                                               p.fault, FAULT_GEMV_WAIT_COPY)) {
                            ok = false;
                            break;
                        }
                        const uint32_t bytes = static_cast<uint32_t>(pr1 - pr0) * pair_bytes;
                        const uint32_t bar = smem_u32(&ctl->b_full[bb]);
                        mbar_arrive_expect_tx(bar, bytes);
                        bulk_load(smem_u32(bring + bb * p.chunk_bytes), q.img + static_cast<int64_t>(pr0) * pair_bytes,
                                  bytes, bar);
                        bissued[bb] = true;
                        blast_parity[bb] = bpar;
                        if (++bb == p.n_b) {
                            bb = 0;
                            bpar ^= 1u;
                        }
                    }
                    if (i >= early) {
                        if (i >= S && !mbar_wait_bounded(smem_u32(&ctl->w_empty[st]), par ^ 1u, abort_flag, p.timeout_ns,
                                                         p.fault, FAULT_GEMV_WAIT_COPY)) {
                            ok = false;
                            break;
                        }
                        const uint32_t bar = smem_u32(&ctl->w_full[st]);
                        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(p.w_bytes));
                        tma_load_2d(smem_u32(wring + st * p.w_bytes), &p.tmap[r.prob], bar, (r.u0 + v) * 32,
                                    r.tile * tile_rows);
                        issued[st] = true;
                        last_parity[st] = par;
                    }
                    if (++st == S) {
                        st = 0;
                        par ^= 1u;
                    }
                }
            }
            // Every issued copy lands before the CTA can exit, also when the consumers stopped
            // early on an expired wait.  These are the latest phases of their buffers, already
            // complete in normal operation.
            int drain_abort = 0;
            for (int s = 0; s < S; ++s)
                if (issued[s])
                    mbar_wait_bounded(smem_u32(&ctl->w_full[s]), last_parity[s], &drain_abort, p.timeout_ns,
                                      p.fault, FAULT_GEMM_DRAIN);
            for (int s = 0; s < p.n_b; ++s)
                if (bissued[s])
                    mbar_wait_bounded(smem_u32(&ctl->b_full[s]), blast_parity[s], &drain_abort, p.timeout_ns,
                                      p.fault, FAULT_GEMM_DRAIN);
        }
    } else if (warp == 1 || warp >= kWarpIssuer1) {
        // ------------------------------------------------------------ MMA issuers
        // Issuer ii issues the MMAs of half ii / 2 for path ii % 2 (and path 2 with issuer 0 of the
        // half): one issuing thread sustains only about one MMA per 50 clocks, so the MMAs are
        // spread over four threads.
        const int issuer = warp == 1 ? 0 : warp - kWarpIssuer1 + 1;
        if (lane == 0 && issuer < n_issuers) {
            const uint32_t idesc = idesc_mxf4_f32(kRows, p.nm);
            // Descriptors are built once; per MMA only their start fields move (the start
            // address is addr >> 4 in the low bits, so a byte offset o adds o >> 4).
            const uint64_t bdesc0 = smem_desc_kmajor_sw128(smem_u32(bring));
            const uint32_t chunk16 = static_cast<uint32_t>(p.chunk_bytes) >> 4;
            const uint32_t pair16 = pair_bytes >> 4;
            const uint32_t path16 = static_cast<uint32_t>(p.nm * 128) >> 4;
            const uint32_t set_cols = static_cast<uint32_t>(mh * kP * p.acc_stride);
            const int h = issuer >> 1, kfirst = issuer & 1;
            int bb = 0, i = 0;
            uint32_t bpar = 0, run = 0;
            bool ok = true, any = false;
            long long u = u0;
            Run r;
            while (ok && next_run(p, u, u1, r)) {
                const Prob &q = p.prob[r.prob];
                const uint32_t ab = run % static_cast<uint32_t>(p.n_acc);
                if (!mbar_wait_bounded(smem_u32(&ctl->acc_empty[ab]), ((run / p.n_acc) & 1u) ^ 1u, abort_flag,
                                       p.timeout_ns, p.fault, FAULT_GEMV_WAIT_MMA)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dh = tmem + acc_col0 + ab * set_cols + static_cast<uint32_t>(h * kP * p.acc_stride);
                int cpair0 = 0;                                     // first pair of the current chunk
                for (int v = 0; v < r.n; ++v, ++i) {
                    if (v % p.cpu == 0) {
                        if (!mbar_wait_bounded(smem_u32(&ctl->b_full[bb]), bpar, abort_flag, p.timeout_ns, p.fault,
                                               FAULT_GEMV_WAIT_COPY)) {
                            ok = false;
                            break;
                        }
                        cpair0 = (r.u0 + v) * kUpp;
                    }
                    const uint64_t bchunk = bdesc0 + static_cast<uint64_t>(static_cast<uint32_t>(bb) * chunk16);
#pragma unroll
                    for (int qq = 0; qq < kUpp; ++qq) {
                        const uint32_t j = a_seq<kUpp>(i, h, qq, mh);
                        const uint32_t slot = j % static_cast<uint32_t>(p.n_a);
                        if (!mbar_wait_bounded(smem_u32(&ctl->a_full[slot]), (j / p.n_a) & 1u, abort_flag,
                                               p.timeout_ns, p.fault, FAULT_GEMV_WAIT_MMA)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const int pr = (r.u0 + v) * kUpp + qq;
                        if (pr < q.pairs) {
                            const uint64_t bp = bchunk + static_cast<uint64_t>(static_cast<uint32_t>(pr - cpair0) * pair16);
                            const uint32_t a0 = tmem + a_col0 + slot * static_cast<uint32_t>(kP * 32);
                            const uint32_t acc = (v != 0 || qq != 0) ? 1u : 0u;
#pragma unroll
                            for (int k = kfirst; k < kP; k += 2) {
                                const uint32_t dk = dh + static_cast<uint32_t>(k * p.acc_stride);
                                const uint32_t ak = a0 + static_cast<uint32_t>(k * 32);
                                const uint64_t bk = bp + static_cast<uint64_t>(static_cast<uint32_t>(k) * path16);
                                tc_mma_mxf4_ts(dk, ak, bk, idesc, tmem, tmem + 16, acc);
                                tc_mma_mxf4_ts(dk, ak + 8, bk + 2, idesc, tmem, tmem + 16, 1u);
                                tc_mma_mxf4_ts(dk, ak + 16, bk + 4, idesc, tmem, tmem + 16, 1u);
                                tc_mma_mxf4_ts(dk, ak + 24, bk + 6, idesc, tmem, tmem + 16, 1u);
                            }
                            any = true;
                        }
                        tc_commit(smem_u32(&ctl->a_empty[slot]));       // A stage free when done
                    }
                    if (!ok) break;
                    if ((v + 1) % p.cpu == 0 || v + 1 == r.n) {
                        tc_commit(smem_u32(&ctl->b_empty[bb]));         // B chunk free when done
                        if (++bb == p.n_b) {
                            bb = 0;
                            bpar ^= 1u;
                        }
                    }
                }
                if (!ok) break;
                tc_commit(smem_u32(&ctl->acc_full[ab]));
                ++run;
            }
            if (!ok && any) {
                tc_commit(smem_u32(&ctl->drain[issuer]));
                int drain_abort = 0;
                mbar_wait_bounded(smem_u32(&ctl->drain[issuer]), 0, &drain_abort, p.timeout_ns, p.fault,
                                  FAULT_GEMM_DRAIN);
            }
        }
    } else if (warp >= kWarpExpand0 && warp < kWarpIssuer1) {
        // ------------------------------------------------------------ expansion of the sign words
        // Group g (warps 6 + 4g .. 9 + 4g, one per lane quarter) fills A stage g: the signs of
        // the (unit, half, pair) triples whose sequence index j is g modulo the stage count.
        const int grp = (warp - kWarpExpand0) >> 2;
        const int q4 = warp & 3;                     // lane quarter this warp may access
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const int n_units = static_cast<int>(u1 - u0);
        if (grp < p.n_a) {
            const uint32_t slot = static_cast<uint32_t>(grp);
            for (int i = 0; i < n_units; ++i) {
                // does this group take a triple of unit i?  (j runs over i * mh * kUpp + 0 ..)
                const uint32_t jb = a_seq<kUpp>(i, 0, 0, mh);
                const uint32_t nper = static_cast<uint32_t>(mh * kUpp);
                const uint32_t first = (slot + static_cast<uint32_t>(p.n_a) - jb % static_cast<uint32_t>(p.n_a)) %
                                       static_cast<uint32_t>(p.n_a);
                if (first >= nper) continue;
                const int st = i % p.n_w;
                if (!warp_wait(smem_u32(&ctl->w_full[st]), static_cast<uint32_t>(i / p.n_w) & 1u, p, ctl,
                               FAULT_GEMV_WAIT_COPY))
                    break;
                bool ok = true;
                for (uint32_t o = first; o < nper; o += static_cast<uint32_t>(p.n_a)) {
                    const uint32_t j = jb + o;
                    const int h = static_cast<int>(o) / kUpp, qq = static_cast<int>(o) % kUpp;
                    // 128-byte box rows, swizzled in 16-byte chunks (chunk c of row r at c ^ (r % 8)),
                    // so a warp's 16-byte reads hit every bank once.  Pair qq of the row is chunks
                    // [4 qq, 4 qq + 4) with two paths, the whole row with three.
                    const int brow = h * kRows + q4 * 32 + lane;
                    const uint8_t *src = wring + st * p.w_bytes + brow * 128;
                    constexpr int kChunks = 8 / kUpp;
                    uint32_t wd[4 * kChunks];
#pragma unroll
                    for (int c = 0; c < kChunks; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(src + 16 * ((qq * kChunks + c) ^ (brow & 7)));
                        wd[4 * c] = v.x; wd[4 * c + 1] = v.y; wd[4 * c + 2] = v.z; wd[4 * c + 3] = v.w;
                    }
                    if (!warp_wait(smem_u32(&ctl->a_empty[slot]), ((j / p.n_a) & 1u) ^ 1u, p, ctl, FAULT_GEMV_WAIT_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < kP; ++k) {
                        uint32_t v[32];
#pragma unroll
                        for (int g = 0; g < kUnitGroups; ++g) {
                            const uint32_t w = wd[g * Geometry<kP>::kGroupWords + k];
                            v[4 * g + 0] = ((w << 3) & 0x88888888u) | 0x22222222u;
                            v[4 * g + 1] = ((w << 2) & 0x88888888u) | 0x22222222u;
                            v[4 * g + 2] = ((w << 1) & 0x88888888u) | 0x22222222u;
                            v[4 * g + 3] = (w & 0x88888888u) | 0x22222222u;
                        }
                        tmem_st_32x32b_x32(tmem + lane_addr + a_col0 + (slot * kP + k) * 32u, v);
                    }
                    tc_wait_st();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(&ctl->a_full[slot]));
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ctl->w_empty[st]));   // this warp is done with the box
                if (!ok) break;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (warps 2..5)
        const int q4 = warp & 3;
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const int row = q4 * 32 + lane;
        const int gt = (warp - 2) * 32 + lane;       // 0..127 inside the epilogue group
        const uint32_t set_cols = static_cast<uint32_t>(mh * kP * p.acc_stride);
        // a, the scales, the workspace and y all come after the previous kernels
        asm volatile("griddepcontrol.wait;" ::: "memory");
        uint32_t gphase = 0, run = 0;
        for (int e = gt; e < p.nprob * kP * kMaxBatch; e += 128) {
            const int l = e / (kP * kMaxBatch), k = (e / kMaxBatch) % kP, beta = e % kMaxBatch;
            ctl->inv[l][k][beta] = beta < p.nb ? p.prob[l].inv[k * p.inv_stride + beta] : 0.0f;
        }
        bool ok = group_sync(ctl, gphase, lane, p);
        const int first_tile = tile_of_unit(p, u0);
        long long u = u0;
        Run r;
        while (ok && next_run(p, u, u1, r)) {
            const uint32_t ab = run % static_cast<uint32_t>(p.n_acc);
            const Prob &q = p.prob[r.prob];
            float a_row[2][kP];                        // a of this thread's rows, loaded before the wait
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int n = r.tile * tile_rows + hh * kRows + row;
#pragma unroll
                for (int k = 0; k < kP; ++k)
                    a_row[hh][k] = (hh < mh && n < q.N) ? q.a[static_cast<int64_t>(k) * q.N + n] : 0.0f;
            }
            if (!warp_wait_idle(smem_u32(&ctl->acc_full[ab]), (run / p.n_acc) & 1u, p, ctl, FAULT_GEMV_WAIT_MMA))
                break;
            tc_fence_after();
            float ypart[2][kMaxBatch];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
                for (int i = 0; i < kMaxBatch; ++i) ypart[hh][i] = 0.0f;
                if (hh >= mh) continue;
#pragma unroll
                for (int k = 0; k < kP; ++k) {
                    const uint32_t dcol = tmem + lane_addr + acc_col0 + ab * set_cols +
                                          static_cast<uint32_t>((hh * kP + k) * p.acc_stride);
                    const float ak = a_row[hh][k];
                    const float *inv = ctl->inv[r.prob][k];
#pragma unroll
                    for (int beta = 0; beta < kMaxBatch; ++beta) {
                        if (beta >= p.nb) break;
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
                        long long t = 0;
#pragma unroll
                        for (int s = Dg::kD - 1; s >= 0; --s)
                            t = 4 * t + static_cast<long long>(__float2int_rn(__uint_as_float(d[s])));
                        ypart[hh][beta] += ak * (static_cast<float>(t) * inv[beta]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->acc_empty[ab]));   // accumulators free for a later run
            ++run;
            // ---- output of the run: y, or the partial and the counter
            const int gtile = q.tile0 + r.tile;
            const int first = unit_owner(U, G, r.tile_begin);
            const int lastc = unit_owner(U, G, r.tile_begin + q.tunits - 1);
            if (first == lastc) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int n = r.tile * tile_rows + hh * kRows + row;
                    if (hh < mh && n < q.N) {
#pragma unroll
                        for (int beta = 0; beta < kMaxBatch; ++beta)
                            if (beta < p.nb) q.y[static_cast<int64_t>(beta) * q.ldy + n] = ypart[hh][beta];
                    }
                }
                continue;
            }
            const int side = (gtile == first_tile) ? 0 : 1;
            float *slot = p.partial + (static_cast<int64_t>(cta) * 2 + side) * p.nb * tile_rows;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                if (hh < mh) {
#pragma unroll
                    for (int beta = 0; beta < kMaxBatch; ++beta)
                        if (beta < p.nb) slot[beta * tile_rows + hh * kRows + row] = ypart[hh][beta];
                }
            // The group barrier orders every thread's partial stores before the counting
            // thread's fence and increment (acquire and release at GPU scope), which tell the
            // last contributor that every partial is visible.
            if (!group_sync(ctl, gphase, lane, p)) break;
            if (gt == 0) {
                __threadfence();
                int old;
                asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], 1;" : "=r"(old) : "l"(&p.tickets[gtile]) : "memory");
                ctl->last = (old == lastc - first) ? 1 : 0;
            }
            if (!group_sync(ctl, gphase, lane, p)) break;
            if (ctl->last) {
                // The partials of contributors first..lastc, added in that (column) order.
                // Loads go out eight at a time so their latencies overlap.  Every contributor
                // but the first starts its range inside this tile, so this tile is its first
                // (slot 0); the first contributor's slot is 1 when its range starts earlier.
                const int side_first = range_begin(U, G, first) < r.tile_begin ? 1 : 0;
                for (int hh = 0; hh < mh; ++hh) {
                    const int tr = hh * kRows + row;
                    const int n = r.tile * tile_rows + tr;
                    for (int beta = 0; beta < p.nb; ++beta) {
                        float sum = 0.0f;
                        for (int i0 = first; i0 <= lastc; i0 += 8) {
                            float v[8];
#pragma unroll
                            for (int dd = 0; dd < 8; ++dd) {
                                const int i = i0 + dd;
                                v[dd] = 0.0f;
                                if (i <= lastc) {
                                    const int si = i == first ? side_first : 0;
                                    v[dd] = __ldcg(p.partial + ((static_cast<int64_t>(i) * 2 + si) * p.nb + beta) * tile_rows + tr);
                                }
                            }
#pragma unroll
                            for (int dd = 0; dd < 8; ++dd)
                                if (i0 + dd <= lastc) sum += v[dd];
                        }
                        if (n < q.N) q.y[static_cast<int64_t>(beta) * q.ldy + n] = sum;
                    }
                }
                if (gt == 0) p.tickets[gtile] = 0;   // ready for the next launch over the batch
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, p.tmem_cols);
    }
}

// Workspace: the partial sums first, in a region of fixed size (the largest grid, batch and
// tile), then the fix-up counters, the row scales and the B images.  The prep kernel writes
// the counters, scales and images of every call, so the workspace needs no initialisation.
constexpr size_t kPartialBytes = static_cast<size_t>(kGemvMaxGrid) * 2 * kMaxBatch * 2 * kRows * sizeof(float);

struct Plan {
    int slice, nm, acc_stride, n_acc, n_a, mh, n_w, n_b, cpu, w_bytes, chunk_bytes, smem;
    uint32_t tmem_cols;
};

// Every A stage serves one half only: its MMA issuers then consume its fills in order (an
// issuer of the other half would wait on the phase after next, whose parity already reads as
// complete).
bool a_stages_per_half(int n_a, int mh, int upp) {
    int half[kMaxAStages];
    for (int s = 0; s < n_a; ++s) half[s] = -1;
    for (int j = 0; j < 8 * n_a * mh * upp; ++j) {
        const int s = j % n_a, h = (j / upp) % mh;
        if (half[s] >= 0 && half[s] != h) return false;
        half[s] = h;
    }
    return true;
}

// Shared- and tensor-memory layout of a launch over `slice` batch rows; false when they do
// not fit at once.  Prefers units of two 128-row halves (one 32 KiB box of signs per unit,
// and every B chunk serves both halves), then four A stages, then two accumulator sets.
bool plan_for(int P, bool f32x, int slice, Plan &L) {
    const int D = f32x ? 12 : 8;
    const int upp = P == 2 ? Geometry<2>::kBoxPairs : Geometry<3>::kBoxPairs;
    L.slice = slice;
    L.nm = (D * slice + 7) / 8 * 8;
    L.acc_stride = (L.nm + 15) / 16 * 16;
    const int a_cols = P * 32;
    const int pair_bytes = P * L.nm * 128;
    const int avail = 227 * 1024 - 1024 - static_cast<int>(sizeof(Ctl));
    for (int mh = 2; mh >= 1; --mh)
        for (int na = kMaxAStages; na >= 2; na -= 2) {
            if (!a_stages_per_half(na, mh, upp)) continue;
            for (int n_acc = 2; n_acc >= 1; --n_acc) {
                const int need = kSfCols + n_acc * mh * P * L.acc_stride + na * a_cols;
                if (need > 512) continue;
                L.mh = mh;
                L.n_a = na;
                L.n_acc = n_acc;
                L.tmem_cols = 32;
                while (static_cast<int>(L.tmem_cols) < need) L.tmem_cols *= 2;
                L.w_bytes = mh * kRows * 128;
                // B chunks of about 32 KiB (whole units), two buffers
                L.cpu = std::max(1, (32 * 1024 / pair_bytes) / upp);
                L.n_b = 2;
                L.chunk_bytes = L.cpu * upp * pair_bytes;
                L.n_w = std::min(kMaxWStages, (avail - L.n_b * L.chunk_bytes) / L.w_bytes);
                if (L.n_w < 2) continue;
                L.smem = L.n_w * L.w_bytes + L.n_b * L.chunk_bytes + static_cast<int>(sizeof(Ctl)) + 1024;
                return true;
            }
        }
    return false;
}

// The plan of a call: the largest batch slice that fits (a bigger batch runs as several main
// launches over slices of the batch rows, all with the first slice's layout).
bool plan_call(int P, bool f32x, int batch, Plan &L) {
    for (int slice = batch; slice >= 1; --slice)
        if (plan_for(P, f32x, slice, L)) return true;
    return false;
}

inline int pairs_of(int K) { return (K + kPairCols - 1) / kPairCols; }
inline size_t up1024(size_t v) { return (v + 1023) / 1024 * 1024; }

struct WsLayout {
    size_t off_tickets, off_inv, off_bmax, off_img, slice_bytes, total;
    int tiles, slices, maxblk;
};

WsLayout ws_layout(const GemvLayer *layers, int count, int P, const Plan &L, int batch) {
    WsLayout w{};
    size_t pair_rows = 0;
    for (int i = 0; i < count; ++i) {
        w.tiles += (layers[i].N + kRows * L.mh - 1) / (kRows * L.mh);
        pair_rows += static_cast<size_t>(pairs_of(layers[i].K));
    }
    w.slices = (batch + L.slice - 1) / L.slice;
    w.slice_bytes = pair_rows * P * L.nm * 128;
    w.off_tickets = kPartialBytes;
    for (int i = 0; i < count; ++i)
        w.maxblk = std::max(w.maxblk, (pairs_of(layers[i].K) * kPairCols + kPrepCols - 1) / kPrepCols);
    w.off_inv = up1024(w.off_tickets + static_cast<size_t>(w.tiles) * sizeof(int));
    w.off_bmax = up1024(w.off_inv + static_cast<size_t>(count) * P * batch * sizeof(float));
    w.off_img = up1024(w.off_bmax + static_cast<size_t>(count) * P * batch * w.maxblk * sizeof(float));
    w.total = w.off_img + w.slices * w.slice_bytes;
    return w;
}

size_t group_bytes(const GemvLayer *layers, int count, int P, bool f32x, int batch) {
    Plan L{};
    if (!plan_call(P, f32x, batch, L)) return 0;
    return ws_layout(layers, count, P, L, batch).total;
}

}  // namespace

size_t gemv_workspace_bytes(int N, int K, int P, int batch) {
    GemvLayer l{};
    l.N = N;
    l.K = K;
    return std::max(group_bytes(&l, 1, P, false, batch), group_bytes(&l, 1, P, true, batch));
}

size_t gemv_group_workspace_bytes(const GemvLayer *layers, int count, int P, bool x_bf16, int batch) {
    return group_bytes(layers, count, P, !x_bf16, batch);
}

cudaError_t launch_gemv_group(const LaunchCtx &ctx, const GemvLayer *layers, int count, int P, bool x_bf16,
                              int batch, void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug) {
    if ((P != 2 && P != 3) || count < 1 || count > kGemvMaxGroup || batch < 1 || batch > kMaxBatch)
        return cudaErrorInvalidValue;
    const bool f32x = !x_bf16;
    const int xsize = f32x ? 4 : 2;
    Plan L{};
    if (!plan_call(P, f32x, batch, L)) return cudaErrorInvalidValue;
    const WsLayout W = ws_layout(layers, count, P, L, batch);
    uint8_t *ws = static_cast<uint8_t *>(workspace);

    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    if (!encode) return cudaErrorNotSupported;
    void (*kern)(GArgs);
    void (*prep)(PrepArgs);
    void (*bmax)(PrepArgs);
    if (P == 2) {
        kern = x_bf16 ? gemv_tc_kernel<false, 2> : gemv_tc_kernel<true, 2>;
        prep = x_bf16 ? gemv_prep_kernel<false, 2> : gemv_prep_kernel<true, 2>;
        bmax = x_bf16 ? gemv_blockmax_kernel<false, 2> : gemv_blockmax_kernel<true, 2>;
    } else {
        kern = x_bf16 ? gemv_tc_kernel<false, 3> : gemv_tc_kernel<true, 3>;
        prep = x_bf16 ? gemv_prep_kernel<false, 3> : gemv_prep_kernel<true, 3>;
        bmax = x_bf16 ? gemv_blockmax_kernel<false, 3> : gemv_blockmax_kernel<true, 3>;
    }
    static ContextFlags opted[4];
    // the opt-in is set once per kernel and context, to the largest size any call asks for
    if (cudaError_t e = ensure_smem_optin(ctx, kern, 227 * 1024, opted[(P - 2) * 2 + (x_bf16 ? 0 : 1)]);
        e != cudaSuccess)
        return e;

    // ---- prep: scales, B images, counters
    PrepArgs pa{};
    long long prep_blocks = 0;
    {
        long long pair_off = 0;
        for (int i = 0; i < count; ++i) {
            const GemvLayer &l = layers[i];
            PrepLayer &q = pa.layer[i];
            q.x = l.x;
            q.b = l.b;
            q.K = l.K;
            q.ldx = l.ldx;
            q.pairs = pairs_of(l.K);
            q.blocks = (q.pairs * kPairCols + kPrepCols - 1) / kPrepCols;
            q.img_off = pair_off * P * L.nm * 128;
            q.vec = (reinterpret_cast<uintptr_t>(l.x) % 16 == 0) && ((static_cast<int64_t>(l.ldx) * xsize) % 16 == 0) &&
                    (reinterpret_cast<uintptr_t>(l.b) % 16 == 0) && ((static_cast<int64_t>(l.K) * 4) % 16 == 0);
            pair_off += q.pairs;
            prep_blocks += static_cast<long long>(q.blocks) * batch;
        }
        pa.img = ws + W.off_img;
        pa.inv = reinterpret_cast<float *>(ws + W.off_inv);
        pa.bmax = reinterpret_cast<float *>(ws + W.off_bmax);
        pa.maxblk = W.maxblk;
        pa.tickets = reinterpret_cast<int *>(ws + W.off_tickets);
        pa.slice_bytes = static_cast<long long>(W.slice_bytes);
        pa.ntickets = W.tiles;
        pa.nprob = count;
        pa.batch = batch;
        pa.slice = L.slice;
        pa.nm = L.nm;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(prep_blocks));
        cfg.blockDim = dim3(kPrepThreads);
        cfg.stream = ctx.stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaError_t e = cudaLaunchKernelEx(&cfg, bmax, pa); e != cudaSuccess) return e;
        if (cudaError_t e = cudaLaunchKernelEx(&cfg, prep, pa); e != cudaSuccess) return e;
    }

    // ---- main
    GArgs args{};
    const int GW = P == 2 ? 2 : 4;
    const int upp = P == 2 ? Geometry<2>::kBoxPairs : Geometry<3>::kBoxPairs;
    long long units = 0;
    int tiles = 0;
    for (int i = 0; i < count; ++i) {
        const GemvLayer &l = layers[i];
        const int words_per_row = static_cast<int>(padded_cols(l.K) / 32) * GW;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(words_per_row), static_cast<cuuint64_t>(l.N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(words_per_row) * 4};
        cuuint32_t box[2] = {32u, static_cast<cuuint32_t>(kRows * L.mh)};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&args.tmap[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(l.packed), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
        Prob &q = args.prob[i];
        q.a = l.a;
        q.N = l.N;
        q.ldy = l.ldy;
        q.tiles = (l.N + kRows * L.mh - 1) / (kRows * L.mh);
        q.pairs = pairs_of(l.K);
        q.tunits = (q.pairs + upp - 1) / upp;
        q.unit0 = units;
        q.tile0 = tiles;
        units += static_cast<long long>(q.tiles) * q.tunits;
        tiles += q.tiles;
    }
    args.partial = reinterpret_cast<float *>(ws);
    args.tickets = reinterpret_cast<int *>(ws + W.off_tickets);
    args.fault = fault_word;
    args.timeout_ns = timeout_ns;
    args.units = units;
    args.nprob = count;
    args.nm = L.nm;
    args.acc_stride = L.acc_stride;
    args.n_acc = L.n_acc;
    args.mh = L.mh;
    args.n_a = L.n_a;
    args.n_w = L.n_w;
    args.n_b = L.n_b;
    args.cpu = L.cpu;
    args.inv_stride = batch;
    args.tmem_cols = L.tmem_cols;
    args.w_bytes = L.w_bytes;
    args.chunk_bytes = L.chunk_bytes;
    const int grid = static_cast<int>(std::min<long long>(units, std::min(ctx.num_sms, kGemvMaxGrid)));

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(L.smem);
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    for (int s = 0; s < W.slices; ++s) {
        const int b0 = s * L.slice;
        args.nb = std::min(L.slice, batch - b0);
        args.debug = s == 0 ? debug : 0;
        for (int i = 0; i < count; ++i) {
            const GemvLayer &l = layers[i];
            Prob &q = args.prob[i];
            q.y = l.y + static_cast<int64_t>(b0) * l.ldy;
            q.inv = reinterpret_cast<const float *>(ws + W.off_inv) + static_cast<int64_t>(i) * P * batch + b0;
            q.img = ws + W.off_img + s * W.slice_bytes + pa.layer[i].img_off;
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
