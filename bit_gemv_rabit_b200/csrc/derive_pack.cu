// derive_pack.cu -- coupled forward derivation of the two sign planes and their packing.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.2 "The Coupled Forward Pass", steps 1-3 (S1 = sign(W), R1 = W - a1 (.) S1 (.) b1,
// S2 = sign(R1)), packed as in Appendix E.1 "Weight Packing" (32 columns per uint32,
// -1 -> bit 1, the two paths' words of a 32-column group side by side as one uint2), in the
// RABIT_LAYOUT_V2 arrangement declared in include/rabit.h.
//
// HBM-bound: W is streamed once (4 or 2 bytes per weight), 2 bits per weight are written.
// A warp owns one 1024-column chunk (32 groups) and walks rows: it keeps the chunk's b
// values in registers, and in step i lane l reads column 32*(w0+i) + l of the row (128
// contiguous bytes per warp load for fp32 W), forms both signs, and __ballot_sync turns the
// 32 lanes' signs into one packed word, so the bit order (column j -> bit j % 32) falls out
// of the lane order.  Lane 0 parks the word pair of step i in shared memory, and the warp
// then stores the row's 32 uint2 groups with one coalesced 256-byte store.  Chunks wholly
// inside the row skip the column bound checks.  R1 is never stored.
#include <algorithm>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kDeriveThreads = 256;

template <bool kBf16>
__device__ __forceinline__ float load_w(const void *W, int64_t idx) {
    if constexpr (kBf16) {
        const unsigned short bits = __ldg(reinterpret_cast<const unsigned short *>(W) + idx);
        return __uint_as_float(static_cast<uint32_t>(bits) << 16);  // exact widening
    } else {
        return __ldg(reinterpret_cast<const float *>(W) + idx);
    }
}

// Signs of 32 columns (one per lane) of row n for step i of a task; the ballots make the two
// packed words, and lane 0 parks them in the warp's shared slot i.
template <bool kFull>
__device__ __forceinline__ void derive_step(float w, float b1, float a1, bool ok, int i, uint2 *slots, int lane) {
    const bool neg1 = w < 0.0f;                                  // S1 = sign(W)
    // R1 = W - a1*S1*b1 with a single rounding: the sign of R1 is exact.
    const float r1 = fmaf(neg1 ? a1 : -a1, b1, w);
    const bool neg2 = r1 < 0.0f;                                 // S2 = sign(R1)
    const uint32_t s1w = __ballot_sync(0xffffffffu, kFull ? neg1 : (ok && neg1));
    const uint32_t s2w = __ballot_sync(0xffffffffu, kFull ? neg2 : (ok && neg2));
    if (lane == 0) slots[i] = make_uint2(s1w, s2w);
}

template <bool kBf16>
__global__ void __launch_bounds__(kDeriveThreads)
derive_pack_kernel(const void *__restrict__ W, int N, int K, int ldw,
                   const float *__restrict__ a, const float *__restrict__ b,
                   uint2 *__restrict__ packed, int Wr) {
    __shared__ uint2 slot_buf[kDeriveThreads / 32][32];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    const int lane = threadIdx.x & 31;
    uint2 *slots = slot_buf[threadIdx.x >> 5];
    const int chunks = (Wr + 31) / 32;  // 1024-column chunks per row
    // The launch makes the warp count a multiple of `chunks`, so a warp keeps one chunk (and
    // its b values) for all the rows it visits.
    const int warp_global = (blockIdx.x * kDeriveThreads + threadIdx.x) >> 5;
    const int warps = (gridDim.x * kDeriveThreads) >> 5;
    const int chunk = warp_global % chunks;
    const int w0 = chunk * 32;
    const bool full = (w0 + 32) * 32 <= K;   // every column of the chunk is inside the row

    float b1[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int j = (w0 + i) * 32 + lane;
        b1[i] = j < K ? __ldg(b + j) : 0.0f;
    }
    for (int n = warp_global / chunks; n < N; n += warps / chunks) {
        const float a1 = __ldg(a + n);
        const int64_t row = static_cast<int64_t>(n) * ldw;
        float w[32];
        if (full) {
#pragma unroll
            for (int i = 0; i < 32; ++i) w[i] = load_w<kBf16>(W, row + (w0 + i) * 32 + lane);
#pragma unroll
            for (int i = 0; i < 32; ++i) derive_step<true>(w[i], b1[i], a1, true, i, slots, lane);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int j = (w0 + i) * 32 + lane;
                w[i] = j < K ? load_w<kBf16>(W, row + j) : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
                derive_step<false>(w[i], b1[i], a1, (w0 + i) * 32 + lane < K, i, slots, lane);
        }
        __syncwarp();
        if (w0 + lane < Wr) packed[static_cast<int64_t>(n) * Wr + w0 + lane] = slots[lane];
        __syncwarp();
    }
}

// Three paths (the residual rule once more: S3 = sign(W - W_hat_1 - W_hat_2)), groups of
// three words plus a zero padding word.  The second residual needs the first one's value,
// not only its sign, so both are formed in binary64 exactly as the definition reads: each
// product a*s*b of two fp32 numbers is exact in binary64 and each subtraction rounds once.
template <bool kBf16>
__global__ void __launch_bounds__(kDeriveThreads)
derive_pack3_kernel(const void *__restrict__ W, int N, int K, int ldw,
                    const float *__restrict__ a, const float *__restrict__ b,
                    uint4 *__restrict__ packed, int Wr) {
    __shared__ uint4 slot_buf[kDeriveThreads / 32][32];
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    const int lane = threadIdx.x & 31;
    uint4 *slots = slot_buf[threadIdx.x >> 5];
    const int chunks = (Wr + 31) / 32;
    const int warp_global = (blockIdx.x * kDeriveThreads + threadIdx.x) >> 5;
    const int warps = (gridDim.x * kDeriveThreads) >> 5;
    const int chunk = warp_global % chunks;
    const int w0 = chunk * 32;
    for (int n = warp_global / chunks; n < N; n += warps / chunks) {
        const double a1 = __ldg(a + n), a2 = __ldg(a + N + n);   // S3 needs no third scale
        const int64_t row = static_cast<int64_t>(n) * ldw;
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
            const int j = (w0 + i) * 32 + lane;
            const bool ok = j < K;
            const double w = ok ? static_cast<double>(load_w<kBf16>(W, row + j)) : 0.0;
            const double b1 = ok ? __ldg(b + j) : 0.0, b2 = ok ? __ldg(b + K + j) : 0.0;
            const bool neg1 = w < 0.0;
            const double r1 = __dsub_rn(w, __dmul_rn(__dmul_rn(a1, neg1 ? -1.0 : 1.0), b1));
            const bool neg2 = r1 < 0.0;
            const double r2 = __dsub_rn(r1, __dmul_rn(__dmul_rn(a2, neg2 ? -1.0 : 1.0), b2));
            const bool neg3 = r2 < 0.0;
            const uint32_t s1w = __ballot_sync(0xffffffffu, ok && neg1);
            const uint32_t s2w = __ballot_sync(0xffffffffu, ok && neg2);
            const uint32_t s3w = __ballot_sync(0xffffffffu, ok && neg3);
            if (lane == 0) slots[i] = make_uint4(s1w, s2w, s3w, 0u);
        }
        __syncwarp();
        if (w0 + lane < Wr) packed[static_cast<int64_t>(n) * Wr + w0 + lane] = slots[lane];
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_derive_pack(const LaunchCtx &ctx, const void *W, bool w_bf16, int N, int K,
                               int ldw, int P, const float *a, const float *b, uint32_t *packed) {
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    // Warps: a multiple of the chunk count (so each warp keeps one chunk), enough for every
    // (row, chunk) task when there are few, at most 8 CTAs per SM.
    const int chunks = (Wr + 31) / 32;
    const int64_t warps_per_block = kDeriveThreads / 32;
    const int64_t want = std::min<int64_t>(static_cast<int64_t>(N) * chunks,
                                           static_cast<int64_t>(ctx.num_sms) * 8 * warps_per_block);
    int64_t warps = std::max<int64_t>(chunks, (want / chunks) * chunks);
    // round up to whole blocks while keeping a multiple of chunks
    while (warps % warps_per_block != 0) warps += chunks;
    const int64_t blocks = warps / warps_per_block;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(kDeriveThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (P == 3) {
        uint4 *out3 = reinterpret_cast<uint4 *>(packed);
        if (w_bf16)
            return cudaLaunchKernelEx(&cfg, derive_pack3_kernel<true>, W, N, K, ldw, a, b, out3, Wr);
        return cudaLaunchKernelEx(&cfg, derive_pack3_kernel<false>, W, N, K, ldw, a, b, out3, Wr);
    }
    uint2 *out = reinterpret_cast<uint2 *>(packed);
    if (w_bf16)
        return cudaLaunchKernelEx(&cfg, derive_pack_kernel<true>, W, N, K, ldw, a, b, out, Wr);
    return cudaLaunchKernelEx(&cfg, derive_pack_kernel<false>, W, N, K, ldw, a, b, out, Wr);
}

}  // namespace rabit
