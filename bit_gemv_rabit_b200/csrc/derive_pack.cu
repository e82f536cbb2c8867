// derive_pack.cu -- coupled forward derivation of the two sign planes and their packing.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs",
// sec. 4.2 "The Coupled Forward Pass", steps 1-3 (S1 = sign(W), R1 = W - a1 (.) S1 (.) b1,
// S2 = sign(R1)), packed as in Appendix E.1 "Weight Packing" (32 columns per uint32,
// -1 -> bit 1, the two paths' words of a 32-column group side by side as one uint2), in the
// RABIT_LAYOUT_V2 arrangement declared in include/rabit.h.
//
// HBM-bound: W is streamed once (4 or 2 bytes per weight), 2 bits per weight are written.
// One warp handles one row and 32 consecutive 32-column groups of it (1024 columns): in
// step i lane l reads column 32*(w0+i) + l (128 contiguous bytes per warp load for fp32 W),
// forms both signs, and __ballot_sync turns the 32 lanes' signs into one packed word, so the
// bit order (column j -> bit j % 32) falls out of the lane order.  Lane i keeps the word
// pair of step i, and the warp then stores its 32 uint2 groups with one coalesced 256-byte
// store.  R1 is never stored.
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

template <bool kBf16>
__global__ void __launch_bounds__(kDeriveThreads)
derive_pack_kernel(const void *__restrict__ W, int N, int K, int ldw,
                   const float *__restrict__ a, const float *__restrict__ b,
                   uint2 *__restrict__ packed, int Wr) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    const int lane = threadIdx.x & 31;
    const int chunks = (Wr + 31) / 32;  // 1024-column chunks per row
    const int64_t num_tasks = static_cast<int64_t>(N) * chunks;
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * kDeriveThreads + threadIdx.x) >> 5;
    const int64_t warp_stride = (static_cast<int64_t>(gridDim.x) * kDeriveThreads) >> 5;

    for (int64_t task = warp_global; task < num_tasks; task += warp_stride) {
        const int n = static_cast<int>(task / chunks);
        const int w0 = static_cast<int>(task % chunks) * 32;
        const float a1 = __ldg(a + n);
        const int64_t row = static_cast<int64_t>(n) * ldw;

        float w[32], b1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int j = (w0 + i) * 32 + lane;
            const bool ok = j < K;
            w[i] = ok ? load_w<kBf16>(W, row + j) : 0.0f;
            b1[i] = ok ? __ldg(b + j) : 0.0f;
        }
        uint32_t mine1 = 0, mine2 = 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int j = (w0 + i) * 32 + lane;
            const bool ok = j < K;
            const bool neg1 = w[i] < 0.0f;                          // S1 = sign(W)
            // R1 = W - a1*S1*b1 with a single rounding: the sign of R1 is exact.
            const float r1 = fmaf(neg1 ? a1 : -a1, b1[i], w[i]);
            const bool neg2 = r1 < 0.0f;                            // S2 = sign(R1)
            const uint32_t s1w = __ballot_sync(0xffffffffu, ok && neg1);
            const uint32_t s2w = __ballot_sync(0xffffffffu, ok && neg2);
            if (lane == i) {
                mine1 = s1w;
                mine2 = s2w;
            }
        }
        if (w0 + lane < Wr)
            packed[static_cast<int64_t>(n) * Wr + w0 + lane] = make_uint2(mine1, mine2);
    }
}

}  // namespace

cudaError_t launch_derive_pack(const LaunchCtx &ctx, const void *W, bool w_bf16, int N, int K,
                               int ldw, const float *a, const float *b, uint32_t *packed) {
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    const int64_t tasks = static_cast<int64_t>(N) * ((Wr + 31) / 32);
    const int64_t warps_per_block = kDeriveThreads / 32;
    int64_t blocks = (tasks + warps_per_block - 1) / warps_per_block;
    const int64_t max_blocks = static_cast<int64_t>(ctx.num_sms) * 8;
    if (blocks > max_blocks) blocks = max_blocks;

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
    uint2 *out = reinterpret_cast<uint2 *>(packed);
    if (w_bf16)
        return cudaLaunchKernelEx(&cfg, derive_pack_kernel<true>, W, N, K, ldw, a, b, out, Wr);
    return cudaLaunchKernelEx(&cfg, derive_pack_kernel<false>, W, N, K, ldw, a, b, out, Wr);
}

}  // namespace rabit
