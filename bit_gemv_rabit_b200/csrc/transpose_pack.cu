// transpose_pack.cu -- the packed sign planes of W^T from those of W (input gradient).
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs", sec. 4.1:
// for y = W_hat x with W_hat = sum_k a_k (.) S_k (.) b_k, the input gradient is
// dL/dx = W_hat^T dY, and W_hat^T = sum_k b_k (.) S_k^T (.) a_k has the stacked form of the
// forward layer with the roles of a and b exchanged.  Its sign planes S_k^T, packed as
// Appendix E.1 "Weight Packing" packs a K x N matrix (RABIT_LAYOUT_V2), let the forward GEMM
// compute the input gradient.  The signs do not change during the backward pass, so one
// transpose serves every micro-batch of a step.
//
// A CTA transposes a tile of 256 rows x 256 columns of every plane.  The tile's words come
// into shared memory with coalesced loads (8 groups x G words of each input row, in a row
// padded by one word so column reads are free of bank conflicts), each warp turns 32 x 32-bit
// blocks around (lane l holds input row l's word and ends with output row l's), and the
// transposed tile leaves with coalesced stores.  The block transpose is the recursive one:
// for j = 16, 8, 4, 2, 1, lanes l and l ^ j exchange words and swap the off-diagonal j x j
// sub-blocks of every 2j x 2j block (five shuffles instead of 32 ballots).
#include <cstdint>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kTile = 256;              // rows and columns of a CTA tile
constexpr int kTileGroups = kTile / 32; // 32-bit blocks per tile side
constexpr int kThreads = 256;

template <int G>   // words per 32-column group: 2 (two paths) or 4 (three paths and a zero word)
__global__ void __launch_bounds__(kThreads)
transpose_pack_kernel(const uint32_t *__restrict__ in, int N, int K, int wr_in, int P,
                      uint32_t *__restrict__ out, int wr_out) {
    constexpr int kRow = kTileGroups * G + 1;          // padded words per staged row
    extern __shared__ uint32_t smem[];
    uint32_t *tin = smem;                              // [kTile][kRow]: input rows n0 ..
    uint32_t *tout = smem + kTile * kRow;              // [kTile][kRow]: output rows j0 ..
    const int j0 = blockIdx.x * kTile, n0 = blockIdx.y * kTile;
    const int win = wr_in * G, wout = wr_out * G;      // words per input / output row
    // The input planes may come from the previous kernel on the stream (derive_pack).
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    for (int e = threadIdx.x; e < kTile * kTileGroups * G; e += kThreads) {
        const int r = e / (kTileGroups * G), c = e - r * (kTileGroups * G);
        const int n = n0 + r, w = (j0 / 32) * G + c;
        tin[r * kRow + c] = (n < N && w < win) ? __ldg(in + static_cast<int64_t>(n) * win + w) : 0u;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t = warp; t < kTileGroups * kTileGroups * G; t += kThreads / 32) {
        const int k = t % G, blk = t / G, bi = blk / kTileGroups, bj = blk - bi * kTileGroups;
        uint32_t mine = 0u;
        if (k < P) {                                   // (the padding word of a group stays 0)
            mine = tin[(32 * bi + lane) * kRow + bj * G + k];
            // bit c of row r -> bit r of row c.  low: the columns c with (c & j) == 0.
            constexpr uint32_t kLow[5] = {0x0000FFFFu, 0x00FF00FFu, 0x0F0F0F0Fu, 0x33333333u, 0x55555555u};
#pragma unroll
            for (int step = 0; step < 5; ++step) {
                const int j = 16 >> step;
                const uint32_t low = kLow[step], high = ~low;
                const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, j);
                mine = (lane & j) ? (((other & high) >> j) | (mine & high))     // lower row of the pair
                                  : ((mine & low) | ((other & low) << j));      // upper row of the pair
            }
        }
        // output row j0 + 32 bj + lane, output group n0 / 32 + bi, path k
        tout[(32 * bj + lane) * kRow + bi * G + k] = mine;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kTile * kTileGroups * G; e += kThreads) {
        const int r = e / (kTileGroups * G), c = e - r * (kTileGroups * G);
        const int j = j0 + r, w = (n0 / 32) * G + c;
        if (j < K && w < wout) out[static_cast<int64_t>(j) * wout + w] = tout[r * kRow + c];
    }
}

}  // namespace

cudaError_t launch_transpose_pack(const LaunchCtx &ctx, const uint32_t *packed, int N, int K, int P,
                                  uint32_t *packed_t) {
    if (P != 2 && P != 3) return cudaErrorInvalidValue;
    const int G = P == 2 ? 2 : 4;
    const int wr_in = static_cast<int>(padded_cols(K) / 32);    // groups per row of W
    const int wr_out = static_cast<int>(padded_cols(N) / 32);   // groups per row of W^T
    void (*kern)(const uint32_t *, int, int, int, int, uint32_t *, int) =
        P == 2 ? transpose_pack_kernel<2> : transpose_pack_kernel<4>;
    const int smem = 2 * kTile * (kTileGroups * G + 1) * static_cast<int>(sizeof(uint32_t));
    static ContextFlags opted[2];
    if (cudaError_t e = ensure_smem_optin(ctx, kern, smem, opted[P == 2 ? 0 : 1]); e != cudaSuccess) return e;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    // output rows j cover K rounded up to whole tiles; output groups cover the padded N
    cfg.gridDim = dim3(static_cast<unsigned>((K + kTile - 1) / kTile),
                       static_cast<unsigned>((wr_out * 32 + kTile - 1) / kTile));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, packed, N, K, wr_in, P, packed_t, wr_out);
}

}  // namespace rabit
