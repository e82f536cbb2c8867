// gemm.cu -- prefill / QAT-forward path of the residual-binary linear layer on tcgen05.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs", sec. 4.2:
// the forward pass multiplies by the effective weight W_hat^(2) = sum_k a_k (.) S_k (.) b_k
// (sec. 4.1 stacking).  At large M this is a dense contraction, computed here as
//     y[m][n] = sum_k sum_j A_k[n][j] * X'_k[m][j],
//     A_k[n][j] = fp16(a_k[n]) * S_k[n][j]       (expanded from the packed bits)
//     X'_k[m][j] = fp16(x[m][j] * b_k[j])        (written to the caller's workspace)
// with both paths concatenated along the contraction dimension (64-column blocks of path 1
// and path 2 alternate), so one fp32 accumulator holds the whole output tile.
//
// One launch serves one layer or a group of up to four independent layers with the same
// token count (e.g. the gate and up projections of an MLP): their tiles share the persistent
// CTAs.  Tiles of a long contraction cost more, so the host deals them longest first, each
// to the least loaded CTA, and passes every CTA's list in the kernel arguments; all roles of
// a CTA walk the same list.
//
// Kernel structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: X' tiles (256 tokens x 64 columns, 128-byte swizzle) into a
//               4-stage shared-memory ring.
//   warp 1      allocates tensor memory; one lane issues tcgen05.mma (M=128 weight rows,
//               N=256 tokens, K=16) with A read from tensor memory, B from shared memory.
//   warps 2..5  expansion: thread t of the warpgroup owns TMEM lane t = weight row n0+t;
//               it loads that row's packed words (one 16-byte load covers both paths' words
//               of 64 columns) and writes fp16 +-a_k[n] pairs into the
//               stage's A columns with tcgen05.st; after the last K block of a tile the same
//               warps drain the accumulator with tcgen05.ld and store y (each store
//               instruction covers 32 consecutive n: 128 contiguous bytes).
// The expanded operand never touches shared memory; shared-memory traffic is the TMA
// writes and the tensor core's reads of X'.
//
// Contraction order inside each 32-column group: position 2c holds column c and 2c+1 holds
// column c+16 (c < 16).  One left shift then brings bits c and c+16 of a packed word to the
// fp16 sign positions 15 and 31, so a pair costs a shift and one 3-input logic op.  The
// X' writer applies the same permutation; a contraction is invariant under it.
//
// All waits are bounded (rabit_device.cuh); an expired wait aborts the CTA cleanly and sets
// a fault bit the host reads with rabit_read_fault.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>
#include <queue>
#include <vector>

#include "rabit.h"
#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kBM = 128;             // weight rows per tile (MMA M, TMEM lanes)
constexpr int kBN = 256;             // tokens per tile (MMA N)
constexpr int kBK = 64;              // contraction columns per stage (one 128 B swizzle row)
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kStageBytes = kBN * kBK * 2;  // 32 KiB of fp16
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;      // accumulator: columns [0, 256)
constexpr uint32_t kACol = 256;      // A stages: columns [256 + 32 s, 256 + 32 s + 32)
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

constexpr int kMaxGemmGroup = 4;
constexpr int kMaxGrid = 160;
constexpr int kMaxListedTiles = 6144;   // tiles a launch may list (kernel-parameter space)

struct GemmProb {
    const uint32_t *packed;
    const float *a;
    float *y;
    int N, K, Kp, ldy;
    int tiles_m;             // token tiles
    int tile0;               // the layer's first tile in the launch
};

struct GemmMaps {
    CUtensorMap x[kMaxGemmGroup];   // X' of each layer: [P][M][Kp] fp16
};

struct GemmArgs {
    GemmProb prob[kMaxGemmGroup];
    uint32_t *fault;
    uint64_t timeout_ns;
    int nprob, M, num_tiles;
    int debug;
    int listed;              // 1: CTA c takes order[begin[c] .. begin[c+1]); 0: tiles c, c + grid, ...
    uint16_t begin[kMaxGrid + 1];
    uint16_t order[kMaxListedTiles];
};

struct SmemCtl {
    uint64_t full_b[kStages];
    uint64_t full_a[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t half_bits(float v) {
    return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(v)));
}

// The CTA's i-th tile, and the layer it belongs to.
__device__ __forceinline__ int cta_tile(const GemmArgs &p, int i) {
    return p.listed ? static_cast<int>(p.order[p.begin[blockIdx.x] + i]) : static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
}
__device__ __forceinline__ int cta_tile_count(const GemmArgs &p) {
    return p.listed ? p.begin[blockIdx.x + 1] - p.begin[blockIdx.x]
                    : (p.num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
}
__device__ __forceinline__ int prob_of_tile(const GemmArgs &p, int tile) {
    int l = 0;
    while (l + 1 < p.nprob && tile >= p.prob[l + 1].tile0) ++l;
    return l;
}

template <int kP>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    SmemCtl *ctl = reinterpret_cast<SmemCtl *>(smem + kStages * kStageBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = cta_tile_count(p);
    volatile int *abort_flag = &ctl->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ctl->full_b[s]), 1);
            mbar_init(smem_u32(&ctl->full_a[s]), 4);
            mbar_init(smem_u32(&ctl->empty[s]), 1);
        }
        mbar_init(smem_u32(&ctl->acc_full), 1);
        mbar_init(smem_u32(&ctl->acc_empty), 4);
        mbar_init(smem_u32(&ctl->drain), 1);
        ctl->abort = 0;
        fence_mbarrier_init();
        for (int l = 0; l < p.nprob; ++l) prefetch_tensormap(&maps.x[l]);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctl->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    // Inputs may be produced by the previous kernel on the stream (programmatic launch).
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            uint32_t last_parity[kStages];
            bool issued[kStages];
            for (int s = 0; s < kStages; ++s) issued[s] = false;
            for (int ti = 0; ok && ti < ntiles; ++ti) {
                const int tile = cta_tile(p, ti);
                const int l = prob_of_tile(p, tile);
                const GemmProb &q = p.prob[l];
                const int m0 = ((tile - q.tile0) % q.tiles_m) * kBN;
                const int nkb = kP * (q.Kp / kBK);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&ctl->empty[s]), ph ^ 1u, abort_flag,
                                           p.timeout_ns, p.fault, FAULT_GEMM_WAIT_TMA)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = smem_u32(&ctl->full_b[s]);
                    mbar_arrive_expect_tx(bar, kStageBytes);
                    const int path = kb % kP;           // K blocks cycle through the paths
                    const int kcol = (kb / kP) * kBK;
                    tma_load_3d(smem_u32(smem + s * kStageBytes), &maps.x[l], bar, kcol, m0, path);
                    issued[s] = true;
                    last_parity[s] = ph;
                }
            }
            // Let every copy already in flight land before the CTA can exit, also when another
            // role stopped early on an expired wait (the abort flag may be raised, so drain with
            // a private flag).  These are the latest phases of their stages, complete already in
            // normal operation.
            (void)ok;
            int drain_abort = 0;
            for (int s = 0; s < kStages; ++s)
                if (issued[s])
                    mbar_wait_bounded(smem_u32(&ctl->full_b[s]), last_parity[s], &drain_abort,
                                      p.timeout_ns, p.fault, FAULT_GEMM_DRAIN);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_f16_f32(kBM, kBN);
            uint32_t it = 0, local_tile = 0;
            bool ok = true;
            bool any_issued = false;
            for (int ti = 0; ok && ti < ntiles; ++ti, ++local_tile) {
                const int nkb = kP * (p.prob[prob_of_tile(p, cta_tile(p, ti))].Kp / kBK);
                if (!mbar_wait_bounded(smem_u32(&ctl->acc_empty), (local_tile & 1u) ^ 1u, abort_flag,
                                       p.timeout_ns, p.fault, FAULT_GEMM_WAIT_EPILOGUE)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
                    if (!mbar_wait_bounded(smem_u32(&ctl->full_b[s]), ph, abort_flag, p.timeout_ns,
                                           p.fault, FAULT_GEMM_WAIT_MMA) ||
                        !mbar_wait_bounded(smem_u32(&ctl->full_a[s]), ph, abort_flag, p.timeout_ns,
                                           p.fault, FAULT_GEMM_WAIT_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_base = smem_u32(smem + s * kStageBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t bdesc = smem_desc_kmajor_sw128(b_base + kk * 32);
                        tc_mma_f16_ts(tmem + kAccCol, tmem + kACol + s * 32 + kk * 8, bdesc, idesc,
                                      (kb | kk) != 0 ? 1u : 0u);
                    }
                    any_issued = true;
                    tc_commit(smem_u32(&ctl->empty[s]));  // frees A and B stage s when done
                }
                if (!ok) break;
                tc_commit(smem_u32(&ctl->acc_full));
            }
            if (!ok && any_issued) {
                // Wait for every MMA issued so far before tensor memory is released.
                tc_commit(smem_u32(&ctl->drain));
                int drain_abort = 0;
                mbar_wait_bounded(smem_u32(&ctl->drain), 0, &drain_abort, p.timeout_ns, p.fault,
                                  FAULT_GEMM_DRAIN);
            }
        }
    } else {
        // ------------------------------------------------------------ expansion + epilogue
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int row = q * 32 + lane;          // row within the tile == TMEM lane
        const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
        uint32_t it = 0, local_tile = 0;
        bool ok = true;
        for (int ti = 0; ok && ti < ntiles; ++ti, ++local_tile) {
            const int tile = cta_tile(p, ti);
            const GemmProb &q = p.prob[prob_of_tile(p, tile)];
            const int Wr = q.Kp / 32;               // 32-column groups per row
            const int kblocks_per_path = q.Kp / kBK;
            const int nkb = kP * kblocks_per_path;
            const int m0 = ((tile - q.tile0) % q.tiles_m) * kBN;
            const int n0 = ((tile - q.tile0) / q.tiles_m) * kBM;
            const int n = n0 + row;
            const bool row_valid = n < q.N;
            uint32_t a2[kP];
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                const uint32_t h = row_valid ? half_bits(__ldg(q.a + k * q.N + n)) : 0u;
                a2[k] = h | (h << 16);
            }
            // The packed words of one 64-column block (two 32-column groups) of this row:
            // two paths: one 16-byte load {path1 w, path2 w, path1 w+1, path2 w+1};
            // three paths: two 16-byte loads {path1, path2, path3, pad} of groups w and w+1.
            struct Block { uint4 g0, g1; };
            constexpr int kGroupWords = kP == 2 ? 2 : 4;     // words per 32-column group
            const uint4 *row_ptr = reinterpret_cast<const uint4 *>(q.packed + static_cast<int64_t>(n) * Wr * kGroupWords);
            auto load_block = [&](int blk) -> Block {
                Block r{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
                if (row_valid) {
                    if constexpr (kP == 2) {
                        r.g0 = __ldg(row_ptr + blk);
                    } else {
                        r.g0 = __ldg(row_ptr + 2 * blk);
                        r.g1 = __ldg(row_ptr + 2 * blk + 1);
                    }
                }
                return r;
            };
            Block cur = load_block(0);
            Block nxt = kblocks_per_path > 1 ? load_block(1) : Block{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
                const int path = kb % kP;
                uint32_t wlo, whi;                               // columns [64 blk, +32) and [+32, +64)
                if constexpr (kP == 2) {
                    wlo = path ? cur.g0.y : cur.g0.x;
                    whi = path ? cur.g0.w : cur.g0.z;
                } else {
                    wlo = path == 0 ? cur.g0.x : (path == 1 ? cur.g0.y : cur.g0.z);
                    whi = path == 0 ? cur.g1.x : (path == 1 ? cur.g1.y : cur.g1.z);
                }
                const uint32_t amag = path == 0 ? a2[0] : (path == 1 ? a2[1] : a2[kP - 1]);
                if (path == kP - 1) {
                    cur = nxt;
                    const int nb = kb / kP + 2;
                    if (nb < kblocks_per_path) nxt = load_block(nb);
                }
                uint32_t v[32];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    v[c] = ((wlo << (15 - c)) & 0x80008000u) ^ amag;
                    v[16 + c] = ((whi << (15 - c)) & 0x80008000u) ^ amag;
                }
                if (!mbar_wait_bounded(smem_u32(&ctl->empty[s]), ph ^ 1u, abort_flag, p.timeout_ns,
                                       p.fault, FAULT_GEMM_WAIT_EXPAND)) {
                    ok = false;
                }
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                tmem_st_32x32b_x32(tmem + lane_addr + kACol + s * 32, v);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                const bool skip = (p.debug & 1) && it == 0;  // fault injection: never arrive once
                if (lane == 0 && !skip) mbar_arrive(smem_u32(&ctl->full_a[s]));
            }
            if (!ok) break;
            // Epilogue: accumulator -> registers -> y.
            if (!mbar_wait_bounded(smem_u32(&ctl->acc_full), local_tile & 1u, abort_flag,
                                   p.timeout_ns, p.fault, FAULT_GEMM_WAIT_EPILOGUE)) {
                ok = false;
            }
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                uint32_t acc[32];
                tmem_ld_32x32b_x32(tmem + lane_addr + kAccCol + c0, acc);
                tc_wait_ld();
                if (row_valid) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int m = m0 + c0 + i;
                        if (m < p.M) q.y[static_cast<int64_t>(m) * q.ldy + n] = __uint_as_float(acc[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ctl->acc_empty));
        }
    }

    asm volatile("griddepcontrol.launch_dependents;");
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// X'_k[m][32g + 2c + h] = fp16(x[m][32g + c + 16h] * b_k[32g + c + 16h]) for c < 16,
// 0 beyond K.  Layout [P][M][Kp]; one thread writes one (c, c+16) pair as a 32-bit word.
__global__ void __launch_bounds__(256)
prep_x_kernel(const uint16_t *__restrict__ x, int ldx, const float *__restrict__ b, int K,
              int Kp, int M, int P, uint32_t *__restrict__ xp) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int64_t pairs_per_row = Kp / 2;
    const int64_t total = static_cast<int64_t>(P) * M * pairs_per_row;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t pr = i % pairs_per_row;
        const int64_t rowi = i / pairs_per_row;       // k * M + m
        const int k = static_cast<int>(rowi / M);
        const int m = static_cast<int>(rowi % M);
        const int g = static_cast<int>(pr / 16), c = static_cast<int>(pr % 16);
        const int j0 = 32 * g + c, j1 = j0 + 16;
        float v0 = 0.0f, v1 = 0.0f;
        const uint16_t *xr = x + static_cast<int64_t>(m) * ldx;
        if (j0 < K) v0 = __uint_as_float(static_cast<uint32_t>(xr[j0]) << 16) * __ldg(b + k * K + j0);
        if (j1 < K) v1 = __uint_as_float(static_cast<uint32_t>(xr[j1]) << 16) * __ldg(b + k * K + j1);
        xp[i] = half_bits(v0) | (half_bits(v1) << 16);
    }
}

}  // namespace

void *tensor_map_encode_entry() {
    static void *fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = ptr;
    }
    return fn;
}

// Scratch for rabit_gemm_noalloc: a fixed buffer in the library's device image, so callers
// that may not allocate device memory can still run the GEMM.  In host code this name is
// only a host-side stand-in, never a device address: gemm_noalloc_scratch() looks up the
// device address, and that address is what the kernels receive.
static __device__ __align__(256) uint8_t g_gemm_noalloc_scratch[RABIT_GEMM_NOALLOC_SCRATCH_BYTES];

cudaError_t gemm_noalloc_scratch(const LaunchCtx &ctx, void **ptr, size_t *bytes) {
    // Looked up once per context, with the launch's device current: the symbol's address
    // belongs to the context the module was loaded in.
    static ContextCache<void *> cache;
    const int st = cache.get(ctx.device, ctx.context, [](void **out) {
        return static_cast<int>(cudaGetSymbolAddress(out, g_gemm_noalloc_scratch));
    }, ptr);
    if (st != 0) return static_cast<cudaError_t>(st);
    *bytes = sizeof(g_gemm_noalloc_scratch);
    return cudaSuccess;
}

size_t gemm_workspace_bytes(int N, int K, int P, int M) {
    (void)N;
    return static_cast<size_t>(P) * static_cast<size_t>(M) * static_cast<size_t>(padded_cols(K)) * 2;
}

namespace {
inline size_t up256(size_t v) { return (v + 255) / 256 * 256; }
}  // namespace

size_t gemm_group_workspace_bytes(const GemvLayer *layers, int count, int P, int M) {
    size_t total = 0;
    for (int i = 0; i < count; ++i) total += up256(gemm_workspace_bytes(layers[i].N, layers[i].K, P, M));
    return total;
}

cudaError_t launch_gemm_group(const LaunchCtx &ctx, const GemvLayer *layers, int count, int P, int M,
                              void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug_flags) {
    if ((P != 2 && P != 3) || count < 1 || count > kMaxGemmGroup) return cudaErrorInvalidValue;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;

    // 1. Tensor maps over each layer's part of the workspace, viewed as [P][M][Kp] fp16.
    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    if (!encode) return cudaErrorNotSupported;
    GemmMaps maps{};
    static GemmArgs args;               // large (the tile lists); filled and copied per launch
    static std::mutex args_mutex;
    std::lock_guard<std::mutex> guard(args_mutex);
    args = GemmArgs{};
    uint8_t *xp[kMaxGemmGroup];
    {
        size_t off = 0;
        int tiles = 0;
        for (int i = 0; i < count; ++i) {
            const GemvLayer &l = layers[i];
            const int Kp = static_cast<int>(padded_cols(l.K));
            xp[i] = static_cast<uint8_t *>(workspace) + off;
            off += up256(gemm_workspace_bytes(l.N, l.K, P, M));
            cuuint64_t dims[3] = {static_cast<cuuint64_t>(Kp), static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(P)};
            cuuint64_t strides[2] = {static_cast<cuuint64_t>(Kp) * 2, static_cast<cuuint64_t>(M) * Kp * 2};
            cuuint32_t box[3] = {kBK, kBN, 1};
            cuuint32_t estr[3] = {1, 1, 1};
            CUresult r = encode(&maps.x[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, xp[i], dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
            GemmProb &q = args.prob[i];
            q.packed = l.packed;
            q.a = l.a;
            q.y = l.y;
            q.N = l.N;
            q.K = l.K;
            q.Kp = Kp;
            q.ldy = l.ldy;
            q.tiles_m = (M + kBN - 1) / kBN;
            q.tile0 = tiles;
            tiles += q.tiles_m * ((l.N + kBM - 1) / kBM);
        }
        args.num_tiles = tiles;
    }
    args.nprob = count;
    args.M = M;
    args.fault = fault_word;
    args.timeout_ns = timeout_ns;
    args.debug = debug_flags;
    const int grid = std::min(args.num_tiles, std::min(ctx.num_sms, kMaxGrid));

    // 2. The tile lists: longest contraction first, each tile to the least loaded CTA (ties:
    //    the lowest CTA), so every run deals the same tiles to the same CTAs.
    args.listed = args.num_tiles <= kMaxListedTiles ? 1 : 0;
    if (args.listed) {
        std::vector<int> tiles(args.num_tiles);
        for (int t = 0; t < args.num_tiles; ++t) tiles[t] = t;
        auto cost = [&](int t) {
            int l = 0;
            while (l + 1 < count && t >= args.prob[l + 1].tile0) ++l;
            return args.prob[l].Kp;
        };
        std::stable_sort(tiles.begin(), tiles.end(), [&](int x, int y) { return cost(x) > cost(y); });
        std::vector<std::vector<int>> lists(grid);
        using Slot = std::pair<long long, int>;                       // (load, CTA)
        std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
        for (int c = 0; c < grid; ++c) heap.push({0, c});
        for (int t : tiles) {
            Slot sl = heap.top();
            heap.pop();
            lists[sl.second].push_back(t);
            heap.push({sl.first + cost(t), sl.second});
        }
        int pos = 0;
        for (int c = 0; c < grid; ++c) {
            args.begin[c] = static_cast<uint16_t>(pos);
            for (int t : lists[c]) args.order[pos++] = static_cast<uint16_t>(t);
        }
        args.begin[grid] = static_cast<uint16_t>(pos);
    }

    // 3. Shared-memory opt-in.  Steps 1 to 3 can fail, so they come before anything is
    //    enqueued: a call that returns an error has put no work on the stream.
    void (*kern)(GemmMaps, GemmArgs) = P == 2 ? gemm_kernel<2> : gemm_kernel<3>;
    static ContextFlags opted[2];
    if (cudaError_t e = ensure_smem_optin(ctx, kern, kSmemBytes, opted[P - 2]); e != cudaSuccess) return e;

    // 4. X'_k = fp16(x (.) b_k) of each layer, permuted within 32-column groups.
    for (int i = 0; i < count; ++i) {
        const GemvLayer &l = layers[i];
        const int Kp = args.prob[i].Kp;
        const int64_t total = static_cast<int64_t>(P) * M * (Kp / 2);
        int64_t blocks = (total + 255) / 256;
        if (blocks > static_cast<int64_t>(ctx.num_sms) * 16) blocks = static_cast<int64_t>(ctx.num_sms) * 16;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(blocks));
        cfg.blockDim = dim3(256);
        cfg.stream = ctx.stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, prep_x_kernel, static_cast<const uint16_t *>(l.x), l.ldx, l.b, l.K,
                                           Kp, M, P, reinterpret_cast<uint32_t *>(xp[i]));
        if (e != cudaSuccess) return e;
    }

    // 5. Persistent tcgen05 kernel.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, maps, args);
}

cudaError_t launch_gemm(const LaunchCtx &ctx, const uint32_t *packed, const float *a,
                        const float *b, int N, int K, int P, const uint16_t *x, int M, int ldx,
                        float *y, int ldy, void *workspace, uint32_t *fault_word,
                        uint64_t timeout_ns, int debug_flags) {
    GemvLayer l{packed, a, b, N, K, x, ldx, y, ldy};
    return launch_gemm_group(ctx, &l, 1, P, M, workspace, fault_word, timeout_ns, debug_flags);
}

}  // namespace rabit
