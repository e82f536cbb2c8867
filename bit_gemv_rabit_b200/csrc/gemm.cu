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

struct GemmArgs {
    const uint32_t *packed;
    const float *a;
    float *y;
    uint32_t *fault;
    uint64_t timeout_ns;
    int N, K, M, Kp, ldy;
    int tiles_m, num_tiles;
    int debug;
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

template <int kP>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmArgs p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    SmemCtl *ctl = reinterpret_cast<SmemCtl *>(smem + kStages * kStageBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kblocks_per_path = p.Kp / kBK;
    const int nkb = kP * kblocks_per_path;
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
        prefetch_tensormap(&tmap_x);
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
            for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
                const int m0 = (tile % p.tiles_m) * kBN;
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
                    tma_load_3d(smem_u32(smem + s * kStageBytes), &tmap_x, bar, kcol, m0, path);
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
            for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++local_tile) {
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
        const int Wr = p.Kp / 32;               // 32-column groups per row
        uint32_t it = 0, local_tile = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++local_tile) {
            const int m0 = (tile % p.tiles_m) * kBN;
            const int n0 = (tile / p.tiles_m) * kBM;
            const int n = n0 + row;
            const bool row_valid = n < p.N;
            uint32_t a2[kP];
#pragma unroll
            for (int k = 0; k < kP; ++k) {
                const uint32_t h = row_valid ? half_bits(__ldg(p.a + k * p.N + n)) : 0u;
                a2[k] = h | (h << 16);
            }
            // The packed words of one 64-column block (two 32-column groups) of this row:
            // two paths: one 16-byte load {path1 w, path2 w, path1 w+1, path2 w+1};
            // three paths: two 16-byte loads {path1, path2, path3, pad} of groups w and w+1.
            struct Block { uint4 g0, g1; };
            constexpr int kGroupWords = kP == 2 ? 2 : 4;     // words per 32-column group
            const uint4 *row_ptr = reinterpret_cast<const uint4 *>(p.packed + static_cast<int64_t>(n) * Wr * kGroupWords);
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
                        if (m < p.M) p.y[static_cast<int64_t>(m) * p.ldy + n] = __uint_as_float(acc[i]);
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

cudaError_t launch_gemm(const LaunchCtx &ctx, const uint32_t *packed, const float *a,
                        const float *b, int N, int K, int P, const uint16_t *x, int M, int ldx,
                        float *y, int ldy, void *workspace, uint32_t *fault_word,
                        uint64_t timeout_ns, int debug_flags) {
    if (P != 2 && P != 3) return cudaErrorInvalidValue;
    const int Kp = static_cast<int>(padded_cols(K));

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;

    // 1. Tensor map over the workspace viewed as [P][M][Kp] fp16.
    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(tensor_map_encode_entry());
    if (!encode) return cudaErrorNotSupported;
    CUtensorMap tmap;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(Kp), static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(P)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(Kp) * 2, static_cast<cuuint64_t>(M) * Kp * 2};
    cuuint32_t box[3] = {kBK, kBN, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, workspace, dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;

    // 2. Shared-memory opt-in.  Steps 1 and 2 can fail, so they come before anything is
    //    enqueued: a call that returns an error has put no work on the stream.
    void (*kern)(CUtensorMap, GemmArgs) = P == 2 ? gemm_kernel<2> : gemm_kernel<3>;
    static ContextFlags opted[2];
    if (cudaError_t e = ensure_smem_optin(ctx, kern, kSmemBytes, opted[P - 2]); e != cudaSuccess) return e;

    // 3. X'_k = fp16(x (.) b_k), permuted within 32-column groups.
    {
        const int64_t total = static_cast<int64_t>(P) * M * (Kp / 2);
        int64_t blocks = (total + 255) / 256;
        if (blocks > static_cast<int64_t>(ctx.num_sms) * 16) blocks = static_cast<int64_t>(ctx.num_sms) * 16;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(blocks));
        cfg.blockDim = dim3(256);
        cfg.stream = ctx.stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, prep_x_kernel, x, ldx, b, K, Kp, M, P,
                                           static_cast<uint32_t *>(workspace));
        if (e != cudaSuccess) return e;
    }

    // 4. Persistent tcgen05 kernel.
    GemmArgs args;
    args.packed = packed;
    args.a = a;
    args.y = y;
    args.fault = fault_word;
    args.timeout_ns = timeout_ns;
    args.N = N;
    args.K = K;
    args.M = M;
    args.Kp = Kp;
    args.ldy = ldy;
    args.tiles_m = (M + kBN - 1) / kBN;
    const int tiles_n = (N + kBM - 1) / kBM;
    args.num_tiles = args.tiles_m * tiles_n;
    args.debug = debug_flags;

    int grid = args.num_tiles < ctx.num_sms ? args.num_tiles : ctx.num_sms;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, args);
}

}  // namespace rabit
