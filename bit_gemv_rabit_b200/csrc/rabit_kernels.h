// rabit_kernels.h -- host-side launchers shared between the librabit translation units.
// Each launcher assumes its arguments were validated by the C ABI layer (rabit_abi.cu).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "ctx_cache.h"

namespace rabit {

// Launch configuration shared by every kernel launch: programmatic dependent launch lets a
// kernel's prologue overlap the tail of the previous kernel on the same stream.  `device`
// and `context` identify where the launch goes (context = cuCtxGetId of the current
// context, 0 if it could not be read): per-context settings are keyed on them.
struct LaunchCtx {
    cudaStream_t stream;
    int num_sms;
    bool pdl;
    int device;
    uint64_t context;
};

// Raises `kern`'s dynamic shared-memory limit to `bytes` in the current context the first
// time a launch there needs it (the attribute belongs to the context the module is loaded
// in, so a new context after a device reset gets it again).
template <typename Kern>
inline cudaError_t ensure_smem_optin(const LaunchCtx &ctx, Kern kern, int bytes, ContextFlags &seen) {
    if (seen.done(ctx.device, ctx.context)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) seen.mark(ctx.device, ctx.context);
    return e;
}

inline int64_t padded_cols(int K) { return ((static_cast<int64_t>(K) + 127) / 128) * 128; }

// P = 2 or 3 paths.
cudaError_t launch_derive_pack(const LaunchCtx &ctx, const void *W, bool w_bf16, int N, int K,
                               int ldw, int P, const float *a, const float *b, uint32_t *packed);

cudaError_t launch_gemv(const LaunchCtx &ctx, const uint32_t *packed, const float *a,
                        const float *b, int N, int K, int P, const void *x, bool x_bf16, int batch,
                        int ldx, float *y, int ldy, uint32_t *fault_word, uint64_t timeout_ns);

// Tensor-core decode (gemv_tc.cu): a prep kernel (row scales, the B operand images, the
// fix-up counters) and the main kernel.  The workspace holds the partial sums of the row tiles
// shared between CTAs, one counter per 128-row tile, the row scales and the B images; every
// call rewrites what it uses, so it needs no initialisation.
constexpr int kGemvMaxGrid = 160;
constexpr int kGemvMaxGroup = 8;   // layers one grouped launch may take
struct GemvLayer {
    const uint32_t *packed;
    const float *a, *b;
    int N, K;
    const void *x;
    int ldx;
    float *y;
    int ldy;
};
// Enough for either activation type.
size_t gemv_workspace_bytes(int N, int K, int P, int batch);
size_t gemv_group_workspace_bytes(const GemvLayer *layers, int count, int P, bool x_bf16, int batch);
cudaError_t launch_gemv_group(const LaunchCtx &ctx, const GemvLayer *layers, int count, int P, bool x_bf16,
                              int batch, void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug);
cudaError_t launch_gemv_tc(const LaunchCtx &ctx, const uint32_t *packed, const float *a, const float *b,
                           int N, int K, int P, const void *x, bool x_bf16, int batch, int ldx, float *y,
                           int ldy, void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug);

// Packed sign planes of W^T (K x N) from those of W (transpose_pack.cu).
cudaError_t launch_transpose_pack(const LaunchCtx &ctx, const uint32_t *packed, int N, int K, int P,
                                  uint32_t *packed_t);

// The driver's cuTensorMapEncodeTiled (as a PFN_cuTensorMapEncodeTiled_v12000), or null.
void *tensor_map_encode_entry();

size_t scale_grads_workspace_bytes(int N, int K, int P);
cudaError_t launch_scale_grads(const LaunchCtx &ctx, const float *G, int ldg, const uint32_t *packed,
                               const float *a, const float *b, int N, int K, int P, float *grad_a,
                               float *grad_b, void *workspace, uint32_t *fault_word, uint64_t timeout_ns,
                               int debug = 0);

// Iterative Residual SVID initialisation (svid.cu).
size_t svid_workspace_bytes(int N, int K, int P);
cudaError_t launch_svid_init(const LaunchCtx &ctx, const float *W, int ldw, int N, int K, int P, int T,
                             int power_iters, float power_tol, const float *s_in, const float *s_out,
                             float alpha_in, float alpha_out, float *a, float *b, uint32_t *packed,
                             void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug = 0);

size_t gemm_workspace_bytes(int N, int K, int P, int M);
// Up to 4 layers with the same token count in one launch (gemm.cu); x of each layer is bf16.
size_t gemm_group_workspace_bytes(const GemvLayer *layers, int count, int P, int M);
cudaError_t launch_gemm_group(const LaunchCtx &ctx, const GemvLayer *layers, int count, int P, int M,
                              void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug_flags);
// Device address (in the launch's context) and size of the library's fixed GEMM scratch
// buffer (rabit_gemm_noalloc).
cudaError_t gemm_noalloc_scratch(const LaunchCtx &ctx, void **ptr, size_t *bytes);
cudaError_t launch_gemm(const LaunchCtx &ctx, const uint32_t *packed, const float *a,
                        const float *b, int N, int K, int P, const uint16_t *x, int M, int ldx,
                        float *y, int ldy, void *workspace, uint32_t *fault_word,
                        uint64_t timeout_ns, int debug_flags);

}  // namespace rabit
