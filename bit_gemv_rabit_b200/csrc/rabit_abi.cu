// rabit_abi.cu -- the extern "C" boundary of librabit (declared in include/rabit.h).
//
// Each entry point validates every argument on the host before anything is enqueued
// (pure argument checks first, then the device checks), then calls one launcher.  Nothing
// here computes any part of the layer: all arithmetic runs in the CUDA kernels.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "rabit.h"
#include "rabit_kernels.h"

namespace {

// Per-device fault word: bit set by a kernel whose bounded wait expired.
__device__ uint32_t g_fault_word = 0;

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = rabit::kCtxCacheDevices;
struct DeviceInfo {
    std::atomic<int> state;  // 0 unknown, 1 ok (sm_100), 2 wrong arch; set last, under g_devices_mutex
    int num_sms;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_devices_mutex;
// Device address of g_fault_word, per device, for the context it was looked up in.
rabit::ContextCache<uint32_t *> g_fault_ptr;

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return RABIT_ERR_CUDA;
}

// Largest batch a single rabit_gemv call computes on the CUDA-core kernel by default.
constexpr int kGemvCudaCoreMaxBatch = 4;

bool env_flag(const char *name) {
    const char *v = std::getenv(name);
    return v && v[0] && std::strcmp(v, "0") != 0;
}

// Unique id (cuCtxGetId) of the context current on the calling thread, or 0 when there is
// none yet or the driver does not provide the calls.  The id is never reused by the driver,
// unlike the CUcontext handle, so a context created after a reset never matches an old one.
uint64_t current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext *);
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetCurrent get_current = [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        return (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess) ? reinterpret_cast<GetCurrent>(fn) : nullptr;
    }();
    static GetId get_id = [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        return (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess) ? reinterpret_cast<GetId>(fn) : nullptr;
    }();
    if (!get_current || !get_id) return 0;
    CUcontext c = nullptr;
    if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
    unsigned long long id = 0;
    if (get_id(c, &id) != CUDA_SUCCESS) return 0;
    return static_cast<uint64_t>(id);
}

// Validates the current device; fills ctx.  Returns RABIT_OK or an error status.
int device_ctx(void *stream, rabit::LaunchCtx &ctx, uint32_t **fault_ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return RABIT_ERR_ARCH;
    DeviceInfo &info = g_devices[dev];
    int state = info.state.load(std::memory_order_acquire);
    if (state == 0) {
        std::lock_guard<std::mutex> lock(g_devices_mutex);
        state = info.state.load(std::memory_order_relaxed);
        if (state == 0) {
            int major = 0, minor = 0, sms = 0;
            if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
                return cuda_fail(e);
            if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
                return cuda_fail(e);
            if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
                return cuda_fail(e);
            info.num_sms = sms;
            state = (major == 10 && minor == 0) ? 1 : 2;
            info.state.store(state, std::memory_order_release);
        }
    }
    if (state != 1 || env_flag("RABIT_TEST_FORCE_ARCH_MISMATCH")) return RABIT_ERR_ARCH;
    ctx.stream = static_cast<cudaStream_t>(stream);
    ctx.num_sms = info.num_sms;
    ctx.pdl = !(std::getenv("RABIT_PDL") && std::strcmp(std::getenv("RABIT_PDL"), "0") == 0);
    ctx.device = dev;
    ctx.context = current_context_id();
    if (fault_ptr) {
        // The lookup makes the device's primary context current if it was not yet, so the
        // context id is read again afterwards for the entry and for the launch.
        uint32_t *fp = nullptr;
        const int st = g_fault_ptr.get(dev, ctx.context, [&](uint32_t **out) {
            void *p = nullptr;
            const cudaError_t err = cudaGetSymbolAddress(&p, g_fault_word);
            *out = static_cast<uint32_t *>(p);
            if (err == cudaSuccess) ctx.context = current_context_id();
            return static_cast<int>(err);
        }, &fp);
        if (st != 0) return cuda_fail(static_cast<cudaError_t>(st));
        *fault_ptr = fp;
    }
    return RABIT_OK;
}

bool aligned(const void *p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

// Bound on every device-side wait: 2 s, far above any real wait, unless overridden.
uint64_t wait_timeout_ns() {
    uint64_t timeout_ns = 2000000000ull;
    if (const char *t = std::getenv("RABIT_WAIT_TIMEOUT_MS")) {
        const long long ms = std::atoll(t);
        if (ms > 0) timeout_ns = static_cast<uint64_t>(ms) * 1000000ull;
    }
    return timeout_ns;
}

int finish_launch(cudaError_t e) {
    if (e != cudaSuccess) return cuda_fail(e);
    return RABIT_OK;
}

}  // namespace

extern "C" {

size_t rabit_packed_words(int N, int K, int P) {
    if (N < 1 || K < 1 || P < 1) return 0;
    const size_t group = P == 2 ? 2 : (P == 1 ? 1 : 4);
    return static_cast<size_t>(N) * static_cast<size_t>(rabit::padded_cols(K) / 32) * group;
}

size_t rabit_gemm_workspace_bytes(int N, int K, int P, int M) {
    if (N < 1 || K < 1 || P < 1 || M < 1) return 0;
    return rabit::gemm_workspace_bytes(N, K, P, M);
}

int rabit_derive_pack(const void *W, int w_dtype, int N, int K, int ldw, int P, const float *a,
                      const float *b, uint32_t *packed, void *stream) {
    if (w_dtype != RABIT_F32 && w_dtype != RABIT_BF16) return RABIT_ERR_INVALID_ARG;
    if (!W || !a || !b || !packed) return RABIT_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || P < 1 || ldw < K) return RABIT_ERR_SHAPE;
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!aligned(packed, 16)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    int st = device_ctx(stream, ctx, nullptr);
    if (st != RABIT_OK) return st;
    return finish_launch(rabit::launch_derive_pack(ctx, W, w_dtype == RABIT_BF16, N, K, ldw, P, a, b, packed));
}

size_t rabit_gemv_workspace_bytes(int N, int K, int P, int batch) {
    if (N < 1 || K < 1 || P < 1 || batch < 1 || batch > 16) return 0;
    return rabit::gemv_workspace_bytes(N, K, P, batch);
}

namespace {
// Checks one layer of a decode call (rabit_gemv, rabit_gemv_grouped); RABIT_OK or an error.
int check_gemv_layer(const rabit_gemv_layer &l, int P, int x_dtype, int batch) {
    if (!l.packed || !l.a || !l.b || !l.x || !l.y) return RABIT_ERR_INVALID_ARG;
    if (l.N < 1 || l.K < 1 || l.ldx < l.K || l.ldy < l.N) return RABIT_ERR_SHAPE;
    if (!aligned(l.packed, 16)) return RABIT_ERR_ALIGNMENT;
    if (!aligned(l.x, x_dtype == RABIT_BF16 ? 2 : 4) || !aligned(l.y, 4)) return RABIT_ERR_ALIGNMENT;
    (void)P;
    (void)batch;
    return RABIT_OK;
}
}  // namespace

int rabit_gemv(const uint32_t *packed, const float *a, const float *b, int N, int K, int P,
               const void *x, int x_dtype, int batch, int ldx, float *y, int ldy, void *workspace,
               size_t workspace_bytes, void *stream) {
    if (x_dtype != RABIT_F32 && x_dtype != RABIT_BF16) return RABIT_ERR_INVALID_ARG;
    if (!packed || !a || !b || !x || !y) return RABIT_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || P < 1 || batch < 1 || batch > 16 || ldx < K || ldy < N)
        return RABIT_ERR_SHAPE;
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!aligned(packed, 16)) return RABIT_ERR_ALIGNMENT;
    if (!aligned(x, x_dtype == RABIT_BF16 ? 2 : 4) || !aligned(y, 4)) return RABIT_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < rabit::gemv_workspace_bytes(N, K, P, batch)) return RABIT_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    // Kernel choice.  A single layer at batch <= 4 goes to the CUDA-core kernel (gemv.cu): one
    // launch with a small fixed cost, which decides at these sizes.  Larger batches go to the
    // tensor-core path (gemv_tc.cu: prep kernels, then the sign stream on tcgen05), whose
    // digit-sliced MMAs take all batch rows at once.  RABIT_GEMV_KERNEL=dp2a or =tc forces one.
    bool tensor_cores = batch > kGemvCudaCoreMaxBatch;
    if (const char *which = std::getenv("RABIT_GEMV_KERNEL")) {
        if (std::strcmp(which, "dp2a") == 0) tensor_cores = false;
        if (std::strcmp(which, "tc") == 0) tensor_cores = true;
    }
    if (!tensor_cores)
        return finish_launch(rabit::launch_gemv(ctx, packed, a, b, N, K, P, x, x_dtype == RABIT_BF16,
                                                batch, ldx, y, ldy, fault, wait_timeout_ns()));
    const int debug = env_flag("RABIT_TEST_GEMV_WITHHOLD_COPY") ? 2 : 0;
    return finish_launch(rabit::launch_gemv_tc(ctx, packed, a, b, N, K, P, x, x_dtype == RABIT_BF16, batch,
                                               ldx, y, ldy, workspace, fault, wait_timeout_ns(), debug));
}

size_t rabit_gemv_grouped_workspace_bytes(const rabit_gemv_layer *layers, int count, int P, int x_dtype,
                                          int batch) {
    if (!layers || count < 1 || count > RABIT_GEMV_MAX_GROUP) return 0;
    if ((P != 2 && P != 3) || batch < 1 || batch > 16) return 0;
    if (x_dtype != RABIT_F32 && x_dtype != RABIT_BF16) return 0;
    rabit::GemvLayer g[RABIT_GEMV_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
        if (layers[i].N < 1 || layers[i].K < 1) return 0;
        g[i] = rabit::GemvLayer{layers[i].packed, layers[i].a, layers[i].b, layers[i].N, layers[i].K,
                                layers[i].x, layers[i].ldx, layers[i].y, layers[i].ldy};
    }
    return rabit::gemv_group_workspace_bytes(g, count, P, x_dtype == RABIT_BF16, batch);
}

int rabit_gemv_grouped(const rabit_gemv_layer *layers, int count, int P, int x_dtype, int batch,
                       void *workspace, size_t workspace_bytes, void *stream) {
    if (x_dtype != RABIT_F32 && x_dtype != RABIT_BF16) return RABIT_ERR_INVALID_ARG;
    if (!layers || count < 1 || count > RABIT_GEMV_MAX_GROUP) return RABIT_ERR_INVALID_ARG;
    if (P < 1 || batch < 1 || batch > 16) return RABIT_ERR_SHAPE;
    rabit::GemvLayer g[RABIT_GEMV_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
        const int st = check_gemv_layer(layers[i], P, x_dtype, batch);
        if (st != RABIT_OK) return st;
        g[i] = rabit::GemvLayer{layers[i].packed, layers[i].a, layers[i].b, layers[i].N, layers[i].K,
                                layers[i].x, layers[i].ldx, layers[i].y, layers[i].ldy};
    }
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < rabit::gemv_group_workspace_bytes(g, count, P, x_dtype == RABIT_BF16, batch))
        return RABIT_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    const int debug = env_flag("RABIT_TEST_GEMV_WITHHOLD_COPY") ? 2 : 0;
    return finish_launch(rabit::launch_gemv_group(ctx, g, count, P, x_dtype == RABIT_BF16, batch, workspace, fault,
                                                  wait_timeout_ns(), debug));
}

int rabit_gemm(const uint32_t *packed, const float *a, const float *b, int N, int K, int P,
               const uint16_t *x_bf16, int M, int ldx, float *y, int ldy, void *workspace,
               size_t workspace_bytes, void *stream) {
    if (!packed || !a || !b || !x_bf16 || !y) return RABIT_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || P < 1 || M < 1 || ldx < K || ldy < N) return RABIT_ERR_SHAPE;
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!aligned(packed, 16) || !aligned(x_bf16, 16) || (ldx % 8) != 0 || !aligned(y, 4))
        return RABIT_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < rabit::gemm_workspace_bytes(N, K, P, M))
        return RABIT_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    const uint64_t timeout_ns = wait_timeout_ns();
    const int debug = env_flag("RABIT_TEST_SKIP_ONE_ARRIVE") ? 1 : 0;
    return finish_launch(rabit::launch_gemm(ctx, packed, a, b, N, K, P, x_bf16, M, ldx, y, ldy,
                                            workspace, fault, timeout_ns, debug));
}

size_t rabit_gemm_grouped_workspace_bytes(const rabit_gemv_layer *layers, int count, int P, int M) {
    if (!layers || count < 1 || count > RABIT_GEMM_MAX_GROUP || (P != 2 && P != 3) || M < 1) return 0;
    rabit::GemvLayer g[RABIT_GEMM_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
        if (layers[i].N < 1 || layers[i].K < 1) return 0;
        g[i] = rabit::GemvLayer{layers[i].packed, layers[i].a, layers[i].b, layers[i].N, layers[i].K,
                                layers[i].x, layers[i].ldx, layers[i].y, layers[i].ldy};
    }
    return rabit::gemm_group_workspace_bytes(g, count, P, M);
}

int rabit_gemm_grouped(const rabit_gemv_layer *layers, int count, int P, int M, void *workspace,
                       size_t workspace_bytes, void *stream) {
    if (!layers || count < 1 || count > RABIT_GEMM_MAX_GROUP) return RABIT_ERR_INVALID_ARG;
    if (P < 1 || M < 1) return RABIT_ERR_SHAPE;
    rabit::GemvLayer g[RABIT_GEMM_MAX_GROUP];
    for (int i = 0; i < count; ++i) {
        const rabit_gemv_layer &l = layers[i];
        if (!l.packed || !l.a || !l.b || !l.x || !l.y) return RABIT_ERR_INVALID_ARG;
        if (l.N < 1 || l.K < 1 || l.ldx < l.K || l.ldy < l.N) return RABIT_ERR_SHAPE;
        if (!aligned(l.packed, 16) || !aligned(l.x, 16) || (l.ldx % 8) != 0 || !aligned(l.y, 4))
            return RABIT_ERR_ALIGNMENT;
        g[i] = rabit::GemvLayer{l.packed, l.a, l.b, l.N, l.K, l.x, l.ldx, l.y, l.ldy};
    }
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!workspace || workspace_bytes < rabit::gemm_group_workspace_bytes(g, count, P, M))
        return RABIT_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    const int debug = env_flag("RABIT_TEST_SKIP_ONE_ARRIVE") ? 1 : 0;
    return finish_launch(rabit::launch_gemm_group(ctx, g, count, P, M, workspace, fault, wait_timeout_ns(), debug));
}

int rabit_transpose_pack(const uint32_t *packed, int N, int K, int P, uint32_t *packed_t, void *stream) {
    if (!packed || !packed_t) return RABIT_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || P < 1) return RABIT_ERR_SHAPE;
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!aligned(packed, 16) || !aligned(packed_t, 16)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    int st = device_ctx(stream, ctx, nullptr);
    if (st != RABIT_OK) return st;
    return finish_launch(rabit::launch_transpose_pack(ctx, packed, N, K, P, packed_t));
}

// The input gradient is the forward GEMM of the transposed layer: signs S_k^T (K x N), the
// per-output scale b_k (length K) and the per-input scale a_k (length N), activations dY.
int rabit_grad_x(const uint32_t *packed_t, const float *a, const float *b, int N, int K, int P,
                 const uint16_t *dy_bf16, int M, int ldd, float *grad_x, int ldg, void *workspace,
                 size_t workspace_bytes, void *stream) {
    return rabit_gemm(packed_t, b, a, K, N, P, dy_bf16, M, ldd, grad_x, ldg, workspace, workspace_bytes, stream);
}

// For callers that may not allocate device memory: the scratch comes from the library's
// fixed buffer instead of a caller workspace (see include/rabit.h).
int rabit_gemm_noalloc(const uint32_t *packed, const float *a, const float *b, int N, int K, int P,
                       const uint16_t *x_bf16, int M, int ldx, float *y, int ldy, void *stream) {
    if (!packed || !a || !b || !x_bf16 || !y) return RABIT_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || P < 1 || M < 1 || ldx < K || ldy < N) return RABIT_ERR_SHAPE;
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!aligned(packed, 16) || !aligned(x_bf16, 16) || (ldx % 8) != 0 || !aligned(y, 4))
        return RABIT_ERR_ALIGNMENT;
    const size_t need = rabit::gemm_workspace_bytes(N, K, P, M);
    if (need > RABIT_GEMM_NOALLOC_SCRATCH_BYTES) return RABIT_ERR_WORKSPACE;
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    void *scratch = nullptr;
    size_t scratch_bytes = 0;
    cudaError_t e = rabit::gemm_noalloc_scratch(ctx, &scratch, &scratch_bytes);
    if (e != cudaSuccess) return cuda_fail(e);
    if (need > scratch_bytes) return RABIT_ERR_WORKSPACE;
    const uint64_t timeout_ns = wait_timeout_ns();
    const int debug = env_flag("RABIT_TEST_SKIP_ONE_ARRIVE") ? 1 : 0;
    return finish_launch(rabit::launch_gemm(ctx, packed, a, b, N, K, P, x_bf16, M, ldx, y, ldy,
                                            scratch, fault, timeout_ns, debug));
}

size_t rabit_scale_grads_workspace_bytes(int N, int K, int P) {
    if (N < 1 || K < 1 || P < 1) return 0;
    return rabit::scale_grads_workspace_bytes(N, K, P);
}

int rabit_scale_grads(const float *G, int ldg, const uint32_t *packed, const float *a, const float *b,
                      int N, int K, int P, float *grad_a, float *grad_b, void *workspace,
                      size_t workspace_bytes, void *stream) {
    if (!G || !packed || !a || !b || !grad_a || !grad_b) return RABIT_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || P < 1 || ldg < K) return RABIT_ERR_SHAPE;
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!aligned(packed, 16) || !aligned(G, 4) || !aligned(grad_a, 4) || !aligned(grad_b, 4))
        return RABIT_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < rabit::scale_grads_workspace_bytes(N, K, P))
        return RABIT_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    const int debug = env_flag("RABIT_TEST_SCALE_GRADS_WITHHOLD_COPY") ? 1 : 0;
    return finish_launch(rabit::launch_scale_grads(ctx, G, ldg, packed, a, b, N, K, P, grad_a, grad_b,
                                                   workspace, fault, wait_timeout_ns(), debug));
}

size_t rabit_svid_init_workspace_bytes(int N, int K, int P) {
    if (N < 1 || K < 1 || (P != 2 && P != 3)) return 0;
    return rabit::svid_workspace_bytes(N, K, P);
}

int rabit_svid_init(const float *W, int N, int K, int ldw, int P, int T, int power_iters, float power_tol,
                    const float *s_in, const float *s_out, float alpha_in, float alpha_out, float *a,
                    float *b, uint32_t *packed, void *workspace, size_t workspace_bytes, void *stream) {
    if (!W || !s_in || !s_out || !a || !b || !packed) return RABIT_ERR_INVALID_ARG;
    if (!std::isfinite(alpha_in) || !std::isfinite(alpha_out)) return RABIT_ERR_INVALID_ARG;
    if (!(power_tol >= 0.0f) || !std::isfinite(power_tol)) return RABIT_ERR_INVALID_ARG;
    if (N < 1 || K < 1 || ldw < K || T < 1 || T > RABIT_SVID_MAX_ITERS || power_iters < 1 ||
        power_iters > RABIT_SVID_MAX_ITERS)
        return RABIT_ERR_SHAPE;
    if (P != 2 && P != 3) return RABIT_ERR_UNSUPPORTED;
    if (!aligned(packed, 16) || !aligned(W, 4) || !aligned(s_in, 4) || !aligned(s_out, 4) || !aligned(a, 4) ||
        !aligned(b, 4))
        return RABIT_ERR_ALIGNMENT;
    if (!workspace || workspace_bytes < rabit::svid_workspace_bytes(N, K, P)) return RABIT_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return RABIT_ERR_ALIGNMENT;
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    return finish_launch(rabit::launch_svid_init(ctx, W, ldw, N, K, P, T, power_iters, power_tol, s_in, s_out, alpha_in,
                                                 alpha_out, a, b, packed, workspace, fault, wait_timeout_ns(),
                                                 env_flag("RABIT_TEST_SVID_WITHHOLD_ARRIVAL") ? 1 : 0));
}

int rabit_read_fault(void *stream, uint32_t *flags, int clear) {
    rabit::LaunchCtx ctx;
    uint32_t *fault = nullptr;
    int st = device_ctx(stream, ctx, &fault);
    if (st != RABIT_OK) return st;
    cudaError_t e = cudaStreamSynchronize(ctx.stream);
    if (e != cudaSuccess) return cuda_fail(e);
    uint32_t v = 0;
    e = cudaMemcpy(&v, fault, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (clear) {
        e = cudaMemset(fault, 0, sizeof(uint32_t));
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return cuda_fail(e);
    }
    if (flags) *flags = v;
    return v ? RABIT_ERR_TIMEOUT : RABIT_OK;
}

int rabit_last_cuda_error(void) { return t_last_cuda_error; }

const char *rabit_status_string(int status) {
    switch (status) {
        case RABIT_OK: return "RABIT_OK";
        case RABIT_ERR_INVALID_ARG: return "RABIT_ERR_INVALID_ARG";
        case RABIT_ERR_ALIGNMENT: return "RABIT_ERR_ALIGNMENT";
        case RABIT_ERR_SHAPE: return "RABIT_ERR_SHAPE";
        case RABIT_ERR_UNSUPPORTED: return "RABIT_ERR_UNSUPPORTED";
        case RABIT_ERR_WORKSPACE: return "RABIT_ERR_WORKSPACE";
        case RABIT_ERR_ARCH: return "RABIT_ERR_ARCH";
        case RABIT_ERR_CUDA: return "RABIT_ERR_CUDA";
        case RABIT_ERR_TIMEOUT: return "RABIT_ERR_TIMEOUT";
        default: return "RABIT_ERR_UNKNOWN";
    }
}

}  // extern "C"
