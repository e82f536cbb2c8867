// svid.cu -- initialisation of the residual-binary layer: Iterative Residual SVID on the
// importance-preconditioned weight.
//
// "RaBiT: Residual-Aware Binarization Training for Accurate and Efficient LLMs", sec. 4.3
// "Stable Initialization for Functional Preservation":
//     W' = s_out^alpha_out (.) W (.) s_in^alpha_in
//     for t = 1..T, paths i = 1..P in order:
//         R_i = W' - sum_{j != i} What_j        (the latest update of every other path)
//         (B_i, g_i', h_i') = SVID(R_i),   What_i = g_i' (.) B_i (.) h_i'
//     g_i = s_out^-alpha_out (.) g_i',   h_i = s_in^-alpha_in (.) h_i'
// with What_j = 0 before a path's first update (iteration 1 is the greedy decomposition).
// SVID(R) = (sign R, g', h'), g' h'^T the leading rank-1 part sigma u v^T of |R| split as
// sqrt(sigma) u, sqrt(sigma) v; the pages leave SVID to the cited prior work, whose
// sign-value-independent decomposition this is.
//
// Design (HBM-bound passes, CUDA cores):
//  * Residual pass, once per (t, i): a warp per 32-column group reads the group's W values
//    (128 contiguous bytes), the other paths' packed words (one broadcast load each) and
//    scales, writes R (fp32, rows 16-byte aligned) and a ballot of the signs straight into
//    path i of the packed output -- the same layout the decode and prefill kernels read.
//  * Power iteration for (sigma, u, v), warm-started from the path's vectors of the previous
//    iteration, in ONE cooperative launch per (t, i) that runs every power step.  A step is
//    one pass over R that yields both u' = |R| v and v' = |R|^T u (|R| from R itself): CTA c
//    owns a block of rows, so each u'_n is a CTA reduction, and writes its column partial
//    sums of |R_nj| u_n; after a grid barrier CTA c adds the G partials of its slice of
//    columns (in CTA order) into v'; after a second barrier every CTA forms ||u'|| and ||v'||
//    from the per-CTA squares (in CTA order), so all CTAs take the same decisions: normalise
//    (own rows of u, own columns of v), stop when the steps are spent or when u and v moved
//    by at most the caller's tolerance in the step before, and on the last step write
//    g' = sqrt(sigma) u, h' = sqrt(sigma) v.  Every sum has a fixed order (deterministic).
//  * u and v start positive and |R| is nonnegative, so they stay the Perron vectors.
#include <algorithm>
#include <cmath>

#include "rabit_device.cuh"
#include "rabit_kernels.h"

namespace rabit {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void pdl_enter() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}

constexpr int kPowThreads = 512;
constexpr int kPowWarps = kPowThreads / 32;
constexpr int kPowVec = 2;                              // float4 columns per thread per row
constexpr int kPowChunk = kPowThreads * 4 * kPowVec;     // columns of one sweep over the rows
constexpr int kPowRows = 8;                             // rows in flight per thread
constexpr int kPowFlush = 256;                          // row dots held per warp before adding
constexpr int kMaxPowGrid = 160;                        // CTAs of the power launch, at most

// Workspace carve-up (every part 256-byte aligned).
struct SvidWs {
    float *R;          // [N][ldr] residual of the path being updated
    float *so, *si;    // s_out^alpha_out [N], s_in^alpha_in [K]
    float *gp, *hp;    // g' [P][N], h' [P][K] in the preconditioned domain
    float *U, *V;      // unit singular vectors per path [P][N], [P][K] (warm starts)
    float *uacc, *vacc;      // u' [N], v' [K] of the current power step
    float *part;             // [kMaxPowGrid][ldr] per-CTA column partial sums
    double *nsq;             // [2][4][kMaxPowGrid] per-CTA sums by step parity: |u'|^2, |v'|^2,
                             // |u - u_prev|^2, |v - v_prev|^2
    unsigned *sync;          // [0] grid-barrier counter, [1] abort flag (zeroed by the residual pass)
    size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

__host__ __device__ inline int64_t residual_pitch(int K) { return (static_cast<int64_t>(K) + 3) / 4 * 4; }

SvidWs svid_layout(void *base, int N, int K, int P) {
    SvidWs w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return reinterpret_cast<char *>(reinterpret_cast<uintptr_t>(base) + o);
    };
    w.R = reinterpret_cast<float *>(take(static_cast<size_t>(N) * residual_pitch(K) * 4));
    w.so = reinterpret_cast<float *>(take(static_cast<size_t>(N) * 4));
    w.si = reinterpret_cast<float *>(take(static_cast<size_t>(K) * 4));
    w.gp = reinterpret_cast<float *>(take(static_cast<size_t>(P) * N * 4));
    w.hp = reinterpret_cast<float *>(take(static_cast<size_t>(P) * K * 4));
    w.U = reinterpret_cast<float *>(take(static_cast<size_t>(P) * N * 4));
    w.V = reinterpret_cast<float *>(take(static_cast<size_t>(P) * K * 4));
    w.uacc = reinterpret_cast<float *>(take(static_cast<size_t>(N) * 4));
    w.vacc = reinterpret_cast<float *>(take(static_cast<size_t>(K) * 4));
    w.part = reinterpret_cast<float *>(take(static_cast<size_t>(kMaxPowGrid) * residual_pitch(K) * 4));
    w.nsq = reinterpret_cast<double *>(take(static_cast<size_t>(8) * kMaxPowGrid * 8));
    w.sync = reinterpret_cast<unsigned *>(take(2 * sizeof(unsigned)));
    w.total = off;
    return w;
}

// Preconditioning vectors, zero scales, uniform unit start vectors.
__global__ void __launch_bounds__(kThreads)
svid_prep_kernel(const float *__restrict__ s_in, const float *__restrict__ s_out, float alpha_in,
                 float alpha_out, int N, int K, int P, SvidWs w) {
    pdl_enter();
    const float un = 1.0f / sqrtf(static_cast<float>(N)), vk = 1.0f / sqrtf(static_cast<float>(K));
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < N; t += stride) {
        w.so[t] = powf(__ldg(s_out + t), alpha_out);
        for (int p = 0; p < P; ++p) {
            w.gp[p * static_cast<int64_t>(N) + t] = 0.0f;
            w.U[p * static_cast<int64_t>(N) + t] = un;
        }
    }
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < K; t += stride) {
        w.si[t] = powf(__ldg(s_in + t), alpha_in);
        for (int p = 0; p < P; ++p) {
            w.hp[p * static_cast<int64_t>(K) + t] = 0.0f;
            w.V[p * static_cast<int64_t>(K) + t] = vk;
        }
    }
}

// R_i = W' - sum_{p != i} g_p' (.) B_p (.) h_p', its signs into path i of the packed output;
// also resets the power launch's grid barrier.
template <int kP>
__global__ void __launch_bounds__(kThreads)
svid_residual_kernel(const float *__restrict__ W, int ldw, int N, int K, int Wr, int path,
                     uint32_t *__restrict__ packed, SvidWs w) {
    constexpr int G = kP == 2 ? 2 : 4;  // words per 32-column group in the packed layout
    pdl_enter();
    if (blockIdx.x == 0 && threadIdx.x < 2) w.sync[threadIdx.x] = 0u;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t groups = static_cast<int64_t>(N) * Wr;
    const int64_t ldr = residual_pitch(K);
    for (int64_t gi = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; gi < groups;
         gi += nwarps) {
        const int n = static_cast<int>(gi / Wr);
        const int j = static_cast<int>(gi - static_cast<int64_t>(n) * Wr) * 32 + lane;
        const bool ok = j < K;
        float r = 0.0f;
        if (ok) {
            r = w.so[n] * __ldg(W + static_cast<int64_t>(n) * ldw + j) * w.si[j];
#pragma unroll
            for (int p = 0; p < kP; ++p) {
                if (p == path) continue;
                const bool neg = (packed[gi * G + p] >> lane) & 1u;
                const float m = w.gp[p * static_cast<int64_t>(N) + n] * w.hp[p * static_cast<int64_t>(K) + j];
                r = neg ? r + m : r - m;
            }
            w.R[static_cast<int64_t>(n) * ldr + j] = r;
        }
        const uint32_t bits = __ballot_sync(0xffffffffu, ok && r < 0.0f);   // sign(v) = -1 iff v < 0
        if (lane == 0) {
            packed[gi * G + path] = bits;
            if (kP == 3 && path == 0) packed[gi * G + 3] = 0u;                 // padding word
        }
    }
}

// Sum over the lanes of a warp in a fixed tree (the same result in every lane).
template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// sum_i x[i]^2 over [0, n) in a fixed order (lane-strided, then the tree), by one warp.
__device__ __forceinline__ double warp_sumsq(const float *x, int n, int lane) {
    double s = 0.0;
    for (int i = lane; i < n; i += 32) s += static_cast<double>(x[i]) * x[i];
    return warp_sum(s);
}

constexpr int kPerLane = (kMaxPowGrid + 31) / 32;      // per-CTA values a lane adds up

// sum_c x[r][c] over c in [0, G) for kR rows of stride kMaxPowGrid, in a fixed order (lane c
// mod 32 adds its values in turn, then the tree), by one warp; every load is issued first.
template <int kR>
__device__ __forceinline__ void warp_totals(const double *x, int G, int lane, double (&out)[kR]) {
    double v[kR][kPerLane];
#pragma unroll
    for (int r = 0; r < kR; ++r)
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
            const int c = lane + 32 * i;
            v[r][i] = c < G ? x[r * kMaxPowGrid + c] : 0.0;
        }
#pragma unroll
    for (int r = 0; r < kR; ++r) {
        double t = 0.0;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) t += v[r][i];
        out[r] = warp_sum(t);
    }
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

struct PowerArgs {
    const float *R;
    int64_t ldr;
    int N, K, path, steps;
    float tol;
    SvidWs w;
    uint32_t *fault;
    uint64_t timeout_ns;
    int debug;                                 // 1: CTA 0 withholds its first arrival (test switch)
};

// Grid barrier of the cooperative power launch: the counter reaches `target` when every CTA
// has arrived.  The wait is bounded; when it expires (or another CTA gave up) the fault bit
// and the abort flag are set and every CTA leaves the kernel.
__device__ bool grid_sync(const PowerArgs &p, unsigned target, int *s_ok) {
    __syncthreads();
    if (threadIdx.x == 0) {
        bool ok = true;
        __threadfence();                       // this CTA's writes before its arrival
        if (!(p.debug == 1 && blockIdx.x == 0 && target == gridDim.x)) atomicAdd(&p.w.sync[0], 1u);
        if (ld_acquire_gpu(&p.w.sync[0]) < target) {
            const uint64_t t0 = global_timer_ns();
            while (ld_acquire_gpu(&p.w.sync[0]) < target) {
                if (*reinterpret_cast<volatile unsigned *>(&p.w.sync[1])) { ok = false; break; }
                if (global_timer_ns() - t0 > p.timeout_ns) {
                    atomicOr(p.fault, FAULT_SVID_BARRIER);
                    atomicExch(&p.w.sync[1], 1u);
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        __threadfence();
        *s_ok = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_ok != 0;
}

// Every power step of one (t, i) update, one CTA per SM (cooperative launch).
__global__ void __launch_bounds__(kPowThreads, 1)
svid_power_kernel(const __grid_constant__ PowerArgs p) {
    __shared__ float red[kPowWarps][kPowFlush];   // per-warp parts of the row dots
    __shared__ double nsh[4];
    __shared__ double red2[kPowWarps][2];
    __shared__ int s_ok;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x, G = gridDim.x, N = p.N, K = p.K;
    const int r0 = static_cast<int>(static_cast<int64_t>(N) * c / G);
    const int r1 = static_cast<int>(static_cast<int64_t>(N) * (c + 1) / G);
    const int k0 = static_cast<int>(static_cast<int64_t>(K) * c / G);
    const int k1 = static_cast<int>(static_cast<int64_t>(K) * (c + 1) / G);
    const SvidWs &w = p.w;
    float *U = w.U + p.path * static_cast<int64_t>(N), *V = w.V + p.path * static_cast<int64_t>(K);
    float *part = w.part + static_cast<int64_t>(c) * p.ldr;
    bool v_from_acc = false;                   // current v: V, or v' / ||v'|| of the last step
    float ib_prev = 0.0f;
    unsigned target = 0;
    for (int s = 0; s < p.steps; ++s) {
        // ---- pass over the CTA's rows: u'_n = sum_j |R_nj| v_j, column partials sum_n |R_nj| u_n
        for (int cb = 0; cb < K; cb += kPowChunk) {
            float4 vv[kPowVec], cp[kPowVec];
#pragma unroll
            for (int m = 0; m < kPowVec; ++m) {
                const int j = cb + 4 * (tid + kPowThreads * m);
                float e[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    e[q] = j + q < K ? (v_from_acc ? w.vacc[j + q] * ib_prev : V[j + q]) : 0.0f;
                vv[m] = make_float4(e[0], e[1], e[2], e[3]);
                cp[m] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
            for (int n0 = r0; n0 < r1; n0 += kPowRows) {
                float4 x[kPowRows][kPowVec];
                float un[kPowRows], d[kPowRows];
#pragma unroll
                for (int i = 0; i < kPowRows; ++i) {
                    const bool row_ok = n0 + i < r1;
                    un[i] = row_ok ? U[n0 + i] : 0.0f;
#pragma unroll
                    for (int m = 0; m < kPowVec; ++m) {
                        const int j = cb + 4 * (tid + kPowThreads * m);
                        x[i][m] = (row_ok && j < K)
                                      ? __ldcg(reinterpret_cast<const float4 *>(p.R + (n0 + i) * p.ldr + j))
                                      : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                        if (j + 3 >= K) {              // columns past K (row padding) are not data
                            if (j + 1 >= K) x[i][m].y = 0.0f;
                            if (j + 2 >= K) x[i][m].z = 0.0f;
                            if (j + 3 >= K) x[i][m].w = 0.0f;
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < kPowRows; ++i) {
                    float acc = 0.0f;
#pragma unroll
                    for (int m = 0; m < kPowVec; ++m) {
                        const float4 a = make_float4(fabsf(x[i][m].x), fabsf(x[i][m].y), fabsf(x[i][m].z),
                                                     fabsf(x[i][m].w));
                        acc = fmaf(a.x, vv[m].x, acc);
                        acc = fmaf(a.y, vv[m].y, acc);
                        acc = fmaf(a.z, vv[m].z, acc);
                        acc = fmaf(a.w, vv[m].w, acc);
                        cp[m].x = fmaf(a.x, un[i], cp[m].x);
                        cp[m].y = fmaf(a.y, un[i], cp[m].y);
                        cp[m].z = fmaf(a.z, un[i], cp[m].z);
                        cp[m].w = fmaf(a.w, un[i], cp[m].w);
                    }
                    d[i] = warp_sum(acc);
                }
                // Each warp's part of the row dots waits in shared memory; every kPowFlush rows
                // (and at the end of the sweep) the CTA adds them up, warp 0's part first.
                const int slot = (n0 - r0) % kPowFlush;
                if (lane == 0) {
#pragma unroll
                    for (int i = 0; i < kPowRows; ++i) red[warp][slot + i] = d[i];
                }
                if (slot + kPowRows == kPowFlush || n0 + kPowRows >= r1) {
                    const int nb = n0 - slot;          // first row of the rows held
                    const int nr = min(kPowFlush, r1 - nb);
                    __syncthreads();
                    for (int i = tid; i < nr; i += kPowThreads) {
                        float t = 0.0f;
#pragma unroll
                        for (int q = 0; q < kPowWarps; ++q) t += red[q][i];
                        w.uacc[nb + i] = cb == 0 ? t : w.uacc[nb + i] + t;   // same thread every sweep
                    }
                    __syncthreads();
                }
            }
#pragma unroll
            for (int m = 0; m < kPowVec; ++m) {
                const int j = cb + 4 * (tid + kPowThreads * m);
                if (j < K) *reinterpret_cast<float4 *>(part + j) = cp[m];   // (part pitch = ldr)
            }
        }
        double *nsq = w.nsq + static_cast<int64_t>(s & 1) * 4 * kMaxPowGrid;   // this step's sums
        const double *moved = w.nsq + static_cast<int64_t>((s + 1) & 1) * 4 * kMaxPowGrid + 2 * kMaxPowGrid;
        __syncthreads();
        if (warp == 0) {
            const double t = warp_sumsq(w.uacc + r0, r1 - r0, lane);
            if (lane == 0) nsq[c] = t;
        }
        target += static_cast<unsigned>(G);
        if (!grid_sync(p, target, &s_ok)) return;
        // ---- v'_j for this CTA's columns: the G partials added in CTA order (lane q mod 32
        // adds its CTAs in turn, then the tree), four columns per warp at a time
        for (int jb = k0 + warp; jb < k1; jb += 4 * kPowWarps) {
            float v[4][kPerLane];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int i = 0; i < kPerLane; ++i) {
                    const int j = jb + u * kPowWarps, q = lane + 32 * i;
                    v[u][i] = (j < k1 && q < G) ? w.part[static_cast<int64_t>(q) * p.ldr + j] : 0.0f;
                }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float t = 0.0f;
#pragma unroll
                for (int i = 0; i < kPerLane; ++i) t += v[u][i];
                t = warp_sum(t);
                const int j = jb + u * kPowWarps;
                if (lane == 0 && j < k1) w.vacc[j] = t;
            }
        }
        __syncthreads();
        if (warp == 0) {
            const double t = warp_sumsq(w.vacc + k0, k1 - k0, lane);
            if (lane == 0) nsq[kMaxPowGrid + c] = t;
        }
        target += static_cast<unsigned>(G);
        if (!grid_sync(p, target, &s_ok)) return;
        // ---- norms (every CTA the same), then normalise or finish
        if (warp == 0) {
            double t[2], m[2] = {0.0, 0.0};
            warp_totals<2>(nsq, G, lane, t);
            // how far u and v moved in the previous step (written before this step's barriers)
            if (s > 0) warp_totals<2>(moved, G, lane, m);
            if (lane == 0) { nsh[0] = t[0]; nsh[1] = t[1]; nsh[2] = m[0]; nsh[3] = m[1]; }
        }
        __syncthreads();
        const double na = sqrt(nsh[0]), nb = sqrt(nsh[1]);
        const float ia = na > 0.0 ? static_cast<float>(1.0 / na) : 0.0f;
        const float ib = nb > 0.0 ? static_cast<float>(1.0 / nb) : 0.0f;
        const double tol2 = static_cast<double>(p.tol) * p.tol;
        const bool settled = p.tol > 0.0f && s > 0 && nsh[2] <= tol2 && nsh[3] <= tol2;
        if (s == p.steps - 1 || settled) {
            const float rs = static_cast<float>(sqrt(na));    // sqrt(sigma)
            float *gp = w.gp + p.path * static_cast<int64_t>(N), *hp = w.hp + p.path * static_cast<int64_t>(K);
            for (int n = r0 + tid; n < r1; n += kPowThreads) {
                const float u = w.uacc[n] * ia;
                gp[n] = rs * u;
                if (na > 0.0) U[n] = u;
            }
            for (int j = k0 + tid; j < k1; j += kPowThreads) {
                const float v = w.vacc[j] * ib;
                hp[j] = nb > 0.0 ? rs * v : 0.0f;
                if (nb > 0.0) V[j] = v;
            }
            return;
        }
        // A zero product keeps the old vector.  V is read by other CTAs only while the last
        // step's v' is zero, and then nobody writes it.  The squared moves of this CTA's
        // rows of u and columns of v go to the next step's decision.
        double du = 0.0, dv = 0.0;
        if (na > 0.0)
            for (int n = r0 + tid; n < r1; n += kPowThreads) {
                const float u = w.uacc[n] * ia;
                du += static_cast<double>(u - U[n]) * (u - U[n]);
                U[n] = u;
            }
        if (nb > 0.0)
            for (int j = k0 + tid; j < k1; j += kPowThreads) {
                const float v = w.vacc[j] * ib;
                dv += static_cast<double>(v - V[j]) * (v - V[j]);
                V[j] = v;
            }
        du = warp_sum(du);
        dv = warp_sum(dv);
        if (lane == 0) { red2[warp][0] = du; red2[warp][1] = dv; }
        __syncthreads();
        if (tid == 0) {
            double su = 0.0, sv = 0.0;
            for (int q = 0; q < kPowWarps; ++q) { su += red2[q][0]; sv += red2[q][1]; }
            nsq[2 * kMaxPowGrid + c] = su;
            nsq[3 * kMaxPowGrid + c] = sv;
        }
        v_from_acc = nb > 0.0;
        if (v_from_acc) ib_prev = ib;
        __syncthreads();                       // this CTA's u before the next pass reads it
    }
}

// Scales mapped back to the original domain: a_p = g_p' / s_out^alpha_out, b_p = h_p' / s_in^alpha_in.
__global__ void __launch_bounds__(kThreads)
svid_finish_kernel(int N, int K, int P, float *__restrict__ a, float *__restrict__ b, SvidWs w) {
    pdl_enter();
    const int stride = gridDim.x * blockDim.x;
    for (int p = 0; p < P; ++p) {
        for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < N; n += stride)
            a[p * static_cast<int64_t>(N) + n] = w.gp[p * static_cast<int64_t>(N) + n] / w.so[n];
        for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < K; j += stride)
            b[p * static_cast<int64_t>(K) + j] = w.hp[p * static_cast<int64_t>(K) + j] / w.si[j];
    }
}

template <typename... KArgs, typename... Args>
cudaError_t launch(const LaunchCtx &ctx, int grid, int block, void (*kern)(KArgs...), Args... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ctx.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(block));
    cfg.stream = ctx.stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

size_t svid_workspace_bytes(int N, int K, int P) { return svid_layout(nullptr, N, K, P).total; }

cudaError_t launch_svid_init(const LaunchCtx &ctx, const float *W, int ldw, int N, int K, int P, int T,
                             int power_iters, float power_tol, const float *s_in, const float *s_out,
                             float alpha_in, float alpha_out, float *a, float *b, uint32_t *packed,
                             void *workspace, uint32_t *fault_word, uint64_t timeout_ns, int debug) {
    if ((P != 2 && P != 3) || T < 1 || power_iters < 1) return cudaErrorInvalidValue;
    const SvidWs w = svid_layout(workspace, N, K, P);
    const int Wr = static_cast<int>(padded_cols(K) / 32);
    const int64_t vec_len = std::max<int64_t>(N, K);
    const int vec_grid = static_cast<int>(std::min<int64_t>((vec_len + kThreads - 1) / kThreads, ctx.num_sms * 4));
    const int64_t warps = static_cast<int64_t>(N) * Wr;
    const int res_grid = static_cast<int>(std::min<int64_t>((warps * 32 + kThreads - 1) / kThreads,
                                                            static_cast<int64_t>(ctx.num_sms) * 16));
    // The power launch's CTAs wait on one another, so all must be resident: one per SM.
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, svid_power_kernel, kPowThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    const int pow_grid = std::min(ctx.num_sms, kMaxPowGrid);
    PowerArgs pa{};
    pa.ldr = residual_pitch(K);
    pa.R = w.R;
    pa.N = N;
    pa.K = K;
    pa.steps = power_iters;
    pa.tol = power_tol;
    pa.w = w;
    pa.fault = fault_word;
    pa.timeout_ns = timeout_ns;
    pa.debug = debug;
    cudaLaunchAttribute coop[1];
    coop[0].id = cudaLaunchAttributeCooperative;
    coop[0].val.cooperative = 1;
    cudaLaunchConfig_t pcfg = {};
    pcfg.gridDim = dim3(static_cast<unsigned>(pow_grid));
    pcfg.blockDim = dim3(kPowThreads);
    pcfg.stream = ctx.stream;
    pcfg.attrs = coop;
    pcfg.numAttrs = 1;
    e = launch(ctx, vec_grid, kThreads, svid_prep_kernel, s_in, s_out, alpha_in, alpha_out, N, K, P, w);
    for (int t = 0; t < T && e == cudaSuccess; ++t) {
        for (int i = 0; i < P && e == cudaSuccess; ++i) {
            e = P == 2 ? launch(ctx, res_grid, kThreads, svid_residual_kernel<2>, W, ldw, N, K, Wr, i, packed, w)
                       : launch(ctx, res_grid, kThreads, svid_residual_kernel<3>, W, ldw, N, K, Wr, i, packed, w);
            if (e != cudaSuccess) break;
            pa.path = i;
            e = cudaLaunchKernelEx(&pcfg, svid_power_kernel, pa);
        }
    }
    if (e == cudaSuccess) e = launch(ctx, vec_grid, kThreads, svid_finish_kernel, N, K, P, a, b, w);
    return e;
}

}  // namespace rabit
