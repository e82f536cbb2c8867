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
//  * Residual pass, once per (t, i): a warp per 128 columns of a row (two such pieces in
//    flight) reads W, the other paths' packed words (broadcast loads) and the scales, writes
//    R (fp32, rows 16-byte aligned) and the signs straight into path i of the packed output
//    -- the same layout the decode and prefill kernels read.
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
// also resets the power launch's grid barrier.  A warp takes 128 columns of a row (four
// consecutive columns a lane, a float4 of W when its rows are 16-byte aligned) and two such
// pieces at a time, so enough of W is in flight to stream it; eight lanes make one 32-column
// sign word.
template <int kP, bool kVecW>
__global__ void __launch_bounds__(kThreads)
svid_residual_kernel(const float *__restrict__ W, int ldw, int N, int K, int Wr, int path,
                     uint32_t *__restrict__ packed, SvidWs w) {
    constexpr int G = kP == 2 ? 2 : 4;  // words per 32-column group in the packed layout
    pdl_enter();
    if (blockIdx.x == 0 && threadIdx.x < 2) w.sync[threadIdx.x] = 0u;
    const int lane = threadIdx.x & 31, sub = lane & 7, grp = lane >> 3;
    const int nblk = Wr / 4;                 // 128-column blocks per row (Wr is a multiple of 4)
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t units = static_cast<int64_t>(N) * nblk;
    const int64_t ldr = residual_pitch(K);
    for (int64_t u0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; u0 < units;
         u0 += 2 * nwarps) {
        float x[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {           // both pieces' loads go out first
            const int64_t u = u0 + h * nwarps;
            const int n = static_cast<int>(u / nblk);
            const int j = static_cast<int>(u - static_cast<int64_t>(n) * nblk) * 128 + 4 * lane;
            const float *src = W + static_cast<int64_t>(n) * ldw + j;
            if (u < units && kVecW && j + 3 < K) {
                const float4 v = __ldcs(reinterpret_cast<const float4 *>(src));
                x[h][0] = v.x; x[h][1] = v.y; x[h][2] = v.z; x[h][3] = v.w;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) x[h][q] = (u < units && j + q < K) ? __ldcs(src + q) : 0.0f;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t u = u0 + h * nwarps;
            if (u >= units) break;               // (warp-uniform)
            const int n = static_cast<int>(u / nblk);
            const int blk = static_cast<int>(u - static_cast<int64_t>(n) * nblk);
            const int j = blk * 128 + 4 * lane;
            const int64_t word = (static_cast<int64_t>(n) * Wr + blk * 4 + grp) * G;   // this lane's group
            const float so = w.so[n];
            uint32_t other[kP];
#pragma unroll
            for (int p = 0; p < kP; ++p) other[p] = p == path ? 0u : packed[word + p];
            float r[4];
            uint32_t nib = 0u;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                r[q] = 0.0f;
                if (j + q < K) {
                    float v = so * x[h][q] * w.si[j + q];
#pragma unroll
                    for (int p = 0; p < kP; ++p) {
                        if (p == path) continue;
                        const bool neg = (other[p] >> (4 * sub + q)) & 1u;
                        const float m = w.gp[p * static_cast<int64_t>(N) + n] * w.hp[p * static_cast<int64_t>(K) + j + q];
                        v = neg ? v + m : v - m;
                    }
                    r[q] = v;
                    nib |= (v < 0.0f ? 1u : 0u) << q;    // sign(v) = -1 iff v < 0
                }
            }
            if (j < K)                            // (the row pitch covers the whole float4)
                *reinterpret_cast<float4 *>(w.R + static_cast<int64_t>(n) * ldr + j) = make_float4(r[0], r[1], r[2], r[3]);
            uint32_t bits = nib << (4 * sub);     // the eight lanes of a group make its word
            bits |= __shfl_xor_sync(0xffffffffu, bits, 1);
            bits |= __shfl_xor_sync(0xffffffffu, bits, 2);
            bits |= __shfl_xor_sync(0xffffffffu, bits, 4);
            if (sub == 0) {
                packed[word + path] = bits;
                if (kP == 3 && path == 0) packed[word + 3] = 0u;                 // padding word
            }
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
        // The CTA's writes (ordered before this thread's by the CTA barrier) are released with
        // the arrival and acquired by every CTA that sees the count complete.
        if (!(p.debug == 1 && blockIdx.x == 0 && target == gridDim.x))
            asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&p.w.sync[0]) : "memory");
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
    const int64_t moved_off = 2 * kMaxPowGrid;     // slots [2], [3] of a parity: the moves
    bool v_from_acc = false;                   // current v: V, or v' / ||v'|| of the last step
    float ib_prev = 0.0f;
    unsigned target = 0;
    for (int s = 0; s < p.steps; ++s) {
        double usq = 0.0;                      // this thread's part of |u'|^2 (own rows)
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
                        t = cb == 0 ? t : w.uacc[nb + i] + t;   // same thread every sweep
                        w.uacc[nb + i] = t;
                        if (cb + kPowChunk >= K) usq += static_cast<double>(t) * t;
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
        // this step's per-CTA sums: [0] |u'|^2, [1] |v'|^2, [2] [3] the moves of the step before
        double *nsq = w.nsq + static_cast<int64_t>(s & 1) * 4 * kMaxPowGrid;
        usq = warp_sum(usq);
        if (lane == 0) red2[warp][0] = usq;
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int q = 0; q < kPowWarps; ++q) t += red2[q][0];
            nsq[c] = t;
        }
        target += static_cast<unsigned>(G);
        if (!grid_sync(p, target, &s_ok)) return;
        // ---- v'_j for this CTA's columns: the G partials added in CTA order (lane q mod 32
        // adds its CTAs in turn, then the tree), four columns per warp at a time
        double vsq = 0.0;                      // lane 0: this warp's part of |v'|^2
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
                if (lane == 0 && j < k1) {
                    w.vacc[j] = t;
                    vsq += static_cast<double>(t) * t;
                }
            }
        }
        if (lane == 0) red2[warp][1] = vsq;
        __syncthreads();
        if (tid == 0) {
            double t = 0.0;
            for (int q = 0; q < kPowWarps; ++q) t += red2[q][1];
            nsq[kMaxPowGrid + c] = t;
        }
        target += static_cast<unsigned>(G);
        if (!grid_sync(p, target, &s_ok)) return;
        // ---- norms (every CTA the same), then normalise or finish.  This thread's first row
        // and column are fetched while warp 0 adds the per-CTA sums.
        const int nf = r0 + tid, jf = k0 + tid;
        const float uf = nf < r1 ? w.uacc[nf] : 0.0f, uf_old = nf < r1 ? U[nf] : 0.0f;
        const float vf = jf < k1 ? w.vacc[jf] : 0.0f, vf_old = jf < k1 ? V[jf] : 0.0f;
        if (warp == 0) {
            double t[4];
            warp_totals<4>(nsq, G, lane, t);   // the moves were written before this step's barriers
            if (lane == 0) { nsh[0] = t[0]; nsh[1] = t[1]; nsh[2] = s > 0 ? t[2] : 0.0; nsh[3] = s > 0 ? t[3] : 0.0; }
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
            for (int n = nf; n < r1; n += kPowThreads) {
                const float u = (n == nf ? uf : w.uacc[n]) * ia;
                gp[n] = rs * u;
                if (na > 0.0) U[n] = u;
            }
            for (int j = jf; j < k1; j += kPowThreads) {
                const float v = (j == jf ? vf : w.vacc[j]) * ib;
                hp[j] = nb > 0.0 ? rs * v : 0.0f;
                if (nb > 0.0) V[j] = v;
            }
            return;
        }
        // A zero product keeps the old vector.  V is read by other CTAs only while the last
        // step's v' is zero, and then nobody writes it.  The squared moves of this CTA's
        // rows of u and columns of v go to the next step's decision (slots [2], [3] of the
        // next step's parity).
        double du = 0.0, dv = 0.0;
        if (na > 0.0)
            for (int n = nf; n < r1; n += kPowThreads) {
                const float u = (n == nf ? uf : w.uacc[n]) * ia, uo = n == nf ? uf_old : U[n];
                du += static_cast<double>(u - uo) * (u - uo);
                U[n] = u;
            }
        if (nb > 0.0)
            for (int j = jf; j < k1; j += kPowThreads) {
                const float v = (j == jf ? vf : w.vacc[j]) * ib, vo = j == jf ? vf_old : V[j];
                dv += static_cast<double>(v - vo) * (v - vo);
                V[j] = v;
            }
        du = warp_sum(du);
        dv = warp_sum(dv);
        if (lane == 0) { red2[warp][0] = du; red2[warp][1] = dv; }
        __syncthreads();
        if (tid == 0) {
            double su = 0.0, sv = 0.0;
            for (int q = 0; q < kPowWarps; ++q) { su += red2[q][0]; sv += red2[q][1]; }
            double *next = w.nsq + static_cast<int64_t>((s + 1) & 1) * 4 * kMaxPowGrid;
            next[moved_off + c] = su;
            next[moved_off + kMaxPowGrid + c] = sv;
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
    const int64_t warps = static_cast<int64_t>(N) * (Wr / 4);    // one per 128 columns of a row
    const int res_grid = static_cast<int>(std::min<int64_t>((warps * 32 + kThreads - 1) / kThreads,
                                                            static_cast<int64_t>(ctx.num_sms) * 16));
    const bool vec_w = reinterpret_cast<uintptr_t>(W) % 16 == 0 && ldw % 4 == 0;
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
            void (*res)(const float *, int, int, int, int, int, uint32_t *, SvidWs) =
                P == 2 ? (vec_w ? svid_residual_kernel<2, true> : svid_residual_kernel<2, false>)
                       : (vec_w ? svid_residual_kernel<3, true> : svid_residual_kernel<3, false>);
            e = launch(ctx, res_grid, kThreads, res, W, ldw, N, K, Wr, i, packed, w);
            if (e != cudaSuccess) break;
            pa.path = i;
            e = cudaLaunchKernelEx(&pcfg, svid_power_kernel, pa);
        }
    }
    if (e == cudaSuccess) e = launch(ctx, vec_grid, kThreads, svid_finish_kernel, N, K, P, a, b, w);
    return e;
}

}  // namespace rabit
