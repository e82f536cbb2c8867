// ctx_cache.h -- per-device values that stay valid only for one CUDA context.
//
// A device address of a `__device__` symbol, or a function attribute set with
// cudaFuncSetAttribute, belongs to the context the module was loaded in.  After the
// primary context is reset (cudaDeviceReset, or a driver-level reset of the primary
// context) the next runtime call creates a new context, the library's module is loaded
// again, and the symbol may move.  These caches therefore key every entry on the unique
// id of the context it was filled in (cuCtxGetId) and refill an entry whose id differs
// from the calling thread's current context.
//
// Header-only and free of CUDA includes, so the host test suite can compile it with a
// plain C++ compiler and drive it with fake context ids.
#pragma once

#include <atomic>
#include <cstdint>
#include <mutex>

namespace rabit {

constexpr int kCtxCacheDevices = 64;

// One value per device, refilled when the context id changes.  Every access takes the
// mutex: the calls that use it are microseconds long, and a lock-free reader could pair
// one context's id with another context's value.
template <typename T>
class ContextCache {
public:
    // Returns fill()'s status (0 = success) and sets *out.  `ctx` is the id of the
    // context current on the calling thread; 0 means it could not be read, which never
    // matches a stored id, so such a call always refills.  fill(T*) computes the value in
    // the current context; a failed fill leaves the entry empty.
    template <typename Fill>
    int get(int dev, uint64_t ctx, Fill fill, T *out) {
        if (dev < 0 || dev >= kCtxCacheDevices) return fill(out);
        std::lock_guard<std::mutex> lock(mutex_);
        if (ctx != 0 && ctx_[dev] == ctx) {
            *out = value_[dev];
            return 0;
        }
        T v{};
        const int st = fill(&v);
        if (st != 0) {
            ctx_[dev] = 0;
            return st;
        }
        value_[dev] = v;
        ctx_[dev] = ctx;
        ++fills_;
        *out = v;
        return 0;
    }

    // Number of successful fills so far (for tests).
    long fills() {
        std::lock_guard<std::mutex> lock(mutex_);
        return fills_;
    }

private:
    std::mutex mutex_;
    uint64_t ctx_[kCtxCacheDevices] = {};
    T value_[kCtxCacheDevices] = {};
    long fills_ = 0;
};

// Records, per device, the context in which a one-time per-context setting (such as a
// kernel's dynamic shared-memory opt-in) was made.  Two threads making the first call at
// once may both make the setting, which is harmless.
class ContextFlags {
public:
    bool done(int dev, uint64_t ctx) const {
        return ctx != 0 && dev >= 0 && dev < kCtxCacheDevices &&
               ctx_[dev].load(std::memory_order_acquire) == ctx;
    }
    void mark(int dev, uint64_t ctx) {
        if (dev >= 0 && dev < kCtxCacheDevices) ctx_[dev].store(ctx, std::memory_order_release);
    }

private:
    std::atomic<uint64_t> ctx_[kCtxCacheDevices] = {};
};

}  // namespace rabit
