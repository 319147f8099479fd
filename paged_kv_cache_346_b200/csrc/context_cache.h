// Host-side values that belong to one CUDA context: device addresses of the
// library's __device__ variables, and which kernels have had their dynamic
// shared-memory limit raised.  They are cached per context, keyed by the
// context's unique id (cuCtxGetId), not by device ordinal: after
// cudaDeviceReset, or with another context made current on the same device,
// the module is loaded anew and an address cached for the old context would
// name memory that is no longer the variable.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace pkv {

// Unique id of the calling thread's current context; 0 when none is current
// (the runtime has not yet initialised one on this thread).
cudaError_t current_context_id(unsigned long long* id);

// A small map context id -> pointer-sized value.  Lookups and inserts take a
// mutex (uncontended: tens of nanoseconds).  When full, the oldest entry is
// replaced: a forgotten context only costs one more lookup.
class PerContext {
   public:
    bool find(unsigned long long id, void** value) {
        if (id == 0) return false;
        std::lock_guard<std::mutex> g(mu_);
        for (int i = 0; i < n_; ++i)
            if (e_[i].id == id) {
                *value = e_[i].value;
                return true;
            }
        return false;
    }
    void put(unsigned long long id, void* value) {
        if (id == 0) return;
        std::lock_guard<std::mutex> g(mu_);
        for (int i = 0; i < n_; ++i)
            if (e_[i].id == id) {
                e_[i].value = value;
                return;
            }
        if (n_ < kSlots) {
            e_[n_++] = {id, value};
        } else {
            e_[next_] = {id, value};
            next_ = (next_ + 1) % kSlots;
        }
    }

   private:
    static constexpr int kSlots = 16;
    struct Entry {
        unsigned long long id;
        void* value;
    };
    std::mutex mu_;
    Entry e_[kSlots] = {};
    int n_ = 0, next_ = 0;
};

// The value for the current context, computed by `make` (which may initialise
// the context) when it is not cached yet.
template <typename F>
cudaError_t per_context_value(PerContext& cache, void** out, F make) {
    unsigned long long id = 0;
    cudaError_t e = current_context_id(&id);
    if (e != cudaSuccess) return e;
    if (cache.find(id, out)) return cudaSuccess;
    e = make(out);
    if (e != cudaSuccess) return e;
    if (id == 0 && current_context_id(&id) != cudaSuccess) id = 0;
    cache.put(id, *out);
    return cudaSuccess;
}

}  // namespace pkv
