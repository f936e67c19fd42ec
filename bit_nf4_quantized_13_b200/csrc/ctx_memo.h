// ctx_memo.h -- host-side memo of per-context set-up results.
//
// Several launchers do one-time set-up before their first launch: raising a
// kernel's dynamic shared-memory limit, asking the occupancy calculator,
// looking up the device address of a __device__ array.  Those results belong
// to a CUDA context, not to the process or the device ordinal: after the
// context is destroyed and made again (cudaDeviceReset, or a host program
// that resets the device between phases) the module is loaded afresh, its
// function attributes are back at their defaults and its __device__ arrays
// may sit at other addresses.  The memo is therefore keyed on the context's
// process-unique id (cuCtxGetId), which the driver never hands out twice in
// one process, unlike the context handle whose value can be reused.
//
// Plain C++ with no CUDA dependency, so the host tests can compile it alone.
#pragma once

#include <stdint.h>

#include <mutex>

namespace qlora {

template <typename T, int kSlots = 16>
class ContextMemo {
public:
    // The value stored for context `ctx_id`, computing it with
    // fill(T* out) -> bool the first time the id is seen.  A failed fill
    // stores nothing (the next call tries again) and returns false.  When
    // all slots are taken the oldest entry is replaced.
    template <typename F>
    bool get(uint64_t ctx_id, T* out, F&& fill) {
        std::lock_guard<std::mutex> lock(mu_);
        for (int i = 0; i < used_; ++i) {
            if (ids_[i] == ctx_id) {
                *out = vals_[i];
                return true;
            }
        }
        T v{};
        if (!fill(&v)) return false;
        int slot;
        if (used_ < kSlots) {
            slot = used_++;
        } else {
            slot = next_evict_;
            next_evict_ = (next_evict_ + 1) % kSlots;
        }
        ids_[slot] = ctx_id;
        vals_[slot] = v;
        *out = v;
        return true;
    }

    int size() {
        std::lock_guard<std::mutex> lock(mu_);
        return used_;
    }

private:
    std::mutex mu_;
    uint64_t ids_[kSlots] = {};
    T vals_[kSlots] = {};
    int used_ = 0;
    int next_evict_ = 0;
};

// The process-unique id of the calling thread's current CUDA context (made
// current first if the runtime has not yet done so for the current device).
// Returns false if there is no usable context.  Defined in ctx_id.cu.
bool current_context_id(uint64_t* id);

}  // namespace qlora
