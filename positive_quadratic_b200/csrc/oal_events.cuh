// oal_events.cuh -- the events one host-side call creates to order its streams.
#pragma once

#include <vector>

#include <cuda_runtime.h>

namespace oal {

// Events of one call, destroyed on every exit path (the runtime releases a destroyed event
// that is still pending once it completes).
struct CallEvents {
    std::vector<cudaEvent_t> ev;
    CallEvents() = default;
    CallEvents(const CallEvents&) = delete;
    CallEvents& operator=(const CallEvents&) = delete;
    ~CallEvents()
    {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
    }
    cudaError_t make(cudaEvent_t* out)
    {
        const cudaError_t e = cudaEventCreateWithFlags(out, cudaEventDisableTiming);
        if (e == cudaSuccess) ev.push_back(*out);
        return e;
    }
};

}  // namespace oal
